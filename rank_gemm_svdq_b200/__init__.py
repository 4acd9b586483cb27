"""Python binding of libsvdq (the SVDQuant W4A4 linear layer for B200, sm_100a).

Argument marshalling only: every step of the layer runs in the C ABI library
(`include/svdq.h`); this module converts numpy arrays / torch tensors to raw
pointers and sizes.  PyTorch supplies device memory and streams.

The library is built in-tree (`rank_gemm_svdq_b200/libsvdq.so`, see build.py).
Importing this module raises if it is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_BLOB, \
    ERR_NO_CONVERGENCE, ERR_CUDA, ERR_TIMEOUT = range(9)
INT4_G64, NVFP4 = 1, 2
F16, BF16 = 1, 2
FMT = {"int4": INT4_G64, "nvfp4": NVFP4}
DTYPE = {"fp16": F16, "bf16": BF16}


class svdq_params(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int32), ("N", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("fmt", ctypes.c_int32), ("act_dtype", ctypes.c_int32), ("smooth", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("reserved", ctypes.c_int32)]


class SVDQError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = f"{what}: {status_string(status)} ({status})" if what else status_string(status)
        if status == ERR_CUDA:
            msg += f" [{_lib.svdq_last_error_string().decode()}]"
        super().__init__(msg)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsvdq.so not built at {LIB_PATH}; run rank_gemm_svdq_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(svdq_params)
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "svdq_blob_bytes": (sz, [P]),
        "svdq_prepare": (ctypes.c_int, [P, vp, vp, vp, i64, vp, sz, vp]),
        "svdq_blob_check": (ctypes.c_int, [P, vp, sz]),
        "svdq_blob_export": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp]),
        "svdq_append_lora": (ctypes.c_int, [P, vp, sz, vp, vp, ctypes.c_int32, P, vp, sz]),
        "svdq_shard_columns": (ctypes.c_int, [P, vp, sz, ctypes.c_int32, ctypes.c_int32, P, vp, sz]),
        "svdq_kv_workspace_bytes": (sz, [i64, ctypes.c_int32]),
        "svdq_kv_encode": (ctypes.c_int, [vp, i64, ctypes.c_int32, ctypes.c_int32, vp, vp, vp, vp, sz, vp]),
        "svdq_kv_decode": (ctypes.c_int, [vp, vp, vp, i64, ctypes.c_int32, ctypes.c_int32, vp, vp]),
        "svdq_kv_attention_workspace_bytes": (sz, [i64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]),
        "svdq_kv_attention": (ctypes.c_int, [vp, ctypes.c_int32, vp, vp, vp, vp, vp, vp, i64, ctypes.c_int32,
                                             ctypes.c_int32, ctypes.c_int32, vp, vp, sz, vp]),
        "svdq_workspace_bytes": (sz, [P, i64]),
        "svdq_linear": (ctypes.c_int, [P, vp, vp, i64, vp, vp, sz, vp]),
        "svdq_quantize_act": (ctypes.c_int, [P, vp, vp, i64, vp, sz, vp]),
        "svdq_gemm": (ctypes.c_int, [P, vp, i64, vp, vp, sz, vp]),
        "svdq_chain_workspace_bytes": (sz, [P, P, i64]),
        "svdq_gemm_chain": (ctypes.c_int, [P, vp, i64, P, vp, vp, sz, vp, sz, vp]),
        "svdq_export_act": (ctypes.c_int, [P, vp, i64, vp, vp, vp, vp]),
        "svdq_get_status": (ctypes.c_int, [vp]),
        "svdq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "svdq_last_error_string": (ctypes.c_char_p, []),
        "svdq_probe_cvt": (ctypes.c_int, [vp, i64, vp, vp, vp]),
        "svdq_probe_div": (ctypes.c_int, [vp, vp, i64, vp, vp, vp]),
        "svdq_probe_tc": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]),
        "svdq_linear_noalloc": (ctypes.c_int, [P, vp, vp, i64, vp, vp]),
        "svdq_probe_timeout": (ctypes.c_int, [i64, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib = _load()
EXPORTED = ("svdq_blob_bytes", "svdq_prepare", "svdq_blob_check", "svdq_blob_export", "svdq_append_lora", "svdq_shard_columns",
            "svdq_workspace_bytes", "svdq_linear", "svdq_quantize_act", "svdq_gemm", "svdq_export_act", "svdq_get_status",
            "svdq_status_string", "svdq_last_error_string", "svdq_probe_cvt", "svdq_probe_div", "svdq_probe_tc",
            "svdq_linear_noalloc", "svdq_probe_timeout", "svdq_kv_workspace_bytes", "svdq_kv_encode",
            "svdq_kv_decode", "svdq_kv_attention_workspace_bytes", "svdq_kv_attention",
            "svdq_chain_workspace_bytes", "svdq_gemm_chain")
NOALLOC_SCRATCH_BYTES = 16 << 20   # SVDQ_NOALLOC_SCRATCH_BYTES


def lib():
    return _lib


def params(K: int, N: int, rank: int, fmt: str, dtype: str, alpha: float = 0.5,
           smooth: bool = True) -> svdq_params:
    return svdq_params(K, N, rank, FMT[fmt], DTYPE[dtype], int(bool(smooth)), float(alpha), 0)


def _ptr(a) -> int | None:
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data
    return a.data_ptr()   # torch tensor


def _check(st: int, what: str):
    if st != OK:
        raise SVDQError(st, what)


def status_string(st: int) -> str:
    return _lib.svdq_status_string(st).decode()


def blob_bytes(p: svdq_params) -> int:
    return _lib.svdq_blob_bytes(ctypes.byref(p))


def workspace_bytes(p: svdq_params, M: int) -> int:
    return _lib.svdq_workspace_bytes(ctypes.byref(p), M)


def prepare(p: svdq_params, Wt: np.ndarray, bias: np.ndarray | None, X_cal: np.ndarray | None):
    """Host preparation: returns (blob uint8 array, sigma float64 [rank+1])."""
    Wt = np.ascontiguousarray(Wt, dtype=np.float32)
    assert Wt.shape == (p.N, p.K)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    if X_cal is None:
        xc, mcal = None, 0
    else:
        xc = np.ascontiguousarray(X_cal).view(np.uint16)
        assert xc.shape[1] == p.K
        mcal = xc.shape[0]
    blob = np.zeros(blob_bytes(p), dtype=np.uint8)
    sigma = np.zeros(p.rank + 1, dtype=np.float64)
    _check(_lib.svdq_prepare(ctypes.byref(p), _ptr(Wt), _ptr(b), _ptr(xc), mcal, _ptr(blob), blob.nbytes,
                             _ptr(sigma)), "svdq_prepare")
    return blob, sigma


def blob_check(p: svdq_params, blob: np.ndarray) -> int:
    return _lib.svdq_blob_check(ctypes.byref(p), _ptr(blob), blob.nbytes)


@dataclass
class BlobContents:
    inv_lambda: np.ndarray
    L1: np.ndarray          # K x r uint16 bits of act dtype
    L2: np.ndarray          # r x N uint16 bits
    wcodes: np.ndarray      # N x K (int8 for INT4, uint8 E2M1 code for NVFP4)
    wscales: np.ndarray     # N x K/64 fp32 or N x K/16 uint8
    s_gx: np.float32
    s_gw: np.float32
    bias: np.ndarray


def append_lora(p: svdq_params, blob: np.ndarray, A: np.ndarray, B: np.ndarray):
    """Blob with the LoRA branch X A B added (A: K x r_lora, B: r_lora x N);
    returns (params with the larger rank, new blob)."""
    A = np.ascontiguousarray(A, dtype=np.float32)
    B = np.ascontiguousarray(B, dtype=np.float32)
    r_lora = A.shape[1]
    assert A.shape == (p.K, r_lora) and B.shape == (r_lora, p.N)
    q = svdq_params(p.K, p.N, p.rank + r_lora, p.fmt, p.act_dtype, p.smooth, p.alpha, 0)
    out = np.zeros(max(blob_bytes(q), 1), np.uint8)
    p_out = svdq_params()
    _check(_lib.svdq_append_lora(ctypes.byref(p), _ptr(blob), blob.nbytes, _ptr(A), _ptr(B), r_lora,
                                 ctypes.byref(p_out), _ptr(out), out.nbytes), "svdq_append_lora")
    return p_out, out


def shard_columns(p: svdq_params, blob: np.ndarray, n0: int, n1: int):
    """Output features [n0, n1) of a prepared layer as a layer of its own;
    returns (params with N = n1 - n0, blob)."""
    q = svdq_params(p.K, n1 - n0, p.rank, p.fmt, p.act_dtype, p.smooth, p.alpha, 0)
    out = np.zeros(max(blob_bytes(q), 1), np.uint8)
    p_out = svdq_params()
    _check(_lib.svdq_shard_columns(ctypes.byref(p), _ptr(blob), blob.nbytes, n0, n1, ctypes.byref(p_out),
                                   _ptr(out), out.nbytes), "svdq_shard_columns")
    return p_out, out


def shard_bounds(N: int, world: int) -> list[tuple[int, int]]:
    """Split N output features into `world` column ranges of whole 256-column
    tiles, as even as possible (the first ranges take the extra tiles)."""
    tiles = N // 256
    assert N % 256 == 0 and 1 <= world <= tiles, (N, world)
    base, extra = divmod(tiles, world)
    out, n0 = [], 0
    for r in range(world):
        n1 = n0 + 256 * (base + (1 if r < extra else 0))
        out.append((n0, n1))
        n0 = n1
    return out


def all_gather_columns(y_local, bounds, group=None):
    """Column-parallel output: every rank holds Y[:, n0:n1] of its own range;
    returns the whole Y (M x N) on every rank (torch.distributed all_gather,
    NCCL between GPUs).  Ranges may differ in width by one tile."""
    import torch
    import torch.distributed as dist
    M = y_local.shape[0]
    width = max(n1 - n0 for n0, n1 in bounds)
    pad = torch.zeros((M, width), dtype=y_local.dtype, device=y_local.device)
    pad[:, :y_local.shape[1]] = y_local
    parts = [torch.empty_like(pad) for _ in bounds]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([t[:, :n1 - n0] for t, (n0, n1) in zip(parts, bounds)], dim=1)


def blob_export(p: svdq_params, blob: np.ndarray) -> BlobContents:
    K, N, r = p.K, p.N, p.rank
    inv = np.zeros(K, np.float32)
    L1 = np.zeros((K, r), np.uint16)
    L2 = np.zeros((r, N), np.uint16)
    wc = np.zeros((N, K), np.uint8)
    ws = np.zeros((N, K // 64), np.float32) if p.fmt == INT4_G64 else np.zeros((N, K // 16), np.uint8)
    ts = np.zeros(2, np.float32)
    b = np.zeros(N, np.float32)
    _check(_lib.svdq_blob_export(ctypes.byref(p), _ptr(blob), _ptr(inv), _ptr(L1), _ptr(L2), _ptr(wc),
                                 _ptr(ws), _ptr(ts), _ptr(b)), "svdq_blob_export")
    if p.fmt == INT4_G64:
        wc = wc.view(np.int8)
    return BlobContents(inv, L1, L2, wc, ws, ts[0], ts[1], b)


def linear(p: svdq_params, blob_dev, X, M: int, Y, workspace, stream=None):
    """Launch Y = Q(X^) Q(R) + (X^ L1) L2 + b on `stream` (torch tensors or raw ints)."""
    st = _lib.svdq_linear(ctypes.byref(p), _ptr(blob_dev), _ptr(X), M, _ptr(Y), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "svdq_linear")


def kv_workspace_bytes(T: int, C: int) -> int:
    return _lib.svdq_kv_workspace_bytes(T, C)


def kv_encode(X, T: int, C: int, dtype: str, codes, scale, zero, workspace, stream=None):
    """Asymmetric per-channel INT8 encode of a T x C cache block (device tensors)."""
    st = _lib.svdq_kv_encode(_ptr(X), T, C, DTYPE[dtype], _ptr(codes), _ptr(scale), _ptr(zero), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "svdq_kv_encode")


def kv_decode(codes, scale, zero, T: int, C: int, dtype: str, Y, stream=None):
    st = _lib.svdq_kv_decode(_ptr(codes), _ptr(scale), _ptr(zero), T, C, DTYPE[dtype], _ptr(Y), _stream(stream))
    _check(st, "svdq_kv_decode")


def kv_attention_workspace_bytes(T: int, C: int, heads: int, Mq: int) -> int:
    return _lib.svdq_kv_attention_workspace_bytes(T, C, heads, Mq)


def kv_attention(Q, Mq: int, kcodes, kscale, kzero, vcodes, vscale, vzero, T: int, C: int, heads: int, dtype: str,
                 out, workspace, stream=None):
    """Attention of Mq query rows over INT8-coded keys and values (device tensors); out: Mq x C fp32."""
    st = _lib.svdq_kv_attention(_ptr(Q), Mq, _ptr(kcodes), _ptr(kscale), _ptr(kzero), _ptr(vcodes), _ptr(vscale),
                                _ptr(vzero), T, C, heads, DTYPE[dtype], _ptr(out), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "svdq_kv_attention")


def linear_noalloc(p: svdq_params, blob_dev, X, M: int, Y, stream=None):
    """svdq_linear with the library's static scratch as workspace (allocates
    nothing; calls on one device must not overlap)."""
    st = _lib.svdq_linear_noalloc(ctypes.byref(p), _ptr(blob_dev), _ptr(X), M, _ptr(Y), _stream(stream))
    if st == ERR_WORKSPACE:
        raise SVDQError(st, "svdq_linear_noalloc: " + _lib.svdq_last_error_string().decode())
    _check(st, "svdq_linear_noalloc")


def quantize_act(p: svdq_params, blob_dev, X, M: int, workspace, stream=None):
    """Kernel 1 only: X -> quantised activations + down projection in `workspace`."""
    _check(_lib.svdq_quantize_act(ctypes.byref(p), _ptr(blob_dev), _ptr(X), M, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)),
           "svdq_quantize_act")


def gemm(p: svdq_params, blob_dev, M: int, Y, workspace, stream=None):
    """Kernel 2 only: workspace -> Y (after quantize_act on the same stream)."""
    _check(_lib.svdq_gemm(ctypes.byref(p), _ptr(blob_dev), M, _ptr(Y), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream)), "svdq_gemm")


def chain_workspace_bytes(p: svdq_params, p_next: svdq_params, M: int) -> int:
    """Workspace bytes of gemm_chain (0 if the pair of layers cannot chain)."""
    return _lib.svdq_chain_workspace_bytes(ctypes.byref(p), ctypes.byref(p_next), M)


def gemm_chain(p: svdq_params, blob_dev, M: int, p_next: svdq_params, blob_next_dev, workspace, ws_next,
               stream=None):
    """This layer's GEMM emitting the next layer's quantised input into ws_next
    (in place of quantize_act(p_next, ..., Y, ...)); finish with gemm(p_next, ...)."""
    _check(_lib.svdq_gemm_chain(ctypes.byref(p), _ptr(blob_dev), M, ctypes.byref(p_next), _ptr(blob_next_dev),
                                _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(ws_next),
                                ws_next.numel() * ws_next.element_size(), _stream(stream)), "svdq_gemm_chain")


def export_act(p: svdq_params, workspace, M: int, stream=None):
    """Quantised activations after svdq_linear: (codes M x K, scales, u' M x r)."""
    K, r = p.K, p.rank
    codes = np.zeros((M, K), np.uint8)
    scales = np.zeros((M, K // 64), np.float32) if p.fmt == INT4_G64 else np.zeros((M, K // 16), np.uint8)
    u = np.zeros((M, r), np.float32)
    _check(_lib.svdq_export_act(ctypes.byref(p), _ptr(workspace), M, _ptr(codes), _ptr(scales), _ptr(u),
                                _stream(stream)), "svdq_export_act")
    if p.fmt == INT4_G64:
        codes = codes.view(np.int8)
    return codes, scales, u


def get_status(stream=None) -> int:
    return _lib.svdq_get_status(_stream(stream))


def probe_cvt(x, e2m1, e4m3, stream=None):
    _check(_lib.svdq_probe_cvt(_ptr(x), x.numel(), _ptr(e2m1), _ptr(e4m3), _stream(stream)), "svdq_probe_cvt")


def probe_div(v, d, q, q_ieee, stream=None):
    _check(_lib.svdq_probe_div(_ptr(v), _ptr(d), v.numel(), _ptr(q), _ptr(q_ieee), _stream(stream)),
           "svdq_probe_div")


def probe_timeout(limit_ns: int, stream=None):
    _check(_lib.svdq_probe_timeout(limit_ns, _stream(stream)), "svdq_probe_timeout")


def probe_tc(op: int, iters: int, ctas: int, cycles, stream=None):
    _check(_lib.svdq_probe_tc(op, iters, ctas, _ptr(cycles), _stream(stream)), "svdq_probe_tc")


def _stream(s):
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


class Layer:
    """One prepared SVDQuant linear layer resident on a CUDA device.

    Holds the device copy of the blob and a workspace sized for up to
    `max_tokens` tokens; `__call__` runs svdq_linear on torch's current stream.
    """

    def __init__(self, K, N, rank, fmt, dtype, Wt, bias, X_cal, alpha=0.5, smooth=True,
                 max_tokens=4096, device="cuda"):
        import torch
        self.p = params(K, N, rank, fmt, dtype, alpha, smooth)
        self.blob_host, self.sigma = prepare(self.p, Wt, bias, X_cal)
        self.blob = torch.from_numpy(self.blob_host).to(device)
        self.max_tokens = max_tokens
        self.ws = torch.empty(workspace_bytes(self.p, max_tokens), dtype=torch.uint8, device=device)
        self.device = device

    def __call__(self, X, out=None, stream=None):
        import torch
        M = X.shape[0]
        if M > self.max_tokens:
            raise ValueError("more tokens than the workspace holds")
        if out is None:
            out = torch.empty((M, self.p.N), dtype=torch.bfloat16, device=X.device)
        linear(self.p, self.blob, X, M, out, self.ws, stream)
        return out
