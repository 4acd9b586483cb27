"""Chained layers: one NVFP4 layer's GEMM emits the next layer's quantised
input (its E2M1 codes, E4M3 block scales and low-rank input u'), so the first
layer's bf16 output never makes a round trip through HBM.

CPU: the host rules of svdq_chain_workspace_bytes.  GPU: the chained call
against the oracle (next_layer_input, then the next layer's output), and
against the unfused GPU path (svdq_linear of the first layer, then the next
layer's svdq_quantize_act on its output), which must agree bit for bit on
codes and scales."""
import numpy as np
import pytest

import rank_gemm_svdq_b200 as sv
import synth
from oracle import formats, quant, svdquant as sq
from tests import gpu_cases as G

# The next layer's Y against the oracle's two-layer composition.  The 1e-3 bar
# holds per layer on the layer's own input; between the layers the two sides'
# bf16 outputs differ in a fraction of a percent of the elements by one ulp,
# and where such an element sits at an E2M1 rounding boundary the next
# quantiser turns it into a whole code step.  Measured: ~1e-3 (global) on the
# small cases; the bar leaves room for that amplification.
Y2_TOL = 5e-3


def _align(x, a=1024):
    return (x + a - 1) // a * a


def test_chain_workspace_rules():
    p1 = sv.params(512, 768, 32, "nvfp4", "bf16")
    p2 = sv.params(768, 512, 32, "nvfp4", "bf16")
    # above 128 tokens: the partial down projections, one per 256-column output tile (Mp = 512 at 300 tokens)
    assert sv.chain_workspace_bytes(p1, p2, 300) == _align(sv.workspace_bytes(p1, 300)) + _align(3 * 512 * 32 * 4)
    # up to 128 tokens: this layer's bf16 output
    assert sv.chain_workspace_bytes(p1, p2, 100) == _align(sv.workspace_bytes(p1, 100)) + _align(100 * 768 * 2)
    assert sv.chain_workspace_bytes(p1, sv.params(768, 512, 0, "nvfp4", "bf16"), 300) == \
        _align(sv.workspace_bytes(p1, 300))
    for bad in (sv.params(768, 512, 32, "int4", "bf16"), sv.params(768, 512, 32, "nvfp4", "fp16"),
                sv.params(768, 512, 48, "nvfp4", "bf16"), sv.params(1024, 512, 32, "nvfp4", "bf16")):
        assert sv.chain_workspace_bytes(p1, bad, 300) == 0
    assert sv.chain_workspace_bytes(sv.params(512, 768, 32, "int4", "bf16"), p2, 300) == 0


def _pair(wl1, N2, r2, seed):
    """This layer (prepared by the library) and a next layer calibrated on
    this layer's output as the oracle computes it."""
    pp1 = G.prepare(wl1)
    y1 = formats.to_bf16(sq.forward(pp1.x64, pp1.ref))
    wl2 = synth.Workload(name="next", M=wl1.M, K=wl1.N, N=N2, rank=r2, fmt="nvfp4", dtype="bf16", seed=seed)
    wl2.X = synth.f64_to_bf16_bits(y1)
    wl2.Wt = synth.make_weight(seed, N2, wl1.N)
    wl2.bias = synth.make_bias(seed, N2)
    return pp1, G.prepare(wl2), y1


def _run(pp1, pp2, X):
    import torch
    p1, p2 = pp1.p, pp2.p
    M = X.shape[0]
    blob1 = torch.from_numpy(pp1.blob).cuda()
    blob2 = torch.from_numpy(pp2.blob).cuda()
    xd = G.to_device_x(X, "bf16")
    wsz, nsz = sv.chain_workspace_bytes(p1, p2, M), sv.workspace_bytes(p2, M)
    assert wsz > 0
    wbuf = torch.full((wsz + 4096,), G.CANARY, dtype=torch.uint8, device="cuda")
    nbuf = torch.full((nsz + 4096,), G.CANARY, dtype=torch.uint8, device="cuda")
    ws, wsn = wbuf[:wsz], nbuf[:nsz]
    y2buf = torch.full((M + 2, p2.N), -7.0, dtype=torch.bfloat16, device="cuda")
    y2 = y2buf[1:M + 1]
    sv.quantize_act(p1, blob1, xd, M, ws)
    sv.gemm_chain(p1, blob1, M, p2, blob2, ws, wsn)
    sv.gemm(p2, blob2, M, y2, wsn)
    assert sv.get_status() == sv.OK
    torch.cuda.synchronize()
    assert torch.all(wbuf[wsz:] == G.CANARY) and torch.all(nbuf[nsz:] == G.CANARY), "write outside a workspace"
    assert torch.all(y2buf[0] == -7.0) and torch.all(y2buf[M + 1] == -7.0), "write outside Y"
    chained = sv.export_act(p2, wsn, M)
    # the unfused GPU path: this layer's output, then the next layer's activation kernel on it
    ws1 = torch.empty(sv.workspace_bytes(p1, M), dtype=torch.uint8, device="cuda")
    y1 = torch.empty((M, p1.N), dtype=torch.bfloat16, device="cuda")
    sv.linear(p1, blob1, xd, M, y1, ws1)
    ws2 = torch.empty(nsz, dtype=torch.uint8, device="cuda")
    sv.quantize_act(p2, blob2, y1, M, ws2)
    unfused = sv.export_act(p2, ws2, M)
    assert sv.get_status() == sv.OK
    c = sv.blob_export(p2, pp2.blob)
    to_oracle_u = float(c.s_gx) * float(c.s_gw)
    return (chained, unfused, y1.float().cpu().numpy().astype(np.float64),
            y2.float().cpu().numpy().astype(np.float64), to_oracle_u)


def _check(pp1, pp2, X, y1_ref):
    M = X.shape[0]
    chained, unfused, y1_gpu, y2_gpu, to_u = _run(pp1, pp2, X)
    codes, scales, u = chained
    # 1. the fused epilogue quantises exactly as the next layer's activation kernel does
    assert np.array_equal(codes, unfused[0]), "codes differ from the unfused GPU path"
    assert np.array_equal(scales, unfused[1]), "scales differ from the unfused GPU path"
    if pp2.p.rank > 0:
        uerr = np.linalg.norm(u - unfused[2]) / max(np.linalg.norm(unfused[2]), 1e-300)
        assert uerr <= (0.0 if M <= 128 else 1e-5), f"u differs from the unfused GPU path by {uerr}"
    # 2. against the oracle: bit-exact wherever this layer's bf16 output agrees
    #    with the oracle's on the whole 16-value block (elsewhere the block's
    #    codes quantise a slightly different y and must only be valid)
    a = sq.next_layer_input(pp1.x64, pp1.ref, pp2.ref)
    blocks_same = (y1_gpu == y1_ref).reshape(M, -1, 16).all(axis=2)
    bc = codes.reshape(M, -1, 16)
    ac = a.codes.reshape(M, -1, 16)
    assert np.array_equal(bc[blocks_same], ac[blocks_same]), "codes differ from the oracle on agreeing blocks"
    assert np.array_equal(scales[blocks_same], a.scales[blocks_same]), "scales differ on agreeing blocks"
    assert blocks_same.mean() > 0.95
    xh = sq.smooth_act(y1_ref, pp2.ref.inv_lambda).astype(np.float64)
    deq = quant.nvfp4_dequant(codes, scales, pp2.ref.s_gx)
    d = (formats.e4m3_decode(scales).astype(np.float64) * float(pp2.ref.s_gx)).repeat(16, axis=1)
    assert np.all(np.abs(deq - xh) <= 2 * d + 2.0 ** -7 * np.abs(xh)), "a code outside one step of the oracle's value"
    out = {"blocks_bit_exact": float(blocks_same.mean())}
    if pp2.p.rank > 0:
        uerr = np.linalg.norm(u * to_u - a.u) / np.linalg.norm(a.u)
        out["u_rel_err"] = float(uerr)
        assert uerr <= 1e-3, f"u rel err {uerr}"
    # 3. the next layer's output from the chained input
    y2_ref = formats.to_bf16(sq.forward(y1_ref, pp2.ref))
    err = sq.rel_fro(y2_gpu, y2_ref)
    worst, where = G.tile_errors(y2_gpu, y2_ref)
    out.update(y2_rel_err=err, y2_worst_tile=worst)
    assert err <= Y2_TOL and worst <= 2 * Y2_TOL, (err, worst, where)
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,N,N2,r2", [
    (300, 512, 768, 512, 32),   # ragged 256-row tiles, three output tile columns
    (129, 512, 512, 256, 16),   # one token past the few-token route, next rank 16
    (128, 512, 768, 512, 32),   # few tokens: GEMM -> workspace -> next activation kernel
    (1, 256, 512, 256, 32),
    (513, 768, 1024, 768, 0),   # next layer without a low-rank branch
])
def test_gpu_chain_small(gpu, M, K, N, N2, r2):
    wl1 = synth.custom_workload(M, K, N, 32, "nvfp4", "bf16", n_out=5, factor=50.0, seed=60 + M)
    pp1, pp2, y1 = _pair(wl1, N2, r2, seed=61 + M)
    print(M, K, N, N2, r2, _check(pp1, pp2, pp1.wl.X, y1))


@pytest.mark.gpu
def test_gpu_chain_flux_ffn(gpu):
    """FLUX FFN up (4608 x 3072 -> 12288) feeding an FFN down projection
    (12288 -> 3072, rank 32): the up projection's 113 MB bf16 output is never
    written; the down projection's input comes out of the up projection's
    epilogue."""
    wl1 = synth.make_workload("flux_ffn_up_nvfp4")
    pp1, pp2, y1 = _pair(wl1, 3072, 32, seed=7)
    print(_check(pp1, pp2, wl1.X, y1))


def test_chain_rejects_unsupported_pairs_before_any_launch():
    """The chained call checks the pair of layers on the host and returns
    before touching a device pointer (no GPU needed)."""
    import torch
    p1 = sv.params(512, 768, 32, "nvfp4", "bf16")
    dummy = torch.zeros(1024, dtype=torch.uint8)
    cases = [(sv.params(768, 512, 32, "int4", "bf16"), sv.ERR_UNSUPPORTED),
             (sv.params(768, 512, 32, "nvfp4", "fp16"), sv.ERR_UNSUPPORTED),
             (sv.params(768, 512, 48, "nvfp4", "bf16"), sv.ERR_UNSUPPORTED),
             (sv.params(1024, 512, 32, "nvfp4", "bf16"), sv.ERR_INVALID_ARG)]
    for p2, want in cases:
        with pytest.raises(sv.SVDQError) as e:
            sv.gemm_chain(p1, dummy, 300, p2, dummy, dummy, dummy)
        assert e.value.status == want, (p2.K, p2.fmt, p2.act_dtype, p2.rank, e.value.status)
    with pytest.raises(sv.SVDQError) as e:   # this layer INT4
        sv.gemm_chain(sv.params(512, 768, 32, "int4", "bf16"), dummy, 300, sv.params(768, 512, 32, "nvfp4", "bf16"),
                      dummy, dummy, dummy)
    assert e.value.status == sv.ERR_UNSUPPORTED
