"""INT8 KV-cache codec ("VAR-Compressor…" INT8 KV缓存量化): the oracle against
a hand-worked fixture and the rule's invariants (CPU), the CUDA kernels
against the oracle (GPU, bit-exact codes / scales / zero points and decoded
values)."""
import os

import numpy as np
import pytest

import synth
from oracle import kvcache as kv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_int8_asym.txt")


def load_golden():
    chans = []
    for line in open(GOLDEN):
        if not line.strip() or line.startswith("#"):
            continue
        f = line.split()
        pairs = [tuple(map(float, t.split(":"))) for t in f[3:]]
        chans.append((float(f[1]), int(f[2]), [p[0] for p in pairs], [int(p[1]) for p in pairs]))
    return chans


def test_golden_codes():
    chans = load_golden()
    x = np.array([c[2] for c in chans]).T            # T x C
    q, s, z = kv.encode(x)
    assert np.array_equal(s, np.array([c[0] for c in chans], np.float32))
    assert np.array_equal(z, np.array([c[1] for c in chans], np.uint8))
    assert np.array_equal(q, np.array([c[3] for c in chans], np.uint8).T)


def skewed_block(T, C, seed):
    """Channel-driven variance (per-channel scales spread over 3 decades) and
    positive skew (a shifted log-normal), as the page describes the cache."""
    g = synth.normal(seed, "X", T * C).reshape(T, C)
    scale = np.exp(synth.normal(seed, "extra", C) * 1.2)
    x = (np.exp(0.6 * g) - 1.2) * scale[None, :]
    return synth.dtype_to_f64(synth.to_dtype(x, "fp16"), "fp16")


def test_round_trip_error_is_half_a_step():
    x = skewed_block(257, 192, 3)
    q, s, z = kv.encode(x)
    err = np.abs(kv.decode(q, s, z) - x)
    assert np.all(err <= 0.5 * s[None, :] * (1 + 1e-5) + 1e-30)


def test_range_ends_map_to_the_code_ends():
    x = skewed_block(64, 256, 4)
    q, s, z = kv.encode(x)
    lo, hi = np.minimum(x.min(0), 0), np.maximum(x.max(0), 0)
    rows_lo, rows_hi = x.argmin(0), x.argmax(0)
    c = np.arange(x.shape[1])
    assert np.all(q[rows_lo, c][lo < 0] == 0)
    assert np.all(np.isin(q[rows_hi, c][hi > 0], (254, 255)))
    # a zero entry is exact: it decodes to 0
    assert np.all(kv.decode(np.broadcast_to(z, (1, z.size)).copy(), s, z) == 0)


def test_asymmetric_beats_symmetric_on_skewed_data():
    """The page's reason for the zero point: on the skewed cache the
    asymmetric step is finer than a symmetric int8 step (absmax / 127)."""
    x = skewed_block(128, 128, 5)
    q, s, z = kv.encode(x)
    sym = np.abs(x).max(0) / 127.0
    assert np.all(s <= sym * (1 + 1e-6))
    assert np.mean(np.abs(kv.decode(q, s, z) - x)) < 0.75 * np.mean(
        np.abs(np.clip(np.rint(x / sym), -127, 127) * sym - x))


def _block_bits(T, C, dtype, seed):
    """A skewed T x C block as dtype bit patterns (uint16) and its float64 values."""
    g = synth.normal(seed, "X", T * C).reshape(T, C)
    scale = np.exp(synth.normal(seed, "extra", C) * 1.2)
    x = (np.exp(0.6 * g) - 1.2) * scale[None, :]
    x[:, :3] = 0.0                                   # all-zero channels (scale 1, zero point 0)
    bits = synth.to_dtype(x, dtype)
    bits = bits.view(np.uint16) if dtype == "fp16" else bits
    return bits, synth.dtype_to_f64(synth.to_dtype(x, dtype), dtype)


@pytest.mark.gpu
@pytest.mark.parametrize("T,C,dtype", [(1, 256, "bf16"), (300, 512, "fp16"), (257, 768, "bf16"),
                                       (4096, 4096, "bf16")])
def test_gpu_kv_codec_matches_oracle(gpu, T, C, dtype):
    """svdq_kv_encode / svdq_kv_decode against the oracle: codes, scales and
    zero points bit-exact, decoded values bit-exact after rounding to the dtype.
    The largest case (a 4096-token x 4096-channel VAR-like block) is also timed."""
    import torch
    import rank_gemm_svdq_b200 as sv
    bits, x = _block_bits(T, C, dtype, seed=T + C)
    X = torch.from_numpy(bits.view(np.int16)).cuda()
    codes = torch.empty((T, C), dtype=torch.uint8, device="cuda")
    scale = torch.empty(C, dtype=torch.float32, device="cuda")
    zero = torch.empty(C, dtype=torch.uint8, device="cuda")
    ws = torch.empty(sv.kv_workspace_bytes(T, C), dtype=torch.uint8, device="cuda")
    sv.kv_encode(X, T, C, dtype, codes, scale, zero, ws)
    Y = torch.empty((T, C), dtype=torch.int16, device="cuda")
    sv.kv_decode(codes, scale, zero, T, C, dtype, Y)
    torch.cuda.synchronize()
    q, s, z = kv.encode(x)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert np.array_equal(zero.cpu().numpy(), z)
    assert np.array_equal(codes.cpu().numpy(), q)
    ref = synth.to_dtype(kv.decode(q, s, z), dtype)
    ref = ref.view(np.uint16) if dtype == "fp16" else ref
    assert np.array_equal(Y.cpu().numpy().view(np.uint16), ref)
    if T * C >= 1 << 24:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

        def timed(fn):
            ts = []
            for i in range(12):
                flush.fill_(i)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(); fn(); b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) * 1e3)
            return float(np.median(ts[2:]))
        te = timed(lambda: sv.kv_encode(X, T, C, dtype, codes, scale, zero, ws))
        td = timed(lambda: sv.kv_decode(codes, scale, zero, T, C, dtype, Y))
        enc_bytes = T * C * 2 + T * C + C * 5          # X in, codes + scales + zero points out
        dec_bytes = T * C + C * 5 + T * C * 2
        print(f"kv {T}x{C} {dtype}: encode {te:.1f} us = {enc_bytes / te / 1e3:.0f} GB/s, "
              f"decode {td:.1f} us = {dec_bytes / td / 1e3:.0f} GB/s (algorithmic bytes)")


# ------------------------------------------------------------ attention reads
def _kv_pair(T, C, seed):
    kx = skewed_block(T, C, seed)
    vx = skewed_block(T, C, seed + 1000)
    return kv.encode(kx) + kv.encode(vx)


def test_attention_matches_sdpa_on_decoded_cache():
    """The oracle's attention equals the library's scaled dot-product
    attention (torch, float64) over the decoded keys and values, head by head."""
    import torch
    T, C, H = 37, 256, 4
    kq, ks, kz, vq, vs, vz = _kv_pair(T, C, 21)
    Q = synth.dtype_to_f64(synth.to_dtype(synth.normal(22, "X", 3 * C).reshape(3, C), "fp16"), "fp16")
    got = kv.attention(Q, kq, ks, kz, vq, vs, vz, H)
    Kd = torch.from_numpy(kv.decode(kq, ks, kz)); Vd = torch.from_numpy(kv.decode(vq, vs, vz))
    q = torch.from_numpy(Q)
    d = C // H
    for h in range(H):
        cols = slice(h * d, (h + 1) * d)
        ref = torch.nn.functional.scaled_dot_product_attention(q[None, None, :, cols], Kd[None, None, :, cols],
                                                               Vd[None, None, :, cols])[0, 0].numpy()
        assert np.max(np.abs(got[:, cols] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_attention_closed_forms():
    """Zero queries attend uniformly (output = the mean decoded value); a key
    that dominates every score hands back its own value row; permuting the
    cached tokens changes nothing; heads do not mix."""
    T, C, H = 50, 256, 2
    kq, ks, kz, vq, vs, vz = _kv_pair(T, C, 23)
    V = kv.decode(vq, vs, vz)
    out = kv.attention(np.zeros((2, C)), kq, ks, kz, vq, vs, vz, H)
    assert np.allclose(out, np.broadcast_to(V.mean(axis=0), out.shape), rtol=0, atol=1e-12 * np.abs(V).max())
    # token 7's key made huge along the query's direction: it takes all the weight
    Q = np.zeros((1, C)); Q[0, 5] = 1.0; Q[0, 200] = 1.0
    kq2 = kq.copy(); kq2[:, 5] = kz[5]; kq2[:, 200] = kz[200]            # every key 0 on those channels
    kq2[7, 5] = 255 if kz[5] < 128 else 0; kq2[7, 200] = 255 if kz[200] < 128 else 0
    ks2 = ks.copy(); ks2[5] = ks2[200] = np.float32(1e3)
    o = kv.attention(Q * np.sign(kq2[7:8].astype(int) - kz.astype(int)).clip(-1, 1) + 0.0, kq2, ks2, kz, vq, vs, vz, H)
    assert np.allclose(o[0, :128], V[7, :128], rtol=0, atol=1e-9 * np.abs(V).max())
    assert np.allclose(o[0, 128:], V[7, 128:], rtol=0, atol=1e-9 * np.abs(V).max())
    perm = np.random.default_rng(0).permutation(T)
    Qr = synth.dtype_to_f64(synth.to_dtype(synth.normal(24, "X", 2 * C).reshape(2, C), "fp16"), "fp16")
    a = kv.attention(Qr, kq, ks, kz, vq, vs, vz, H)
    b = kv.attention(Qr, kq[perm], ks, kz, vq[perm], vs, vz, H)
    assert np.allclose(a, b, rtol=0, atol=1e-12 * np.abs(a).max())
    Qh = Qr.copy(); Qh[:, 128:] *= 3.0                                  # head 1's queries only
    c = kv.attention(Qh, kq, ks, kz, vq, vs, vz, H)
    assert np.array_equal(c[:, :128], a[:, :128])


def test_attention_argument_checks():
    import rank_gemm_svdq_b200 as sv
    assert sv.kv_attention_workspace_bytes(300, 512, 4, 3) == 4 * 2 * 3 * (128 + 2) * 4
    assert sv.kv_attention_workspace_bytes(0, 512, 4, 3) == 0
    assert sv.kv_attention_workspace_bytes(10, 500, 3, 1) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("T,C,H,Mq,dtype", [(1, 256, 4, 1, "bf16"), (300, 512, 4, 3, "fp16"),
                                            (257, 1024, 16, 16, "bf16"), (4096, 4096, 32, 1, "bf16"),
                                            (4096, 4096, 32, 8, "bf16")])
def test_gpu_attention_reads_match_oracle(gpu, T, C, H, Mq, dtype):
    """svdq_kv_attention over codes written by svdq_kv_encode against the
    oracle's attention over the decoded cache (fp32 output, relative
    Frobenius error <= 1e-5 and per-element <= 1e-4 of the output range);
    two calls give identical bits.  The 4096-token VAR-like cache is timed."""
    import torch
    import rank_gemm_svdq_b200 as sv
    from oracle import svdquant as sq
    kbits, kx = _block_bits(T, C, dtype, seed=T + C + 1)
    vbits, vx = _block_bits(T, C, dtype, seed=T + C + 2)
    qx = synth.normal(T + Mq, "X", Mq * C).reshape(Mq, C)
    qbits = synth.to_dtype(qx, dtype)
    qbits = qbits.view(np.uint16) if dtype == "fp16" else qbits
    Q = synth.dtype_to_f64(synth.to_dtype(qx, dtype), dtype)
    dev = {}
    for name, bits in (("k", kbits), ("v", vbits)):
        X = torch.from_numpy(bits.view(np.int16)).cuda()
        codes = torch.empty((T, C), dtype=torch.uint8, device="cuda")
        scale = torch.empty(C, dtype=torch.float32, device="cuda")
        zero = torch.empty(C, dtype=torch.uint8, device="cuda")
        ws = torch.empty(sv.kv_workspace_bytes(T, C), dtype=torch.uint8, device="cuda")
        sv.kv_encode(X, T, C, dtype, codes, scale, zero, ws)
        dev[name] = (codes, scale, zero)
    Qd = torch.from_numpy(qbits.view(np.int16)).cuda()
    out = torch.empty((Mq, C), dtype=torch.float32, device="cuda")
    wsa = torch.empty(sv.kv_attention_workspace_bytes(T, C, H, Mq), dtype=torch.uint8, device="cuda")
    sv.kv_attention(Qd, Mq, *dev["k"], *dev["v"], T, C, H, dtype, out, wsa)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    kq, ks, kz = kv.encode(kx)
    vq, vs, vz = kv.encode(vx)
    assert np.array_equal(dev["k"][0].cpu().numpy(), kq) and np.array_equal(dev["v"][0].cpu().numpy(), vq)
    ref = kv.attention(Q, kq, ks, kz, vq, vs, vz, H)
    assert sq.rel_fro(got, ref) <= 1e-5, sq.rel_fro(got, ref)
    assert np.max(np.abs(got - ref)) <= 1e-4 * np.max(np.abs(ref))
    out2 = torch.empty_like(out)
    sv.kv_attention(Qd, Mq, *dev["k"], *dev["v"], T, C, H, dtype, out2, wsa)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    if T * C >= 1 << 24:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        ts = []
        for i in range(12):
            flush.fill_(i)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(); sv.kv_attention(Qd, Mq, *dev["k"], *dev["v"], T, C, H, dtype, out, wsa); b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        t = float(np.median(ts[2:]))
        byts = 2 * T * C + Mq * C * 2 + Mq * C * 4 + 10 * C
        print(f"kv attention {T}x{C} heads {H} queries {Mq}: {t:.1f} us = {byts / t / 1e3:.0f} GB/s (algorithmic bytes)")
