"""svdq_linear_noalloc: the allocation-free entry point (static device scratch).

Some callers cannot allocate device memory where the layer runs: a host
framework whose allocator is out of reach at that point, or code that runs
while allocation is forbidden.  svdq_linear_noalloc serves them by taking its
workspace from a scratch array in the library's own static device memory.

This file is named so that pytest collects it last: it must give the same
results whether it runs alone in a fresh process or after every other test has
used the device (and the scratch holds whatever the last call left there).
The GPU test compares it, bit for bit, with svdq_linear on a caller-supplied
workspace over two calls in a row -- the same kernels on the same inputs --
and once with the CPU oracle; the size check needs no GPU.
"""
import numpy as np
import pytest

import rank_gemm_svdq_b200 as sv
import synth
from oracle import formats, svdquant as sq
from tests import gpu_cases as G


def test_noalloc_rejects_workspace_beyond_static_scratch():
    p = sv.params(3072, 3072, 32, "int4", "bf16")
    M = 8192
    assert sv.workspace_bytes(p, M) > sv.NOALLOC_SCRATCH_BYTES
    with pytest.raises(sv.SVDQError, match="exceeds the static scratch"):
        sv.linear_noalloc(p, None, None, M, None)


def test_noalloc_scratch_covers_k3072_at_4608_tokens():
    for fmt in ("int4", "nvfp4"):
        for dt in ("bf16", "fp16"):
            p = sv.params(3072, 12288, 32, fmt, dt)
            assert sv.workspace_bytes(p, 4608) <= sv.NOALLOC_SCRATCH_BYTES


@pytest.mark.gpu
@pytest.mark.parametrize("fmt,M,K,N", [
    ("nvfp4", 300, 512, 768),
    ("int4", 300, 512, 768),
    ("nvfp4", 4608, 3072, 1024),
    ("nvfp4", 4, 4096, 512),     # few tokens and tiles: K split, arrival counters in the scratch
])
def test_noalloc_matches_linear_twice(gpu, fmt, M, K, N):
    import torch
    wl = synth.custom_workload(M, K, N, 32, fmt, "bf16", n_out=5, factor=80.0, seed=M + 3)
    pp = G.prepare(wl)
    p = pp.p
    xd = G.to_device_x(wl.X, wl.dtype)
    blob = torch.from_numpy(pp.blob).cuda()
    ws = torch.empty(sv.workspace_bytes(p, M), dtype=torch.uint8, device="cuda")
    y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    sv.linear(p, blob, xd, M, y_ref, ws)
    ref = y_ref.view(torch.int16).cpu().numpy()
    for _ in range(2):
        y = torch.full((M, N), -7.0, dtype=torch.bfloat16, device="cuda")
        sv.linear_noalloc(p, blob, xd, M, y)
        torch.cuda.synchronize()
        assert np.array_equal(y.view(torch.int16).cpu().numpy(), ref)
    assert sv.get_status() == sv.OK
    # and against the oracle, within the parity tolerance, globally and per tile
    got = y.float().cpu().numpy().astype(np.float64)
    Yref = formats.to_bf16(sq.forward(pp.x64, pp.ref))
    assert sq.rel_fro(got, Yref) <= G.Y_TOL
    assert G.tile_errors(got, Yref)[0] <= G.Y_TOL
