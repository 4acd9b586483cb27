"""svdq_linear_noalloc: the allocation-free entry point (static device scratch).

Named so that it is collected after every other test file: it must give the
same results whether it runs alone or after everything else has used the
device.  The GPU test compares it with svdq_linear (caller-supplied workspace)
on two calls in a row; the size check needs no GPU.
"""
import numpy as np
import pytest

import rank_gemm_svdq_b200 as sv
import synth
from oracle import svdquant as sq
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
@pytest.mark.parametrize("fmt,M", [("nvfp4", 300), ("int4", 300), ("nvfp4", 4608)])
def test_noalloc_matches_linear_twice(gpu, fmt, M):
    import torch
    K, N = (512, 768) if M < 1024 else (3072, 1024)
    wl = synth.custom_workload(M, K, N, 32, fmt, "bf16", n_out=5, factor=80.0, seed=M + 3)
    pp = G.prepare(wl)
    p = pp.p
    xd = G.to_device_x(wl.X, wl.dtype)
    blob = torch.from_numpy(pp.blob).cuda()
    ws = torch.empty(sv.workspace_bytes(p, M), dtype=torch.uint8, device="cuda")
    y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    sv.linear(p, blob, xd, M, y_ref, ws)
    ref = y_ref.float().cpu().numpy().astype(np.float64)
    for _ in range(2):
        y = torch.full((M, N), -7.0, dtype=torch.bfloat16, device="cuda")
        sv.linear_noalloc(p, blob, xd, M, y)
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        assert sq.rel_fro(got, ref) <= G.Y_TOL
    assert sv.get_status() == sv.OK
