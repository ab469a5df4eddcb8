"""cq_lut_gemm_noalloc: the LUT GEMM for callers that cannot allocate device
memory (framework plugins that are handed only inputs and outputs, serving
processes that forbid cudaMalloc after start-up).  Its scratch is a fixed
array inside the library, so these checks call it through the C ABI with
caller-owned inputs/outputs only, twice in a row (the second call reuses the
array the first one left behind), and compare it with the oracle at the
stated tolerance and with cq_lut_gemm bit for bit (the two run the same plan
and kernels).

This file is named to be collected last."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

CASES = [
    # (M, K, N, bits): all need split-K scratch; M > 16 runs a tensor-memory kernel
    (4, 9728, 128, 4),
    (16, 9728, 256, 8),
    (1, 14336, 64, 4),
    (40, 9728, 128, 4),
    (24, 2560, 256, 8),
]


def _inputs(M, K, N, bits, seed):
    g = np.random.default_rng(seed)
    qmax = 2 ** (bits - 1) - 1
    q = g.integers(-qmax, qmax + 1, (M, K)).astype(np.int8)
    s = (g.random(M) * 0.05 + 1e-3).astype(np.float32)
    w_idx, cb = synth.lut_weights(N, K, seed=seed, name=f"noalloc{M}.{K}.{N}")
    return q, s, w_idx, cb


@pytest.mark.parametrize("M,K,N,bits", CASES)
def test_noalloc_matches_oracle_and_workspace_entry_point(M, K, N, bits):
    import lut_clustered_weight_b200 as cq
    assert torch.cuda.is_available()
    dev = "cuda"
    q, s, w_idx, cb = _inputs(M, K, N, bits, seed=M + K + N)
    ws_bytes = cq.cq_lut_gemm_workspace_size(M, N, K, bits)
    assert 0 < ws_bytes <= cq.NOALLOC_SCRATCH_BYTES   # the scratch path is exercised
    qd = torch.from_numpy(oracle.pack_codes(q, bits)).to(dev)
    sd = torch.from_numpy(s).to(dev)
    wd = torch.from_numpy(w_idx).to(dev)
    cd = torch.from_numpy(cb).to(dev)
    y_ws = cq.cq_lut_gemm(qd, sd, K, bits, wd, cd).cpu().numpy()
    yr, mag, _ = oracle.lut_gemm(q, s, w_idx, cb)
    tol = oracle.lut_tolerance(mag)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        rc = cq.lib.cq_lut_gemm_noalloc(qd.data_ptr(), sd.data_ptr(), M, K, bits,
                                        wd.data_ptr(), cd.data_ptr(), N, y.data_ptr(), stream)
        assert rc == cq.CQ_OK, cq.status_string(rc)
        torch.cuda.synchronize()
        yn = y.cpu().numpy()
        assert np.all(np.abs(yn.astype(np.float64) - yr) <= tol)
        assert np.array_equal(yn.view(np.uint32), y_ws.view(np.uint32))


def test_noalloc_rejects_problems_beyond_its_scratch():
    import lut_clustered_weight_b200 as cq
    M, K, N = 16, 9728, 32768
    while cq.cq_lut_gemm_workspace_size(M, N, K, 4) <= cq.NOALLOC_SCRATCH_BYTES:
        N *= 2                       # until the scratch the plan needs exceeds the array
    fake = 1 << 20                   # never dereferenced: the check runs first
    rc = cq.lib.cq_lut_gemm_noalloc(fake, fake, M, K, 4, fake, fake, N, fake, None)
    assert rc == cq.CQ_ERR_UNSUPPORTED
