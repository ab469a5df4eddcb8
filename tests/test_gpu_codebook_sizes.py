"""Adaptive codebook size on the GPU: cq_lut_gemm_ex with 8 / 16 / 32
centroids per row (3 / 4 / 5-bit indices) against the oracle, through the C
ABI, on the single-linear and Qwen3-4B-shaped FFN shapes plus ragged ones."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

DEV = "cuda"

CASES = [
    # (M, K, N, act_bits)
    (1, 2048, 2048, 4),       # the single linear
    (4, 2560, 9728, 8),       # Qwen3-4B-shaped gate (up has the same shape)
    (16, 9728, 2560, 4),      # Qwen3-4B-shaped down
    (1, 96, 64, 8),           # ragged: K not a multiple of 128
    (9, 160, 128, 4),
    (40, 1408, 192, 8),       # several token tiles
]


def _inputs(M, K, N, bits, b, seed):
    g = np.random.default_rng(seed)
    qmax = 2 ** (bits - 1) - 1
    q = g.integers(-qmax, qmax + 1, (M, K)).astype(np.int8)
    q[0, : min(K, 5)] = qmax
    s = (g.random(M) * 0.05 + 1e-3).astype(np.float32)
    w_idx, cb = synth.lut_weights(N, K, seed=seed, name=f"cbsz{M}.{K}.{N}.{b}", idx_bits=b)
    return q, s, w_idx, cb


@pytest.mark.parametrize("b", [3, 5])
@pytest.mark.parametrize("M,K,N,bits", CASES)
def test_lut_gemm_ex_parity(M, K, N, bits, b):
    import lut_clustered_weight_b200 as cq
    q, s, w_idx, cb = _inputs(M, K, N, bits, b, seed=M + K + N + b)
    assert w_idx.shape == (N, K * b // 8) and cb.shape == (N, 2 ** b)
    y = cq.cq_lut_gemm_ex(torch.from_numpy(oracle.pack_codes(q, bits)).to(DEV),
                          torch.from_numpy(s).to(DEV), K, bits, torch.from_numpy(w_idx).to(DEV), b,
                          torch.from_numpy(cb).to(DEV))
    torch.cuda.synchronize()
    yr, mag = oracle.lut_gemm_bits(q, s, w_idx, b, cb)
    err = np.abs(y.cpu().numpy().astype(np.float64) - yr)
    tol = oracle.lut_tolerance(mag)
    assert np.all(err <= tol), f"worst err/tol {(err / tol).max()}"


def test_lut_gemm_ex_4_bits_is_cq_lut_gemm():
    import lut_clustered_weight_b200 as cq
    q, s, w_idx, cb = _inputs(4, 2560, 512, 4, 4, seed=7)
    args = (torch.from_numpy(oracle.pack_codes(q, 4)).to(DEV), torch.from_numpy(s).to(DEV), 2560, 4)
    w, c = torch.from_numpy(w_idx).to(DEV), torch.from_numpy(cb).to(DEV)
    y4 = cq.cq_lut_gemm_ex(*args, w, 4, c)
    y = cq.cq_lut_gemm(*args, w, c)
    torch.cuda.synchronize()
    assert np.array_equal(y4.cpu().numpy().view(np.uint32), y.cpu().numpy().view(np.uint32))


def test_lut_gemm_ex_rejects_other_widths():
    import lut_clustered_weight_b200 as cq
    fake = 1 << 20                   # never dereferenced: the check runs first
    for b in (2, 6, 8):
        rc = cq.lib.cq_lut_gemm_ex(fake, fake, 1, 64, 4, fake, b, fake, 64, fake, fake, 1 << 20,
                                   None)
        assert rc == cq.CQ_ERR_UNSUPPORTED
