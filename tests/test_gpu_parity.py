"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from moe_check import check_moe, moe_inputs_cached, run_moe

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def cq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import lut_clustered_weight_b200 as m
    return m


def _codes_to_dev(q, bits):
    return torch.from_numpy(oracle.pack_codes(q, bits)).to(DEV)


# ---------------------------------------------------------------------------
# rotate + quantize


RQ_CASES = [
    # (M, K, b, bits, outliers)
    (1, 2048, 2048, 4, 4),
    (3, 2560, 512, 4, 4),
    (5, 2560, 512, 8, 4),
    (7, 9728, 256, 4, 4),
    (2, 9728, 256, 8, 0),
    (4, 1408, 128, 4, 8),
    (2, 768, 256, 8, 0),
    (2, 4096, 4096, 8, 4),
    (2, 14336, 2048, 8, 4),
    (2, 8192, 8192, 4, 4),
    (3, 16384, 16, 4, 2),
    (6, 8, 8, 4, 0),
    (5, 24, 1, 8, 1),
    (33, 64, 4, 4, 0),
    (0, 256, 256, 4, 0),
    # many rows, blocks of at most 1024: a row in registers, 32 positions per
    # thread (blocks of 1 to 1024: 0 to 5 levels across threads)
    (600, 1408, 128, 4, 8),
    (700, 4096, 256, 8, 4),
    (593, 64, 8, 4, 0),
    (400, 2048, 1024, 4, 4),
    (320, 1536, 512, 8, 2),
    (301, 96, 32, 4, 0),
    (310, 224, 1, 8, 1),
    (333, 4096, 64, 4, 3),
    # blocks over 1024: levels across warps through shared memory
    (300, 2048, 2048, 4, 4),
    (320, 4096, 4096, 8, 3),
    (296, 8192, 8192, 4, 2),
]


@pytest.mark.parametrize("M,K,b,bits,outl", RQ_CASES)
def test_rotate_quantize_bit_exact(cq, M, K, b, bits, outl):
    x = synth.activations(M, K, seed=1, name=f"rq{M}.{K}.{b}", n_outliers=min(outl, K))
    if M >= 3:
        x[1] = 0                        # zero row
        x[2, : min(K, 7)] = 65504.0      # largest fp16
        x[2, min(K, 7):] *= np.float16(1e-3)
    xd = torch.from_numpy(x).to(DEV)
    q, s = cq.cq_rotate_quantize(xd, b, bits)
    torch.cuda.synchronize()
    qr, sr = oracle.rotate_quantize(x, b, bits)
    qg = oracle.unpack_codes(q.cpu().numpy(), K, bits)
    assert np.array_equal(qg, qr)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), sr.view(np.uint32))


def test_rotate_quantize_exact_ties(cq):
    # b = 1: x_rot = x; with A = 14 every odd x lands on a tie for int4
    x = np.array([[14, 1, 3, 5, -7, 9, -11, 13] * 4], dtype=np.float16)
    for bits in (4, 8):
        q, s = cq.cq_rotate_quantize(torch.from_numpy(x).to(DEV), 1, bits)
        qr, sr = oracle.rotate_quantize(x, 1, bits)
        assert np.array_equal(oracle.unpack_codes(q.cpu().numpy(), 32, bits), qr)
        assert s.item() == sr[0]


@pytest.mark.parametrize("b", [32, 128, 1024, 2048])
def test_rotate_quantize_exact_ties_many_rows(cq, b):
    # x = (10.5, 3.5, 0, ...) per block: the Walsh-Hadamard outputs alternate
    # 14 and 7, so A = 14 and every 7 lands exactly on a tie for int4 (7 * 7 /
    # 14 = 3.5) -- with hundreds of rows, on the register-resident kernel
    M, K = 320, 2048
    x = np.zeros((M, K), dtype=np.float16)
    x[:, 0::b] = 10.5
    x[:, 1::b] = 3.5
    x[1::2] *= -1                       # negative rows: ties on the other side
    x[5, :] = 0                         # a zero row
    x[7, 2::b] = 0.25                   # no longer exact ties on row 7
    for bits in (4, 8):
        q, s = cq.cq_rotate_quantize(torch.from_numpy(x).to(DEV), b, bits)
        torch.cuda.synchronize()
        qr, sr = oracle.rotate_quantize(x, b, bits)
        assert np.array_equal(oracle.unpack_codes(q.cpu().numpy(), K, bits), qr)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), sr.view(np.uint32))


RQ_SP_CASES = [
    # (M, K, b, bits, scale, perm): one CTA / cluster per row, and the
    # warp-per-row kernel (many rows, b <= 256)
    (3, 2560, 512, 4, True, True),
    (2, 2048, 2048, 8, True, False),
    (5, 9728, 256, 4, False, True),
    (700, 1408, 128, 8, True, True),
    (600, 2048, 256, 4, False, True),
    (400, 2048, 2048, 4, True, True),
]


@pytest.mark.parametrize("M,K,b,bits,use_scale,use_perm", RQ_SP_CASES)
def test_rotate_quantize_scale_perm_bit_exact(cq, M, K, b, bits, use_scale, use_perm):
    """Online smoothing scale and channel grouping ahead of the rotation."""
    g = np.random.default_rng(M + K)
    x = synth.activations(M, K, seed=2, name=f"rqsp{M}.{K}")
    scale = (g.random(K) * 1.5 + 0.05).astype(np.float16) if use_scale else None
    perm = g.permutation(K).astype(np.int32) if use_perm else None
    dev = lambda a: None if a is None else torch.from_numpy(a).to(DEV)
    q, s = cq.cq_rotate_quantize(dev(x), b, bits, scale=dev(scale), perm=dev(perm))
    torch.cuda.synchronize()
    qr, sr = oracle.rotate_quantize(x, b, bits, scale=scale, perm=perm)
    assert np.array_equal(oracle.unpack_codes(q.cpu().numpy(), K, bits), qr)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), sr.view(np.uint32))


def test_moe_with_smoothing_scale_and_channel_order(cq):
    """The layer input's smoothing scale / channel order reach the x codes."""
    shape = synth.MoEShape("moe_scaled_perm", H=256, I=192, E=8, top_k=2, n_shared=1, T=24,
                           act_bits=4, had_block_h=64, had_block_i=64)
    inp = synth.moe_inputs(shape, seed=3)
    g = np.random.default_rng(5)
    inp.extra["x_scale"] = (g.random(256) + 0.25).astype(np.float16)
    inp.extra["x_perm"] = g.permutation(256).astype(np.int32)
    res = run_moe(inp)
    st = check_moe(inp, res, e2e=True)
    assert st["e2e_rel_l2"] < 5e-2, st


# ---------------------------------------------------------------------------
# LUT GEMM


LUT_CASES = [
    # (M, K, N, bits)
    (1, 2048, 2048, 4),
    (1, 32, 64, 4),
    (3, 96, 128, 8),
    (8, 160, 64, 4),
    (9, 2560, 256, 4),
    (16, 2560, 512, 8),
    (17, 1408, 192, 4),
    (40, 768, 128, 8),
    (5, 9728, 128, 4),
    (2, 14336, 64, 8),
    # more than 16 rows and N % 128 == 0: the tcgen05 tensor-memory kernel
    (64, 2048, 256, 4),
    (130, 1408, 384, 8),
    (300, 2560, 128, 4),
    (257, 96, 256, 4),
]


def _lut_inputs(M, K, N, bits, seed):
    g = np.random.default_rng(seed)
    qmax = 2 ** (bits - 1) - 1
    q = g.integers(-qmax, qmax + 1, (M, K)).astype(np.int8)
    q[0, : min(K, 5)] = qmax
    if M > 2:
        q[2] = 0
    s = (g.random(M) * 0.05 + 1e-3).astype(np.float32)
    w_idx, cb = synth.lut_weights(N, K, seed=seed, name=f"lut{M}.{K}.{N}")
    return q, s, w_idx, cb


@pytest.mark.parametrize("M,K,N,bits", LUT_CASES)
def test_lut_gemm_parity(cq, M, K, N, bits):
    q, s, w_idx, cb = _lut_inputs(M, K, N, bits, seed=M * 7 + K + N)
    y, S = cq.cq_lut_gemm(_codes_to_dev(q, bits), torch.from_numpy(s).to(DEV), K, bits,
                          torch.from_numpy(w_idx).to(DEV), torch.from_numpy(cb).to(DEV),
                          centroid_sums=True)
    torch.cuda.synchronize()
    yr, mag, Sr = oracle.lut_gemm(q, s, w_idx, cb, centroid_sums=True)
    err = np.abs(y.cpu().numpy().astype(np.float64) - yr)
    tol = oracle.lut_tolerance(mag)
    assert np.all(err <= tol), f"max excess {(err - tol).max()}, worst ratio {(err / tol).max()}"
    assert np.array_equal(S.cpu().numpy(), Sr)


def test_lut_gemm_config0_full(cq):
    """Linear M=1, K=N=2048, A4W4 with the real rotate+quantize front end."""
    s = synth.CFG0
    x, w_idx, cb = synth.linear_inputs(s)
    xd = torch.from_numpy(x).to(DEV)
    q, sx = cq.cq_rotate_quantize(xd, s.had_block, s.act_bits)
    y = cq.cq_lut_gemm(q, sx, s.K, s.act_bits, torch.from_numpy(w_idx).to(DEV),
                       torch.from_numpy(cb).to(DEV))
    torch.cuda.synchronize()
    qr, sr = oracle.rotate_quantize(x, s.had_block, s.act_bits)
    assert np.array_equal(oracle.unpack_codes(q.cpu().numpy(), s.K, 4), qr)
    yr, mag, _ = oracle.lut_gemm(qr, sr, w_idx, cb)
    err = np.abs(y.cpu().numpy() - yr)
    assert np.all(err <= oracle.lut_tolerance(mag))


def test_lut_gemm_repeatable(cq):
    """Split-K partials are reduced in a fixed order: bitwise repeatable."""
    q, s, w_idx, cb = _lut_inputs(4, 9728, 128, 4, seed=3)
    args = (_codes_to_dev(q, 4), torch.from_numpy(s).to(DEV), 9728, 4,
            torch.from_numpy(w_idx).to(DEV), torch.from_numpy(cb).to(DEV))
    y1 = cq.cq_lut_gemm(*args).cpu().numpy()
    y2 = cq.cq_lut_gemm(*args).cpu().numpy()
    assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))


# ---------------------------------------------------------------------------
# MoE / dense FFN, small shapes: every row and token checked


SMALL_MOE = [
    synth.MoEShape("dense_small", H=256, I=512, E=0, top_k=0, n_shared=1, T=5, act_bits=4,
                   had_block_h=128, had_block_i=64),
    synth.MoEShape("dense_small8", H=320, I=384, E=0, top_k=0, n_shared=1, T=16, act_bits=8,
                   had_block_h=64, had_block_i=128),
    synth.MoEShape("moe_small", H=256, I=192, E=8, top_k=2, n_shared=0, T=24, act_bits=4,
                   had_block_h=256, had_block_i=64),
    synth.MoEShape("moe_small_shared", H=192, I=128, E=6, top_k=3, n_shared=2, T=19,
                   act_bits=8, had_block_h=64, had_block_i=128, bias_expert=0, bias=1.0),
    synth.MoEShape("moe_norenorm", H=128, I=64, E=16, top_k=4, n_shared=0, T=9, act_bits=4,
                   had_block_h=128, had_block_i=64, renormalize=0),
    synth.MoEShape("moe_one_token", H=128, I=128, E=4, top_k=1, n_shared=1, T=1, act_bits=4,
                   had_block_h=32, had_block_i=32),
    # > 16 rows per expert: routed and shared experts on the tcgen05 kernel
    synth.MoEShape("moe_tc_small", H=256, I=256, E=4, top_k=2, n_shared=1, T=80, act_bits=4,
                   had_block_h=256, had_block_i=128, bias_expert=1, bias=1.0),
    synth.MoEShape("moe_tc_small8", H=384, I=192, E=2, top_k=1, n_shared=0, T=40, act_bits=8,
                   had_block_h=128, had_block_i=64),
    # hundreds of rows: 256-token tiles and the warp-per-row SwiGLU kernel
    synth.MoEShape("dense_many_rows", H=128, I=256, E=0, top_k=0, n_shared=1, T=600,
                   act_bits=4, had_block_h=128, had_block_i=64),
    synth.MoEShape("moe_many_rows", H=192, I=128, E=4, top_k=2, n_shared=1, T=320, act_bits=8,
                   had_block_h=64, had_block_i=128, I_shared=256),
    # 1400 routing slots: the grouping runs as a histogram launch and two
    # placement CTAs (chunks of 1024 slots)
    synth.MoEShape("moe_route_chunks", H=128, I=128, E=8, top_k=2, n_shared=0, T=700, act_bits=4,
                   had_block_h=128, had_block_i=64),
    # gate/up with one partial slot: SwiGLU in the tensor-core epilogue (fp16 h)
    synth.MoEShape("moe_fused_t64", H=384, I=768, E=16, top_k=2, n_shared=0, T=200, act_bits=4,
                   had_block_h=128, had_block_i=256),
    synth.MoEShape("moe_fused_i1024", H=256, I=1024, E=8, top_k=2, n_shared=0, T=320,
                   act_bits=8, had_block_h=256, had_block_i=256, bias_expert=3, bias=0.5),
]


@pytest.mark.parametrize("shape", SMALL_MOE, ids=lambda s: s.name)
def test_moe_small_full_parity(cq, shape):
    inp = moe_inputs_cached(shape)
    g = run_moe(inp)
    st = check_moe(inp, g, e2e=True)
    assert st["e2e_rel_l2"] < 5e-2, st


# ---------------------------------------------------------------------------
# the five workloads at full size, sampled rows / tokens


@pytest.mark.slow
@pytest.mark.parametrize("M,bits", synth.CFG1_VARIANTS)
def test_config1_dense_ffn(cq, M, bits):
    inp = moe_inputs_cached(synth.cfg1(M, bits))
    g = run_moe(inp)
    check_moe(inp, g, sample_rows=4, sample_tokens=4)


@pytest.mark.slow
def test_config2_qwen3_30b_moe(cq):
    inp = moe_inputs_cached(synth.CFG2)
    g = run_moe(inp)
    check_moe(inp, g, sample_rows=12, sample_tokens=6)


@pytest.mark.slow
def test_config3_mixtral_moe(cq):
    inp = moe_inputs_cached(synth.CFG3)
    g = run_moe(inp)
    check_moe(inp, g, sample_rows=4, sample_tokens=4)


@pytest.mark.slow
def test_dense_prefill_fused_epilogue(cq):
    """A dense SwiGLU FFN at prefill size: the gate/up launch takes whole work
    items per CTA with one partial slot, so SwiGLU runs in its epilogue."""
    s = synth.MoEShape("dense_prefill_fused", H=128, I=4096, E=0, top_k=0, n_shared=1, T=2048,
                       act_bits=4, had_block_h=128, had_block_i=256)
    inp = moe_inputs_cached(s)
    g = run_moe(inp)
    check_moe(inp, g, sample_rows=8, sample_tokens=8)


@pytest.mark.slow
def test_config4_prefill_moe(cq):
    inp = moe_inputs_cached(synth.CFG4)
    g = run_moe(inp)
    check_moe(inp, g, sample_rows=6, sample_tokens=4)
