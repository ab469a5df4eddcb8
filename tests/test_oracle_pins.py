"""Pins for the CPU oracle: each check ties it to something other than itself --
hand-worked values, closed forms, invariants, library routines (numpy,
scipy), or exact brute force with Python integers / fractions."""
from fractions import Fraction
import math

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------------------
# fp16 conversions


def test_f16_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(b) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_f16_encode_rne_matches_numpy():
    g = np.random.default_rng(1)
    v = np.concatenate([
        g.standard_normal(20000) * 10.0 ** g.integers(-9, 5, 20000),
        # exact midpoints between neighbouring fp16 values (ties)
        (np.arange(0, 30000, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
         + np.arange(1, 30001, 7, dtype=np.uint16).view(np.float16).astype(np.float64)) / 2,
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, 2.0 ** -25, 2.0 ** -24, 3 * 2.0 ** -26,
         2.0 ** -14, 2.0 ** -14 - 2.0 ** -25],
    ])
    v = np.concatenate([v, -v])
    ref = v.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f64_to_f16(x) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# Hadamard rotation


@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 64, 256])
def test_hadamard_is_sylvester_and_orthogonal(b):
    H = oracle.hadamard(b)
    assert np.array_equal(H, scipy.linalg.hadamard(b).astype(np.float64))
    assert np.array_equal(H @ H.T, b * np.eye(b))
    assert np.array_equal(H, H.T)


def _fwht_ints(v):
    """Recursive Walsh-Hadamard (Sylvester) transform on Python ints."""
    n = len(v)
    if n == 1:
        return list(v)
    a = _fwht_ints(v[: n // 2])
    c = _fwht_ints(v[n // 2:])
    return [x + y for x, y in zip(a, c)] + [x - y for x, y in zip(a, c)]


@pytest.mark.parametrize("K,b", [(8, 8), (32, 8), (64, 16), (48, 16), (256, 256)])
def test_rotate_exact_against_integer_fwht(K, b):
    g = np.random.default_rng(K * 31 + b)
    x = (g.standard_normal((3, K)) * 10.0 ** g.integers(-6, 4, (3, K))).astype(np.float16)
    x[0, 5] = np.float16(65504.0)
    got = oracle.rotate(x, b)
    for m in range(x.shape[0]):
        # fp16 values as exact integers in units of 2^-24
        units = [int(Fraction(float(v)) * 2 ** 24) for v in x[m].astype(np.float64)]
        ref = []
        for blk in range(K // b):
            ref += _fwht_ints(units[blk * b:(blk + 1) * b])
        assert [int(Fraction(float(v)) * 2 ** 24) for v in got[m]] == ref


def test_rotate_parseval_and_block_structure():
    g = np.random.default_rng(7)
    x = g.standard_normal((4, 512)).astype(np.float16)
    b = 128
    xr = oracle.rotate(x, b)
    xd = x.astype(np.float64)
    for blk in range(4):
        sl = slice(blk * b, (blk + 1) * b)
        np.testing.assert_allclose((xr[:, sl] ** 2).sum(1), b * (xd[:, sl] ** 2).sum(1),
                                   rtol=1e-12)
    # kron(I, H_b) with scipy's Hadamard as a library reduction
    R = np.kron(np.eye(4), scipy.linalg.hadamard(b))
    np.testing.assert_array_equal(xr, xd @ R)


# ---------------------------------------------------------------------------
# quantization


def _brute_quant(xr_row, b, bits):
    qmax = 2 ** (bits - 1) - 1
    fr = [Fraction(float(v)) for v in xr_row]
    A = max(abs(v) for v in fr)
    if A == 0:
        return [0] * len(fr), 0.0
    q = []
    for v in fr:
        t = qmax * v / A
        fl = math.floor(t)
        rem = t - fl
        if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
            fl += 1
        q.append(int(fl))
    return q, float(A)


@pytest.mark.parametrize("bits", [4, 8])
def test_quantize_matches_fraction_brute_force(bits):
    g = np.random.default_rng(bits)
    for trial in range(200):
        K = int(g.choice([2, 4, 6]))
        xr = (g.integers(-3000, 3000, K) * 2.0 ** int(g.integers(-24, 3))).astype(np.float64)
        q, s = oracle.quantize(xr[None, :], 1, bits)
        qb, A = _brute_quant(xr, 1, bits)
        assert q[0].tolist() == qb
        qmax = 2 ** (bits - 1) - 1
        assert s[0] == np.float32(A / qmax)


@pytest.mark.parametrize("bits", [4, 8])
def test_quantize_ties_round_to_even(bits):
    qmax = 2 ** (bits - 1) - 1
    # x / A = (2j + 1) / (2 qmax): exact ties j + 1/2
    A = 2 * qmax
    row = np.array([A] + [2 * j + 1 for j in range(qmax)], dtype=np.float64)
    q, _ = oracle.quantize(row[None, :], 1, bits)
    expect = [qmax] + [j if j % 2 == 0 else j + 1 for j in range(qmax)]
    assert q[0].tolist() == expect
    q2, _ = oracle.quantize(-row[None, :], 1, bits)
    assert q2[0].tolist() == [-v for v in expect]


@pytest.mark.parametrize("bits", [4, 8])
def test_quantize_properties(bits):
    g = np.random.default_rng(11 + bits)
    x = (g.standard_normal((16, 256)) * 3).astype(np.float16)
    b = 64
    xr = oracle.rotate(x, b)
    q, s = oracle.quantize(xr, b, bits)
    qmax = 2 ** (bits - 1) - 1
    assert q.min() >= -qmax and q.max() <= qmax
    am = np.argmax(np.abs(xr), axis=1)
    assert np.array_equal(np.abs(q[np.arange(16), am]), np.full(16, qmax))
    # dequantization error of the normalised rotation is at most half a step
    err = np.abs(xr / math.sqrt(b) - s[:, None].astype(np.float64) * q)
    assert np.all(err <= s[:, None].astype(np.float64) * 0.5 * (1 + 1e-6) + 1e-30)
    # exact scale invariance: q(2^j x) = q(x)
    for j in (-3, 5):
        q2, s2 = oracle.quantize(xr * 2.0 ** j, b, bits)
        assert np.array_equal(q2, q)
        np.testing.assert_array_equal(s2, (s.astype(np.float64) * 2.0 ** j).astype(np.float32))


def test_rotate_quantize_golden(golden_dir):
    for line in (golden_dir / "rotate_quantize_worked.txt").read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        head, xs, qs, ss = [p.strip() for p in line.split("|")]
        b, bits = map(int, head.split())
        x = np.array([float(v) for v in xs.split()], dtype=np.float16)[None, :]
        q, s = oracle.rotate_quantize(x, b, bits)
        assert q[0].tolist() == [int(v) for v in qs.split()], line
        assert s[0] == np.float32(float(ss)), line


def test_pack_unpack_int4_roundtrip():
    g = np.random.default_rng(3)
    q = g.integers(-7, 8, (5, 64)).astype(np.int8)
    p = oracle.pack_codes(q, 4)
    assert p.shape == (5, 32)
    lo = (p & 15).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    assert np.array_equal(np.where(lo >= 8, lo - 16, lo), q[:, 0::2])
    assert np.array_equal(np.where(hi >= 8, hi - 16, hi), q[:, 1::2])
    assert np.array_equal(oracle.unpack_codes(p, 64, 4), q)


# ---------------------------------------------------------------------------
# LUT product


def _rand_lut(g, M, K, N, bits=4):
    qmax = 2 ** (bits - 1) - 1
    q = g.integers(-qmax, qmax + 1, (M, K)).astype(np.int8)
    s = (g.random(M) + 0.1).astype(np.float32)
    idx = g.integers(0, 16, (N, K)).astype(np.uint8)
    cb = (g.standard_normal((N, 16)) * 0.05).astype(np.float16)
    w_idx = (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8)
    return q, s, idx, w_idx, cb


def test_lut_gemm_dense_dequant_matmul():
    g = np.random.default_rng(5)
    q, s, idx, w_idx, cb = _rand_lut(g, 7, 96, 33, bits=8)
    y, mag, S = oracle.lut_gemm(q, s, w_idx, cb, centroid_sums=True)
    W = np.take_along_axis(cb.astype(np.float64), idx.astype(np.int64), axis=1)  # [N, K]
    ref = s.astype(np.float64)[:, None] * (q.astype(np.float64) @ W.T)
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(mag, np.abs(s)[:, None] * (np.abs(q) @ np.abs(W).T),
                               rtol=1e-13, atol=1e-15)
    # centroid sums: a library histogram per (m, n)
    for m in range(q.shape[0]):
        for n in range(idx.shape[0]):
            ref_S = np.bincount(idx[n], weights=q[m].astype(np.float64), minlength=16)
            assert np.array_equal(S[m, n], ref_S.astype(np.int32))
    # closed form: sum over centroids = sum over k, independent of the codebook
    assert np.array_equal(S.sum(-1), np.broadcast_to(q.sum(1, dtype=np.int64)[:, None],
                                                     S.shape[:2]))


def test_lut_gemm_uniform_grid_reduces_to_integer_gemm():
    g = np.random.default_rng(9)
    q, s, idx, w_idx, _ = _rand_lut(g, 5, 128, 17, bits=4)
    delta = 2.0 ** -7
    cb = np.tile(((np.arange(16) - 7.5) * delta).astype(np.float16), (17, 1))
    y, _, _ = oracle.lut_gemm(q, s, w_idx, cb)
    # (c - 7.5) * delta = (2c - 15) * delta / 2: integer GEMM in numpy int64
    Wi = 2 * idx.astype(np.int64) - 15
    ref = s.astype(np.float64)[:, None] * (q.astype(np.int64) @ Wi.T).astype(np.float64) * delta / 2
    np.testing.assert_array_equal(y, ref)


def test_lut_gemm_single_centroid_row():
    g = np.random.default_rng(10)
    q, s, _, _, cb = _rand_lut(g, 3, 64, 4)
    for c in (0, 7, 15):
        idx = np.full((4, 64), c, dtype=np.uint8)
        w_idx = (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8)
        y, _, _ = oracle.lut_gemm(q, s, w_idx, cb)
        ref = s.astype(np.float64)[:, None] * cb[:, c].astype(np.float64)[None, :] \
            * q.sum(1).astype(np.float64)[:, None]
        np.testing.assert_allclose(y, ref, rtol=1e-15)


def test_lut_gemm_brute_force_all_index_patterns_k2():
    g = np.random.default_rng(12)
    cb = (g.standard_normal((1, 16)) * 0.1).astype(np.float16)
    Cf = [Fraction(float(v)) for v in cb[0].astype(np.float64)]
    q = np.array([[5, -3], [-7, 7]], dtype=np.int8)
    s = np.array([0.75, 1.5], dtype=np.float32)
    pats = np.array([[a, b] for a in range(16) for b in range(16)], dtype=np.uint8)  # N=256
    w_idx = (pats[:, 0] | (pats[:, 1] << 4)).astype(np.uint8)[:, None]
    y, _, _ = oracle.lut_gemm(q, s, w_idx, np.repeat(cb, 256, axis=0))
    for n, (a, b) in enumerate(pats):
        for m in range(2):
            exact = Fraction(float(s[m])) * (Cf[a] * int(q[m, 0]) + Cf[b] * int(q[m, 1]))
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)


def test_lut_gemm_golden(golden_dir):
    q = np.array([[3, -2, 7, 1]], dtype=np.int8)
    s = np.array([0.5], dtype=np.float32)
    cb = np.stack([np.arange(16) * 0.25, -np.arange(16.0)]).astype(np.float16)
    rows = []
    for line in (golden_dir / "lut_gemm_worked.txt").read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        n, ids, yv, sv = [p.strip() for p in line.split("|")]
        rows.append((int(n), [int(v) for v in ids.split()], float(yv),
                     {int(a): int(b) for a, b in (t.split(":") for t in sv.split())}))
    idx = np.array([r[1] for r in rows], dtype=np.uint8)
    w_idx = (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8)
    y, _, S = oracle.lut_gemm(q, s, w_idx, cb, centroid_sums=True)
    for n, _, yv, sv in rows:
        assert y[0, n] == yv
        ref = np.zeros(16, dtype=np.int32)
        for c, v in sv.items():
            ref[c] = v
        assert np.array_equal(S[0, n], ref)


# ---------------------------------------------------------------------------
# routing


def test_route_golden(golden_dir):
    d = {}
    for line in (golden_dir / "route_worked.txt").read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        key, rest = line.split(" ", 1)
        d[key] = [[float(v) for v in part.split()] for part in rest.split("|")]
    lg = np.array(d["logits"], dtype=np.float32)
    r = oracle.route(lg, 2, True)
    assert r["ids"].tolist() == [[int(v) for v in row] for row in d["ids"]]
    np.testing.assert_allclose(r["w"], np.array(d["w"]), rtol=1e-15)
    assert r["counts"].tolist() == [int(v) for v in d["counts"][0]]
    assert r["offsets"].tolist() == [int(v) for v in d["offsets"][0]]
    assert r["perm"].tolist() == [int(v) for v in d["perm"][0]]


@pytest.mark.parametrize("T,E,k,renorm", [(64, 128, 8, True), (256, 8, 2, True),
                                          (100, 64, 6, False), (33, 16, 16, True)])
def test_route_against_stable_argsort(T, E, k, renorm):
    g = np.random.default_rng(T + E)
    lg = g.standard_normal((T, E)).astype(np.float32)
    lg[::3, 1] = lg[::3, 0]            # plant ties
    lg[5, :] = 0.25
    r = oracle.route(lg, k, renorm)
    ref_ids = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    assert np.array_equal(r["ids"], ref_ids)
    if renorm:
        ref_w = scipy.special.softmax(np.take_along_axis(lg, ref_ids, 1).astype(np.float64), 1)
    else:
        ref_w = np.take_along_axis(scipy.special.softmax(lg.astype(np.float64), 1), ref_ids, 1)
    np.testing.assert_allclose(r["w"], ref_w, rtol=1e-13)
    assert r["counts"].sum() == T * k
    assert np.array_equal(r["counts"], np.bincount(ref_ids.ravel(), minlength=E))
    assert np.array_equal(r["offsets"], np.concatenate([[0], np.cumsum(r["counts"])]))
    perm = r["perm"]
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    # grouped by expert, stable inside each group, gather then scatter = identity
    flat = r["ids"].ravel()
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    x = g.standard_normal((T * k, 3))
    back = np.empty_like(x)
    back[perm] = x[perm]
    assert np.array_equal(back, x)


# ---------------------------------------------------------------------------
# SwiGLU and combine


def test_swiglu_against_torch_silu():
    g = np.random.default_rng(21)
    a = g.standard_normal(5000) * 4
    u = g.standard_normal(5000) * 3
    h = oracle.swiglu(a, u)
    ref = (torch.nn.functional.silu(torch.from_numpy(a)) * torch.from_numpy(u)).numpy()
    assert np.array_equal(h.view(np.uint16), ref.astype(np.float16).view(np.uint16))
    assert np.all(oracle.swiglu(np.zeros(4), np.ones(4)) == 0)


def test_combine_closed_forms():
    g = np.random.default_rng(22)
    T, k, H = 5, 3, 7
    y = g.standard_normal((T * k, H))
    w = np.zeros((T, k))
    w[np.arange(T), np.arange(T) % k] = 1.0
    out = oracle.combine(y, w)
    np.testing.assert_array_equal(out, y.reshape(T, k, H)[np.arange(T), np.arange(T) % k])
    ysh = g.standard_normal((2, T, H))
    out2 = oracle.combine(y, np.zeros((T, k)), ysh)
    np.testing.assert_allclose(out2, ysh.sum(0), rtol=1e-15)


# ---------------------------------------------------------------------------
# MoE composition


def _tiny_moe(E, k, n_shared, T=6, H=64, I=32, seed=0):
    import synth
    s = synth.MoEShape("tiny", H=H, I=I, E=E, top_k=k, n_shared=n_shared, T=T, act_bits=4,
                       had_block_h=32, had_block_i=16)
    return synth.moe_inputs(s, seed=seed)


def test_moe_single_expert_top1_equals_dense_ffn():
    import synth
    inp = _tiny_moe(E=1, k=1, n_shared=0)
    r = oracle.moe_ffn(inp)
    dense = synth.MoEInputs(inp.shape, inp.x, None, sh_gate_idx=inp.gate_idx,
                            sh_up_idx=inp.up_idx, sh_down_idx=inp.down_idx,
                            sh_gate_cb=inp.gate_cb, sh_up_cb=inp.up_cb, sh_down_cb=inp.down_cb)
    ds = synth.MoEShape("tiny", H=64, I=32, E=0, top_k=0, n_shared=1, T=6, act_bits=4,
                        had_block_h=32, had_block_i=16)
    rd = oracle.moe_ffn(dense, ds)
    np.testing.assert_array_equal(r["out"], rd["out"])


def test_moe_identical_experts_equal_dense_ffn():
    import synth
    inp = _tiny_moe(E=4, k=2, n_shared=0)
    for a in ("gate_idx", "up_idx", "down_idx", "gate_cb", "up_cb", "down_cb"):
        arr = getattr(inp, a)
        setattr(inp, a, np.repeat(arr[:1], 4, axis=0))
    r = oracle.moe_ffn(inp)
    ds = synth.MoEShape("tiny", H=64, I=32, E=0, top_k=0, n_shared=1, T=6, act_bits=4,
                        had_block_h=32, had_block_i=16)
    dense = synth.MoEInputs(ds, inp.x, None, sh_gate_idx=inp.gate_idx[:1],
                            sh_up_idx=inp.up_idx[:1], sh_down_idx=inp.down_idx[:1],
                            sh_gate_cb=inp.gate_cb[:1], sh_up_cb=inp.up_cb[:1],
                            sh_down_cb=inp.down_cb[:1])
    rd = oracle.moe_ffn(dense, ds)
    np.testing.assert_allclose(r["out"], rd["out"], rtol=1e-12, atol=1e-12)


def test_planted_mistakes_are_caught():
    """A dropped term / wrong sign / transposed operand in the LUT product
    would break the dense-dequant reduction: check the reduction notices."""
    g = np.random.default_rng(31)
    q, s, idx, w_idx, cb = _rand_lut(g, 3, 32, 5)
    y, _, _ = oracle.lut_gemm(q, s, w_idx, cb)
    W = np.take_along_axis(cb.astype(np.float64), idx.astype(np.int64), axis=1)
    ref = s.astype(np.float64)[:, None] * (q.astype(np.float64) @ W.T)
    bad_drop = s.astype(np.float64)[:, None] * (q[:, 1:].astype(np.float64) @ W[:, 1:].T)
    bad_nib = (idx[:, 1::2] | (idx[:, 0::2] << 4)).astype(np.uint8)   # swapped nibbles
    y_swap, _, _ = oracle.lut_gemm(q, s, bad_nib, cb)
    assert np.allclose(y, ref, rtol=1e-12)
    assert not np.allclose(bad_drop, ref, rtol=1e-6)
    assert not np.allclose(y_swap, ref, rtol=1e-6)


# ---------------------------------------------------------------------------
# online smoothing scale and channel grouping ahead of the rotation


def _f16_nearest_fraction(v: Fraction) -> float:
    """The fp16 value nearest to the exact rational v, ties to even (written
    from the format: 11 significant bits, exponent >= -14, subnormal quantum
    2^-24), independent of the oracle's encoder and of numpy."""
    if v == 0:
        return 0.0
    a = abs(v)
    e = max(math.floor(math.log2(a)), -14)
    while Fraction(2) ** e > a:          # guard the float log2
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -14)
    quantum = Fraction(2) ** (e - 10)
    n = a / quantum
    lo = math.floor(n)
    r = n - lo
    n = lo + 1 if (r > Fraction(1, 2) or (r == Fraction(1, 2) and lo % 2 == 1)) else lo
    out = float(n * quantum)
    return -out if v < 0 else out


def test_scale_rounds_the_exact_product_to_nearest_even():
    g = np.random.default_rng(41)
    x = (g.standard_normal((3, 64)) * np.array([1, 1e-4, 300.0])[:, None]).astype(np.float16)
    s = (g.random(64) * 4 + 0.01).astype(np.float16)
    out = oracle.scale_permute(x, scale=s)
    # numpy: the fp64 product of two fp16 values is exact; astype rounds to nearest even
    ref = (x.astype(np.float64) * s.astype(np.float64)).astype(np.float16)
    np.testing.assert_array_equal(out.view(np.uint16), ref.view(np.uint16))
    # exact rationals on a sample, including subnormal results
    for (m, k) in [(0, 0), (1, 5), (1, 17), (2, 63), (0, 31)]:
        exact = Fraction(float(x[m, k])) * Fraction(float(s[k]))
        assert float(out[m, k]) == _f16_nearest_fraction(exact)


def test_scale_ties_go_to_even():
    # exact products: 2050 * 0.5 = 1025 and 2054 * 0.25 = 513.5 are fp16 numbers
    x2 = np.array([[2050.0, 2054.0]], dtype=np.float16)
    out = oracle.scale_permute(x2, scale=np.array([0.5, 0.25], dtype=np.float16))
    assert float(out[0, 0]) == 1025.0 and float(out[0, 1]) == 513.5
    # 1025 * 1.5 = 1537.5 and 1027 * 1.5 = 1540.5 lie halfway between fp16
    # neighbours (spacing 1 in [1024, 2048)): ties go to the even one
    h = np.array([[1025.0, 1027.0]], dtype=np.float16)
    out = oracle.scale_permute(h, scale=np.array([1.5, 1.5], dtype=np.float16))
    assert float(out[0, 0]) == 1538.0 and float(out[0, 1]) == 1540.0


def test_permutation_gathers_channels():
    g = np.random.default_rng(43)
    x = g.standard_normal((4, 32)).astype(np.float16)
    perm = g.permutation(32).astype(np.int32)
    out = oracle.scale_permute(x, perm=perm)
    np.testing.assert_array_equal(out, x[:, perm])          # out[:, j] = x[:, perm[j]]
    assert not np.array_equal(out, x[:, np.argsort(perm)])  # not the scatter
    s = (g.random(32) + 0.5).astype(np.float16)
    both = oracle.scale_permute(x, scale=s, perm=perm)
    ref = (x.astype(np.float64) * s.astype(np.float64)).astype(np.float16)[:, perm]
    np.testing.assert_array_equal(both.view(np.uint16), ref.view(np.uint16))


def test_permutation_must_be_a_permutation():
    x = np.zeros((1, 8), dtype=np.float16)
    for bad in ([0, 1, 2, 3, 4, 5, 6, 6], [0, 1, 2, 3, 4, 5, 6, 8], [-1, 1, 2, 3, 4, 5, 6, 7]):
        with pytest.raises(ValueError):
            oracle.scale_permute(x, perm=np.array(bad, dtype=np.int32))


@pytest.mark.parametrize("bits", [4, 8])
def test_power_of_two_scale_keeps_codes_and_scales_s(bits):
    g = np.random.default_rng(47)
    x = g.standard_normal((5, 256)).astype(np.float16)
    q0, s0 = oracle.rotate_quantize(x, 64, bits)
    q1, s1 = oracle.rotate_quantize(x, 64, bits, scale=np.full(256, 0.25, np.float16))
    np.testing.assert_array_equal(q0, q1)
    np.testing.assert_array_equal(s1, s0 * np.float32(0.25))


@pytest.mark.parametrize("bits", [4, 8])
def test_block_permutation_permutes_the_rotated_blocks(bits):
    """Moving whole rotation blocks permutes the rotated blocks; the absmax is
    over the whole row, so codes move with them and the scale is unchanged."""
    g = np.random.default_rng(53)
    b, nb = 32, 6
    x = g.standard_normal((3, b * nb)).astype(np.float16)
    order = g.permutation(nb)
    perm = np.concatenate([np.arange(o * b, o * b + b) for o in order]).astype(np.int32)
    q0, s0 = oracle.rotate_quantize(x, b, bits)
    q1, s1 = oracle.rotate_quantize(x, b, bits, perm=perm)
    np.testing.assert_array_equal(q1, q0[:, perm])
    np.testing.assert_array_equal(s1, s0)


def test_permuted_input_and_weights_give_the_same_product():
    """With b = 1 (no mixing) the codes move with the channels, so permuting
    the activations and the weights' columns alike leaves y unchanged."""
    g = np.random.default_rng(59)
    K, N = 64, 16
    x = g.standard_normal((3, K)).astype(np.float16)
    perm = g.permutation(K).astype(np.int32)
    q, s = oracle.rotate_quantize(x, 1, 4)
    qp, sp = oracle.rotate_quantize(x, 1, 4, perm=perm)
    np.testing.assert_array_equal(qp, q[:, perm])
    idx = g.integers(0, 16, (N, K)).astype(np.uint8)
    cb = (g.standard_normal((N, 16)) * 0.02).astype(np.float16)
    pack = lambda v: (v[:, 0::2] | (v[:, 1::2] << 4)).astype(np.uint8)
    y, _, _ = oracle.lut_gemm(q, s, pack(idx), cb)
    yp, _, _ = oracle.lut_gemm(qp, sp, pack(idx[:, perm]), cb)
    np.testing.assert_allclose(yp, y, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------
# adaptive codebook size: 8 / 16 / 32 centroids, 3 / 4 / 5-bit indices


def _np_unpack_bits(p, K, b):
    """Independent reading of the b-bit format: index k = bits [b*k, b*k+b),
    least significant first, via numpy's little-endian bit unpacking."""
    bits = np.unpackbits(np.asarray(p, dtype=np.uint8), axis=-1, bitorder="little")
    bits = bits[..., : K * b].reshape(p.shape[:-1] + (K, b)).astype(np.int64)
    return (bits << np.arange(b)).sum(axis=-1).astype(np.uint8)


@pytest.mark.parametrize("b", [3, 4, 5])
def test_bit_packed_indices_unpack(b):
    import synth
    g = np.random.default_rng(60 + b)
    idx = g.integers(0, 2 ** b, (7, 96)).astype(np.uint8)
    p = synth.pack_bits(idx, b)
    assert p.shape == (7, 96 * b // 8)
    np.testing.assert_array_equal(_np_unpack_bits(p, 96, b), idx)
    np.testing.assert_array_equal(oracle.unpack_idx_bits(p, 96, b), idx)
    if b == 4:  # the 4-bit case is the nibble format (element 2j in the low nibble)
        np.testing.assert_array_equal(p, (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8))


@pytest.mark.parametrize("b", [3, 5])
def test_lut_gemm_bits_dense_dequant_matmul(b):
    import synth
    g = np.random.default_rng(70 + b)
    M, K, N = 4, 96, 6
    q = g.integers(-7, 8, (M, K)).astype(np.int8)
    s = (g.random(M) * 0.1 + 0.01).astype(np.float32)
    idx = g.integers(0, 2 ** b, (N, K)).astype(np.uint8)
    cb = (g.standard_normal((N, 2 ** b)) * 0.05).astype(np.float16)
    y, mag = oracle.lut_gemm_bits(q, s, synth.pack_bits(idx, b), b, cb)
    W = np.take_along_axis(cb.astype(np.float64), idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(y, s.astype(np.float64)[:, None] * (q.astype(np.float64) @ W.T),
                               rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(mag, np.abs(s.astype(np.float64))[:, None] *
                               (np.abs(q.astype(np.float64)) @ np.abs(W).T), rtol=1e-12)


@pytest.mark.parametrize("b", [3, 5])
def test_lut_gemm_bits_all_index_pairs_exact(b):
    """Every pair of indices at the first two positions (a row of K = 8, so
    that it fills whole bytes; the other codes are zero), against exact
    rationals."""
    import synth
    nc = 2 ** b
    g = np.random.default_rng(80 + b)
    cb = (g.standard_normal((1, nc)) * 0.3).astype(np.float16)
    q = np.array([[3, -5, 0, 0, 0, 0, 0, 0]], dtype=np.int8)
    s = np.array([0.125], dtype=np.float32)
    fill = g.integers(0, nc, 6)
    pairs = np.array([(i, j, *fill) for i in range(nc) for j in range(nc)], dtype=np.uint8)
    cbs = np.repeat(cb, len(pairs), axis=0)
    y, _ = oracle.lut_gemm_bits(q, s, synth.pack_bits(pairs, b), b, cbs)
    for r, (i, j) in enumerate(pairs[:, :2]):
        exact = Fraction(0.125) * (Fraction(float(cb[0, i])) * 3 + Fraction(float(cb[0, j])) * -5)
        assert y[0, r] == float(exact)


def test_lut_gemm_bits_4_agrees_with_the_16_centroid_routine():
    g = np.random.default_rng(90)
    q, s, idx, w_idx, cb = _rand_lut(g, 3, 64, 5)
    y16, mag16, _ = oracle.lut_gemm(q, s, w_idx, cb)
    y4, mag4 = oracle.lut_gemm_bits(q, s, w_idx, 4, cb)
    np.testing.assert_array_equal(y4, y16)
    np.testing.assert_array_equal(mag4, mag16)


@pytest.mark.parametrize("b", [3, 5])
def test_lut_gemm_bits_uniform_grid_is_an_integer_gemm(b):
    import synth
    nc = 2 ** b
    g = np.random.default_rng(95 + b)
    M, K, N = 3, 64, 4
    q = g.integers(-127, 128, (M, K)).astype(np.int8)
    s = np.ones(M, dtype=np.float32)
    idx = g.integers(0, nc, (N, K)).astype(np.uint8)
    delta = 2.0 ** -6
    cb = np.tile(((np.arange(nc) - nc // 2) * delta).astype(np.float16), (N, 1))
    y, _ = oracle.lut_gemm_bits(q, s, synth.pack_bits(idx, b), b, cb)
    ref = (q.astype(np.int64) @ (idx.astype(np.int64) - nc // 2).T) * delta
    np.testing.assert_array_equal(y, ref)
