"""CPU oracle for the CodeQuant LUT MoE linear layer -- TEST INFRASTRUCTURE.

Plain fp64 / int64 C loops (``cq_oracle.c``) behind ctypes, plus the
composition of those steps into the dense SwiGLU FFN and the MoE layer.
Only the tests, the smoke check and the benchmark's CPU-baseline leg may use
this package; the CUDA library never does, and the two share no code.

Passages followed (page titles as on the pages):
  * CodeQuant (abstract): activation outliers smoothed by a rotation, weight
    outliers absorbed into cluster centroids, a LUT kernel for GPU and CPU.
  * CodeQuant2 (abstract; Figure 1): rotation and scaling fused into the model;
    Figure 3: per-row centroid matrix plus binary assignment matrices;
    Figure 4: one-time LUT precompute, then table lookup.
  * CodeQuant2 Tables 1, 2, 9: the A4W4 and A8W4 precision settings.

Readings where the pages are silent (each also listed in the design notes):
  block Walsh-Hadamard in Sylvester order, unnormalised, with 1/sqrt(b) folded
  into the scale; round half to even on the exact rational; qmax = 2^(bits-1)-1;
  low nibble = even k; top-k ties to the lower expert id; softmax renormalised
  over the selected experts; combine in slot order then shared experts.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "cq_oracle.c"
_BUILD = _HERE / "_build"
_LIB = _BUILD / "liboracle.so"

_lib = None


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (-O2, no fast-math, OpenMP)."""
    _BUILD.mkdir(exist_ok=True)
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _BUILD / f"liboracle.{os.getpid()}.so"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-fno-fast-math", "-Wall", str(_SRC), "-o", str(tmp), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def set_threads(n: int) -> None:
    """Host threads the oracle's row loops may use (timing only)."""
    lib().orc_set_threads(int(n))


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(str(build()))
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        _lib.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        _lib.orc_f16_to_f64.restype = D
        _lib.orc_f64_to_f16.argtypes = [D]
        _lib.orc_f64_to_f16.restype = ctypes.c_uint16
        _lib.orc_hadamard_matrix.argtypes = [I64, P]
        _lib.orc_set_threads.argtypes = [I32]
        _lib.orc_set_threads.restype = None
        _lib.orc_rotate.argtypes = [P, I64, I64, I64, P]
        _lib.orc_quantize.argtypes = [P, I64, I64, I64, I32, P, P]
        _lib.orc_rotate_quantize.argtypes = [P, I64, I64, I64, I32, P, P]
        _lib.orc_scale_permute.argtypes = [P, I64, I64, P, P, P]
        _lib.orc_unpack_int4.argtypes = [P, I64, I64, P]
        _lib.orc_pack_int4.argtypes = [P, I64, I64, P]
        _lib.orc_unpack_idx.argtypes = [P, I64, I64, P]
        _lib.orc_unpack_idx_bits.argtypes = [P, I64, I64, I32, P]
        _lib.orc_lut_gemm_nc.argtypes = [P, P, I64, I64, P, P, I32, I64, P, P]
        _lib.orc_lut_gemm.argtypes = [P, P, I64, I64, P, P, I64, P, P, P]
        _lib.orc_route.argtypes = [P, I64, I64, I64, I32, P, P, P, P, P]
        _lib.orc_swiglu.argtypes = [P, P, I64, P]
        _lib.orc_combine.argtypes = [P, P, I64, I64, I64, P, I64, P]
        for f in ("orc_hadamard_matrix", "orc_rotate", "orc_quantize", "orc_rotate_quantize",
                  "orc_scale_permute", "orc_lut_gemm_nc",
                  "orc_lut_gemm", "orc_route"):
            getattr(_lib, f).restype = I32
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments")


# ---------------------------------------------------------------------------
# scalar helpers


def f16_to_f64(bits: int) -> float:
    return lib().orc_f16_to_f64(int(bits))


def f64_to_f16(v: float) -> int:
    return int(lib().orc_f64_to_f16(float(v)))


def f16_array_to_f64(x: np.ndarray) -> np.ndarray:
    """fp16 array -> fp64 via the oracle's own decoder."""
    bits = _c(x, np.float16).view(np.uint16).ravel()
    out = np.array([f16_to_f64(b) for b in bits], dtype=np.float64)
    return out.reshape(np.shape(x))


def hadamard(b: int) -> np.ndarray:
    H = np.empty((b, b), dtype=np.float64)
    _check(lib().orc_hadamard_matrix(b, _p(H)), "hadamard")
    return H


# ---------------------------------------------------------------------------
# rotation and quantization


def rotate(x: np.ndarray, b: int) -> np.ndarray:
    """Exact block Walsh-Hadamard rotation of fp16 rows -> fp64 [M, K]."""
    x = _c(x, np.float16)
    M, K = x.shape
    out = np.empty((M, K), dtype=np.float64)
    _check(lib().orc_rotate(_p(x.view(np.uint16)), M, K, b, _p(out)), "rotate")
    return out


def quantize(x_rot: np.ndarray, b: int, bits: int):
    """Exact per-token absmax quantization -> (q int8 [M, K] unpacked, s fp32 [M])."""
    xr = _c(x_rot, np.float64)
    M, K = xr.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty((M,), dtype=np.float32)
    _check(lib().orc_quantize(_p(xr), M, K, b, bits, _p(q), _p(s)), "quantize")
    return q, s


def scale_permute(x: np.ndarray, scale=None, perm=None) -> np.ndarray:
    """fp16 [M, K] -> fp16 [M, K]: out[m, j] = fp16(x[m, perm[j]] * scale[perm[j]])
    (the identity / 1 where perm / scale is None); ValueError unless perm is a
    permutation of 0..K-1."""
    x = _c(x, np.float16)
    M, K = x.shape
    sc = None if scale is None else _c(scale, np.float16).reshape(K)
    pm = None if perm is None else _c(perm, np.int32).reshape(K)
    out = np.empty((M, K), dtype=np.float16)
    _check(lib().orc_scale_permute(_p(x.view(np.uint16)), M, K,
                                   None if sc is None else _p(sc.view(np.uint16)), _p(pm),
                                   _p(out.view(np.uint16))), "scale_permute")
    return out


def rotate_quantize(x: np.ndarray, b: int, bits: int, scale=None, perm=None):
    """fp16 [M, K] -> (q int8 [M, K] unpacked, s fp32 [M]); with a smoothing
    scale and/or channel permutation applied first (scale_permute)."""
    if scale is not None or perm is not None:
        x = scale_permute(x, scale, perm)
    x = _c(x, np.float16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty((M,), dtype=np.float32)
    _check(lib().orc_rotate_quantize(_p(x.view(np.uint16)), M, K, b, bits, _p(q), _p(s)),
           "rotate_quantize")
    return q, s


def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """Unpacked codes -> the packed activation format (int4: [M, K/2] uint8)."""
    q = _c(q, np.int8)
    if bits == 8:
        return q.copy()
    M, K = q.shape
    p = np.empty((M, K // 2), dtype=np.uint8)
    lib().orc_pack_int4(_p(q), M, K, _p(p))
    return p


def unpack_codes(p: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Packed activation codes -> int8 [M, K]."""
    if bits == 8:
        return _c(p, np.int8).reshape(-1, K).copy()
    p = _c(p, np.uint8).reshape(-1, K // 2)
    M = p.shape[0]
    q = np.empty((M, K), dtype=np.int8)
    lib().orc_unpack_int4(_p(p), M, K, _p(q))
    return q


def unpack_idx(w_idx: np.ndarray, K: int) -> np.ndarray:
    """Packed weight indices [N, K/2] -> uint8 [N, K] in 0..15."""
    w = _c(w_idx, np.uint8).reshape(-1, K // 2)
    N = w.shape[0]
    idx = np.empty((N, K), dtype=np.uint8)
    lib().orc_unpack_idx(_p(w), N, K, _p(idx))
    return idx


# ---------------------------------------------------------------------------
# LUT product


def lut_gemm(q: np.ndarray, s: np.ndarray, w_idx: np.ndarray, codebook: np.ndarray,
             centroid_sums: bool = False):
    """y = s_x * sum_k C[n, I[n,k]] q[m,k].

    q: int8 [M, K] unpacked codes; s: fp32 [M]; w_idx: packed uint8 [N, K/2];
    codebook: fp16 [N, 16].  Returns (y fp64 [M, N], mag fp64 [M, N],
    S int32 [M, N, 16] or None); mag = |s| * sum_k |C q| is the scale of the
    tolerance.
    """
    q = _c(q, np.int8)
    s = _c(s, np.float32)
    M, K = q.shape
    idx = unpack_idx(w_idx, K)
    N = idx.shape[0]
    cb = _c(codebook, np.float16).reshape(N, 16)
    y = np.empty((M, N), dtype=np.float64)
    mag = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N, 16), dtype=np.int32) if centroid_sums else None
    _check(lib().orc_lut_gemm(_p(q), _p(s), M, K, _p(idx), _p(cb.view(np.uint16)), N,
                              _p(y), _p(mag), _p(S)), "lut_gemm")
    return y, mag, S


def unpack_idx_bits(w_idx: np.ndarray, K: int, idx_bits: int) -> np.ndarray:
    """b-bit packed indices uint8 [N, K*b/8] (least significant bit first)
    -> uint8 [N, K]."""
    w = _c(w_idx, np.uint8)
    N = w.shape[0]
    idx = np.empty((N, K), dtype=np.uint8)
    lib().orc_unpack_idx_bits(_p(w), N, K, int(idx_bits), _p(idx))
    return idx


def lut_gemm_bits(q: np.ndarray, s: np.ndarray, w_idx: np.ndarray, idx_bits: int,
                  codebook: np.ndarray):
    """The LUT product with 2^idx_bits centroids per row (adaptive codebook
    size): q int8 [M, K]; w_idx b-bit packed [N, K*b/8]; codebook fp16
    [N, 2^b].  Returns (y fp64 [M, N], mag fp64 [M, N])."""
    q = _c(q, np.int8)
    s = _c(s, np.float32)
    M, K = q.shape
    idx = unpack_idx_bits(w_idx, K, idx_bits)
    N = idx.shape[0]
    nc = 1 << idx_bits
    cb = _c(codebook, np.float16).reshape(N, nc)
    y = np.empty((M, N), dtype=np.float64)
    mag = np.empty((M, N), dtype=np.float64)
    _check(lib().orc_lut_gemm_nc(_p(q), _p(s), M, K, _p(idx), _p(cb.view(np.uint16)), nc, N,
                                 _p(y), _p(mag)), "lut_gemm_bits")
    return y, mag


def lut_tolerance(mag: np.ndarray) -> np.ndarray:
    """|y - y_ref| <= 1e-4 * s_x * sum_k |C q| + 1e-6 (the stated bound)."""
    return 1e-4 * mag + 1e-6


# ---------------------------------------------------------------------------
# routing and the expert FFN


def route(logits: np.ndarray, k: int, renormalize: bool = True):
    """-> dict(ids int32 [T,k], w fp64 [T,k], counts int32 [E], offsets int32
    [E+1], perm int32 [T*k])."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    counts = np.empty((E,), dtype=np.int32)
    offsets = np.empty((E + 1,), dtype=np.int32)
    perm = np.empty((T * k,), dtype=np.int32)
    _check(lib().orc_route(_p(lg), T, E, k, int(bool(renormalize)), _p(ids), _p(w),
                           _p(counts), _p(offsets), _p(perm)), "route")
    return dict(ids=ids, w=w, counts=counts, offsets=offsets, perm=perm)


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """fp16(silu(g) * u), evaluated in fp64."""
    g = _c(g, np.float64)
    u = _c(u, np.float64)
    h = np.empty(g.shape, dtype=np.uint16)
    lib().orc_swiglu(_p(g), _p(u), g.size, _p(h))
    return h.view(np.float16)


def combine(y_slot: np.ndarray, w: np.ndarray, y_shared: np.ndarray | None = None):
    """out[t] = sum_j w[t,j] y_slot[t*k+j] + sum_s y_shared[s, t]  (fp64)."""
    w = _c(w, np.float64)
    T, k = w.shape
    y_slot = _c(y_slot, np.float64).reshape(T * k, -1)
    H = y_slot.shape[1]
    ns = 0
    ysh = None
    if y_shared is not None:
        ysh = _c(y_shared, np.float64).reshape(-1, T, H)
        ns = ysh.shape[0]
    out = np.empty((T, H), dtype=np.float64)
    lib().orc_combine(_p(y_slot), _p(w), T, k, H, _p(ysh), ns, _p(out))
    return out


def expert_ffn(xq: np.ndarray, sx: np.ndarray, gate, up, down, had_block_i: int, bits: int):
    """One expert on the rows (xq, sx): gate/up LUT products, SwiGLU to fp16,
    rotate+quantize h, down LUT product.  gate/up/down are (w_idx, codebook).
    Returns dict(g, u, h, hq, sh, y)."""
    g, _, _ = lut_gemm(xq, sx, *gate)
    u, _, _ = lut_gemm(xq, sx, *up)
    h = swiglu(g, u)
    hq, sh = rotate_quantize(h, had_block_i, bits)
    y, _, _ = lut_gemm(hq, sh, *down)
    return dict(g=g, u=u, h=h, hq=hq, sh=sh, y=y)


def moe_ffn(inp, shape=None):
    """The whole layer on the CPU, no teacher forcing (fp64 except where the
    method quantizes).  ``inp`` is a synth.MoEInputs.  Returns dict with
    out fp64 [T, H] and the intermediate routing tables."""
    s = shape or inp.shape
    xq, sx = rotate_quantize(inp.x, s.had_block_h, s.act_bits,
                             scale=inp.extra.get("x_scale"), perm=inp.extra.get("x_perm"))
    T, H = s.T, s.H
    out = {}
    y_shared = None
    if s.n_shared:
        y_shared = np.zeros((s.n_shared, T, H))
        for j in range(s.n_shared):
            r = expert_ffn(xq, sx, (inp.sh_gate_idx[j], inp.sh_gate_cb[j]),
                           (inp.sh_up_idx[j], inp.sh_up_cb[j]),
                           (inp.sh_down_idx[j], inp.sh_down_cb[j]), s.had_block_i,
                           s.act_bits)
            y_shared[j] = r["y"]
    if s.E:
        rt = route(inp.logits, s.top_k, bool(s.renormalize))
        y_slot = np.zeros((T * s.top_k, H))
        for e in range(s.E):
            sl = rt["perm"][rt["offsets"][e]:rt["offsets"][e + 1]]
            if sl.size == 0:
                continue
            tok = sl // s.top_k
            r = expert_ffn(xq[tok], sx[tok], (inp.gate_idx[e], inp.gate_cb[e]),
                           (inp.up_idx[e], inp.up_cb[e]), (inp.down_idx[e], inp.down_cb[e]),
                           s.had_block_i, s.act_bits)
            y_slot[sl] = r["y"]
        out.update(rt)
        res = combine(y_slot, rt["w"], y_shared)
    else:
        res = y_shared.sum(axis=0)
    out.update(out=res, xq=xq, sx=sx)
    return out
