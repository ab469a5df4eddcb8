"""Seeded synthetic inputs for the CodeQuant LUT MoE linear layer.

This module only draws random numbers and packs them into the input formats
of the layer (fp16 activations with fixed outlier channels, fp32 router
logits, and per-row 16-centroid codebooks with packed 4-bit indices).  It
holds none of the layer's arithmetic: no rotation, no activation
quantization, no lookup-table product, no routing.  Both the CPU oracle and
the CUDA path receive exactly the arrays produced here.

Weight codebooks come from an offline per-row 1-D k-means (Lloyd) fit, the
clustering step that CodeQuant uses to build its centroid matrix and per-row
assignment matrices (CodeQuant2 page, Figure 3).  It only shapes the inputs;
parity never depends on it.

Every tensor draws from its own stream: ``SeedSequence(seed, spawn_key=
(crc32(name),))``, so adding a tensor never changes the others.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np
import torch

# ---------------------------------------------------------------------------
# random streams


def rng(seed: int, name: str) -> np.random.Generator:
    """Independent generator for the tensor called ``name``."""
    ss = np.random.SeedSequence(seed, spawn_key=(zlib.crc32(name.encode()),))
    return np.random.Generator(np.random.PCG64(ss))


# ---------------------------------------------------------------------------
# activations and router logits


def activations(M: int, K: int, *, seed: int, name: str, n_outliers: int = 4,
                outlier_scale: float = 50.0) -> np.ndarray:
    """fp16 [M, K] ~ N(0, 1) with ``n_outliers`` fixed channels scaled up.

    The outlier channels are distinct, drawn once per tensor and shared by all
    tokens (massive-activation channels, as in the workloads the pages study).
    """
    g = rng(seed, name)
    x = g.standard_normal((M, K), dtype=np.float32)
    if n_outliers:
        ch = g.choice(K, size=min(n_outliers, K), replace=False)
        x[:, ch] *= np.float32(outlier_scale)
    return x.astype(np.float16)


def router_logits(T: int, E: int, *, seed: int, name: str,
                  bias_expert: int | None = None, bias: float = 1.0) -> np.ndarray:
    """fp32 [T, E] ~ N(0, 1); optionally ``bias`` added to one expert's column."""
    g = rng(seed, name)
    lg = g.standard_normal((T, E), dtype=np.float32)
    if bias_expert is not None:
        lg[:, bias_expert] += np.float32(bias)
    return lg


# ---------------------------------------------------------------------------
# weights: Gaussian + heavy-tailed outliers, per-row 16-centroid k-means


def raw_weights(N: int, K: int, *, seed: int, name: str, std: float = 0.02,
                outlier_frac: float = 0.01, outlier_scale: float = 0.1,
                outlier_df: float = 3.0) -> np.ndarray:
    """fp32 [N, K]: N(0, std^2); a Bernoulli(outlier_frac) subset of entries is
    replaced by Student-t(outlier_df) * outlier_scale."""
    g = rng(seed, name)
    w = g.standard_normal(N * K, dtype=np.float32)
    w *= np.float32(std)
    if outlier_frac > 0:
        # a Bernoulli process over the flat index: geometric gaps between hits
        n_exp = int(N * K * outlier_frac * 1.2) + 64
        pos = np.cumsum(g.geometric(outlier_frac, size=n_exp)) - 1
        while pos[-1] < N * K:  # practically never: extend
            more = np.cumsum(g.geometric(outlier_frac, size=n_exp)) + pos[-1]
            pos = np.concatenate([pos, more])
        pos = pos[pos < N * K]
        w[pos] = (g.standard_t(outlier_df, size=pos.size) * outlier_scale).astype(np.float32)
    return w.reshape(N, K)


def kmeans_codebook(w: np.ndarray, *, n_centroids: int = 16, iters: int = 10,
                    row_chunk: int = 2048) -> tuple[np.ndarray, np.ndarray]:
    """Per-row 1-D Lloyd k-means.

    Returns ``(idx uint8 [N, K] in 0..15, codebook fp16 [N, 16])``.
    Initialisation: the row's order statistics at quantiles (c + 0.5) / 16.
    A cluster that becomes empty keeps its previous centroid.  After the last
    iteration the centroids are rounded to fp16 and every weight is assigned
    to the nearest fp16 centroid (ties go to the lower index).
    """
    N, K = w.shape
    idx_out = np.empty((N, K), dtype=np.uint8)
    cb_out = np.empty((N, n_centroids), dtype=np.float16)
    pos0 = torch.clamp(((torch.arange(n_centroids, dtype=torch.float64) + 0.5)
                        / n_centroids * K).long(), max=K - 1)
    for r0 in range(0, N, row_chunk):
        x = torch.from_numpy(np.ascontiguousarray(w[r0:r0 + row_chunk])).double()
        xs, _ = torch.sort(x, dim=1)
        cs = torch.nn.functional.pad(torch.cumsum(xs, dim=1), (1, 0))
        c = xs[:, pos0].clone()
        n = x.shape[0]
        zero = torch.zeros((n, 1), dtype=torch.long)
        full = torch.full((n, 1), K, dtype=torch.long)
        for _ in range(iters):
            mid = 0.5 * (c[:, :-1] + c[:, 1:])
            # elements <= mid belong to the lower cluster
            b = torch.searchsorted(xs, mid.contiguous(), right=True)
            bnd = torch.cat([zero, b, full], dim=1)
            cnt = (bnd[:, 1:] - bnd[:, :-1])
            sm = cs.gather(1, bnd[:, 1:]) - cs.gather(1, bnd[:, :-1])
            c = torch.where(cnt > 0, sm / cnt.clamp(min=1), c)
        c16 = c.to(torch.float16)
        cd = c16.double()
        mid = 0.5 * (cd[:, :-1] + cd[:, 1:])
        # number of midpoints strictly below x: a tie goes to the lower index
        idx = torch.searchsorted(mid.contiguous(), x, right=False)
        idx_out[r0:r0 + n] = idx.to(torch.uint8).numpy()
        cb_out[r0:r0 + n] = c16.numpy()
    return idx_out, cb_out


def pack_nibbles(v: np.ndarray) -> np.ndarray:
    """uint8 [..., K] values in 0..15 -> uint8 [..., K/2]; element 2j in the low
    nibble, 2j+1 in the high nibble."""
    v = np.asarray(v, dtype=np.uint8)
    return (v[..., 0::2] & 0xF) | ((v[..., 1::2] & 0xF) << 4)


def pack_bits(v: np.ndarray, bits: int) -> np.ndarray:
    """uint8 [..., K] values below 2^bits -> uint8 [..., K*bits/8]: element k
    in bits [bits*k, bits*k + bits), least significant bit first (bits = 4 is
    pack_nibbles)."""
    v = np.asarray(v, dtype=np.uint8)
    planes = ((v[..., :, None] >> np.arange(bits, dtype=np.uint8)) & 1).astype(np.uint8)
    flat = planes.reshape(v.shape[:-1] + (v.shape[-1] * bits,))
    return np.packbits(flat, axis=-1, bitorder="little")


def lut_weights(N: int, K: int, *, seed: int, name: str,
                idx_bits: int = 4) -> tuple[np.ndarray, np.ndarray]:
    """(w_idx packed uint8 [N, K*b/8], codebook fp16 [N, 2^b]) for one linear
    with 2^idx_bits centroids per row (16 by default)."""
    idx, cb = kmeans_codebook(raw_weights(N, K, seed=seed, name=name),
                              n_centroids=1 << idx_bits)
    return (pack_nibbles(idx) if idx_bits == 4 else pack_bits(idx, idx_bits)), cb


# ---------------------------------------------------------------------------
# the five workloads


def largest_pow2_divisor(K: int, cap: int = 8192) -> int:
    b = 1
    while K % (b * 2) == 0 and b * 2 <= cap:
        b *= 2
    return b


@dataclass
class MoEShape:
    """Shape of one MoE (or dense SwiGLU) layer."""
    name: str
    H: int
    I: int
    E: int
    top_k: int
    n_shared: int
    T: int
    act_bits: int
    had_block_h: int
    had_block_i: int
    renormalize: int = 1
    I_shared: int = 0
    n_outliers: int = 4
    outlier_scale: float = 50.0
    bias_expert: int | None = None
    bias: float = 0.0

    def __post_init__(self):
        if self.I_shared == 0:
            self.I_shared = self.I

    @property
    def had_block_i_shared(self) -> int:
        return self.had_block_i


@dataclass
class LinearShape:
    name: str
    M: int
    K: int
    N: int
    had_block: int
    act_bits: int
    n_outliers: int = 4
    outlier_scale: float = 50.0


# configuration 0: one linear layer
CFG0 = LinearShape("linear_m1_k2048_n2048_a4w4", M=1, K=2048, N=2048, had_block=2048, act_bits=4)


def cfg1(M: int, act_bits: int) -> MoEShape:
    """Qwen3-4B-shaped dense SwiGLU FFN (hidden 2560, intermediate 9728)."""
    return MoEShape(f"qwen3_4b_ffn_m{M}_a{act_bits}w4", H=2560, I=9728, E=0, top_k=0,
                    n_shared=1, T=M, act_bits=act_bits, had_block_h=512, had_block_i=256)


CFG1_VARIANTS = [(M, b) for b in (4, 8) for M in (1, 4, 16)]

CFG2 = MoEShape("qwen3_30b_a3b_moe_t64", H=2048, I=768, E=128, top_k=8, n_shared=0, T=64,
                act_bits=4, had_block_h=2048, had_block_i=256)

CFG3 = MoEShape("mixtral_8x7b_moe_t256", H=4096, I=14336, E=8, top_k=2, n_shared=0, T=256,
                act_bits=8, had_block_h=4096, had_block_i=2048, bias_expert=0, bias=1.0)

CFG4 = MoEShape("prefill_moe_e64_s2_t4096", H=2048, I=1408, E=64, top_k=6, n_shared=2, T=4096,
                act_bits=4, had_block_h=2048, had_block_i=128, n_outliers=8,
                outlier_scale=100.0)


@dataclass
class MoEInputs:
    shape: MoEShape
    x: np.ndarray                       # fp16 [T, H]
    logits: np.ndarray | None           # fp32 [T, E]
    gate_idx: np.ndarray | None = None  # uint8 [E, I, H/2]
    up_idx: np.ndarray | None = None
    down_idx: np.ndarray | None = None  # uint8 [E, H, I/2]
    gate_cb: np.ndarray | None = None   # fp16 [E, I, 16]
    up_cb: np.ndarray | None = None
    down_cb: np.ndarray | None = None   # fp16 [E, H, 16]
    sh_gate_idx: np.ndarray | None = None
    sh_up_idx: np.ndarray | None = None
    sh_down_idx: np.ndarray | None = None
    sh_gate_cb: np.ndarray | None = None
    sh_up_cb: np.ndarray | None = None
    sh_down_cb: np.ndarray | None = None
    extra: dict = field(default_factory=dict)


def _expert_stack(n: int, N: int, K: int, seed: int, prefix: str):
    """Weights of n experts.  Every expert draws from its own named stream, so
    generating them on a thread pool (numpy's bulk draws and torch's CPU ops
    release the interpreter lock) gives exactly the serial result."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    idx = np.empty((n, N, K // 2), dtype=np.uint8)
    cb = np.empty((n, N, 16), dtype=np.float16)

    def one(e):
        idx[e], cb[e] = lut_weights(N, K, seed=seed, name=f"{prefix}.{e}")

    workers = max(1, min(n, (os.cpu_count() or 1), 16))
    if workers == 1:
        for e in range(n):
            one(e)
    else:
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(one, range(n)))
    return idx, cb


def moe_inputs(s: MoEShape, seed: int = 0, *, weights: bool = True) -> MoEInputs:
    """All inputs of one MoE / dense-FFN layer."""
    x = activations(s.T, s.H, seed=seed, name=f"{s.name}.x", n_outliers=s.n_outliers,
                    outlier_scale=s.outlier_scale)
    lg = None
    if s.E > 0:
        lg = router_logits(s.T, s.E, seed=seed, name=f"{s.name}.logits",
                           bias_expert=s.bias_expert, bias=s.bias)
    out = MoEInputs(s, x, lg)
    if not weights:
        return out
    if s.E > 0:
        out.gate_idx, out.gate_cb = _expert_stack(s.E, s.I, s.H, seed, f"{s.name}.gate")
        out.up_idx, out.up_cb = _expert_stack(s.E, s.I, s.H, seed, f"{s.name}.up")
        out.down_idx, out.down_cb = _expert_stack(s.E, s.H, s.I, seed, f"{s.name}.down")
    if s.n_shared > 0:
        out.sh_gate_idx, out.sh_gate_cb = _expert_stack(s.n_shared, s.I_shared, s.H, seed,
                                                        f"{s.name}.shared_gate")
        out.sh_up_idx, out.sh_up_cb = _expert_stack(s.n_shared, s.I_shared, s.H, seed,
                                                    f"{s.name}.shared_up")
        out.sh_down_idx, out.sh_down_cb = _expert_stack(s.n_shared, s.H, s.I_shared, seed,
                                                        f"{s.name}.shared_down")
    return out


def linear_inputs(s: LinearShape, seed: int = 0):
    """(x fp16 [M, K], w_idx uint8 [N, K/2], codebook fp16 [N, 16])."""
    x = activations(s.M, s.K, seed=seed, name=f"{s.name}.x", n_outliers=s.n_outliers,
                    outlier_scale=s.outlier_scale)
    w_idx, cb = lut_weights(s.N, s.K, seed=seed, name=f"{s.name}.w")
    return x, w_idx, cb
