"""Packing-time helpers (offline, host side): the channel order that groups
activation outliers, and the weights repacked in that order.

CodeQuant podcast transcript, "Summary": the weights are reordered before
clustering so that extreme outliers are spread over different groups instead
of sharing one.  With a block Walsh-Hadamard rotation the group of a channel
is its rotation block: a block that holds two outlier channels spreads both
over its outputs and raises the token's absmax, coarsening every code of the
row.  The order below deals the channels, largest first, round-robin over the
blocks, so each block receives at most ceil(n / blocks) of the n largest.

The order is applied twice, consistently: the layer input is gathered online
(cq_rotate_quantize_ex / cq_moe_weights.x_perm) and the weights' K columns
are packed in the same order here, so the product is unchanged while the
rotation sees the grouped channels.
"""
from __future__ import annotations

import numpy as np


def outlier_grouping_perm(magnitude, had_block: int) -> np.ndarray:
    """int32 [K]: perm[j] = the channel placed at position j.

    magnitude: per-channel outlier measure [K] (e.g. max |x| over calibration
    tokens).  Channels are ranked by magnitude (descending, ties to the lower
    channel) and rank r goes to block r % B at position r // B, B = K / had_block.
    """
    mag = np.asarray(magnitude, dtype=np.float64).reshape(-1)
    K = mag.size
    if had_block <= 0 or K % had_block:
        raise ValueError("had_block must divide K")
    nb = K // had_block
    order = np.lexsort((np.arange(K), -mag))          # descending magnitude, stable
    r = np.arange(K)
    pos = (r % nb) * had_block + r // nb
    perm = np.empty(K, dtype=np.int32)
    perm[pos] = order
    return perm


def permute_weight_columns(w_idx: np.ndarray, perm) -> np.ndarray:
    """Packed 4-bit indices uint8 [..., K/2] with the K columns reordered:
    column j of the result is column perm[j] of the input (element 2j in the
    low nibble)."""
    w = np.asarray(w_idx, dtype=np.uint8)
    perm = np.asarray(perm).reshape(-1)
    full = np.empty(w.shape[:-1] + (2 * w.shape[-1],), dtype=np.uint8)
    full[..., 0::2] = w & 0xF
    full[..., 1::2] = w >> 4
    if perm.size != full.shape[-1] or not np.array_equal(np.sort(perm), np.arange(perm.size)):
        raise ValueError("perm must be a permutation of 0..K-1")
    full = full[..., perm]
    return (full[..., 0::2] | (full[..., 1::2] << 4)).astype(np.uint8)
