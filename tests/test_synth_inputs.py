"""The seeded synthetic inputs follow their stated recipe (they stand in for the
pages' models): determinism, outlier channels, heavy-tailed weights, per-row
k-means codebooks with nearest-centroid assignment, biased routing."""
import numpy as np

import synth


def test_named_streams_are_deterministic_and_independent():
    a = synth.activations(4, 64, seed=0, name="x")
    assert np.array_equal(a, synth.activations(4, 64, seed=0, name="x"))
    assert not np.array_equal(a, synth.activations(4, 64, seed=0, name="y"))
    assert not np.array_equal(a, synth.activations(4, 64, seed=1, name="x"))
    assert a.dtype == np.float16 and a.shape == (4, 64)


def test_outlier_channels_are_fixed_across_tokens():
    x = synth.activations(256, 512, seed=0, name="outl", n_outliers=4, outlier_scale=50.0)
    rms = np.sqrt((x.astype(np.float64) ** 2).mean(axis=0))
    hot = np.argsort(-rms)[:4]
    assert np.all(rms[hot] > 20) and np.sort(rms)[-5] < 2.0   # exactly 4 channels x50
    assert np.all(np.abs(x[:, hot]).mean(axis=0) > 20)         # hot in every token block


def test_weights_gaussian_with_one_percent_student_t():
    w = synth.raw_weights(256, 1024, seed=0, name="w")
    assert w.dtype == np.float32
    core = w[np.abs(w) < 0.1]
    assert abs(core.std() - 0.02) < 0.002
    frac_big = np.mean(np.abs(w) > 0.1)     # N(0, 0.02) essentially never exceeds 5 sigma
    assert 0.002 < frac_big < 0.01          # a share of the 1 % t(3) x 0.1 entries


def test_kmeans_codebook_nearest_fp16_centroid():
    w = synth.raw_weights(8, 512, seed=0, name="km")
    idx, cb = synth.kmeans_codebook(w)
    assert idx.shape == (8, 512) and cb.shape == (8, 16) and cb.dtype == np.float16
    assert idx.max() <= 15
    c = cb.astype(np.float64)
    assert np.all(np.diff(c, axis=1) >= 0)                     # 1-D k-means: sorted
    d = np.abs(w[:, :, None].astype(np.float64) - c[:, None, :])
    best = d.min(axis=2)
    got = np.take_along_axis(d, idx[:, :, None].astype(np.int64), axis=2)[:, :, 0]
    assert np.array_equal(got, best)                           # nearest centroid
    # ties go to the lower index
    first = np.argmax(d == best[:, :, None], axis=2)
    assert np.array_equal(idx, first.astype(np.uint8))
    # packing: element 2j low nibble
    p = synth.pack_nibbles(idx)
    assert np.array_equal(p & 15, idx[:, 0::2]) and np.array_equal(p >> 4, idx[:, 1::2])


def test_router_bias_and_workload_shapes():
    lg = synth.router_logits(4096, 8, seed=0, name="r", bias_expert=0, bias=1.0)
    assert abs(lg[:, 0].mean() - 1.0) < 0.1 and abs(lg[:, 1:].mean()) < 0.05
    s = synth.CFG3
    assert (s.H, s.I, s.E, s.top_k, s.T, s.act_bits) == (4096, 14336, 8, 2, 256, 8)
    assert s.bias_expert == 0 and s.had_block_i == 2048
    s = synth.CFG4
    assert (s.H, s.I, s.E, s.top_k, s.n_shared, s.T) == (2048, 1408, 64, 6, 2, 4096)
    assert s.had_block_i == synth.largest_pow2_divisor(1408) == 128
    s = synth.cfg1(16, 8)
    assert (s.H, s.I, s.had_block_h, s.had_block_i) == (2560, 9728, 512, 256)
