"""The shared seeded input generator: determinism, slice independence and distributions."""
import numpy as np

import synth


def test_counter_based_slices_match_full_tensors():
    full = synth.w4a16_weights(0, 256, 128, range(8))
    sub = synth.w4a16_weights(0, 256, 128, [5, 2])
    for key in full:
        assert np.array_equal(sub[key][0], full[key][5])
        assert np.array_equal(sub[key][1], full[key][2])
    x = synth.x_bf16(1, 16, 256)
    assert np.array_equal(synth.x_bf16(1, 4, 256, t0=7), x[7:11])
    lg = synth.logits(2, 12, 64, zipf_s=1.1)
    assert np.array_equal(synth.logits(2, 3, 64, zipf_s=1.1, t0=4), lg[4:7])
    q, s = synth.x_e4m3(3, 6, 256)
    q2, s2 = synth.x_e4m3(3, 2, 256, t0=3)
    assert np.array_equal(q2, q[3:5]) and np.array_equal(s2, s[3:5])


def test_seeds_and_tensors_are_distinct_streams():
    a = synth.x_bf16(0, 4, 256)
    assert not np.array_equal(a, synth.x_bf16(1, 4, 256))
    w = synth.w4a16_weights(0, 256, 256, [0])
    assert not np.array_equal(w["w13_q"][0, :, :8], w["w2_q"][0, :, :8])


def test_distributions():
    w = synth.w4a16_weights(0, 1024, 512, [0])
    nib = np.stack([(w["w13_q"].view(np.uint32) >> (4 * j)) & 0xF for j in range(8)]).ravel()
    hist = np.bincount(nib, minlength=16) / nib.size
    assert np.all(np.abs(hist - 1 / 16) < 0.005)
    sc = (w["w13_s"].astype(np.uint32) << 16).view(np.float32)
    assert sc.min() >= 0.005 * (1 - 2 ** -8) and sc.max() <= 0.02 * (1 + 2 ** -8)
    lg = synth.logits(0, 256, 384)
    assert abs(lg.mean()) < 0.01 and abs(lg.std() - 1) < 0.01
    b = synth.zipf_bias(0, 384, 1.1)
    assert sorted(np.round(np.exp(-b / 1.1)).astype(int).tolist()) == list(range(1, 385))
    q, s = synth.x_e4m3(0, 4, 512)
    assert np.all(s > 0) and q.max() <= 0xFE
