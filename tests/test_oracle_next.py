"""Pins for the oracle's monotonicity safeguard (review: "Assumptions & free
parameters", Assumption 1 of Theorem 1; referee comment 2): per block the
previous mask is kept exactly when it is a valid N:M block with a strictly
larger kept sum of |W|; otherwise the new mask stands."""
import numpy as np

import oracle
import synth


def test_safeguard_keeps_strictly_heavier_valid_blocks():
    _, W = synth.make_matrix(64, 256, "f32", "normal", 1.0, 3)
    new, _, _ = oracle.mask(W, 8, 16, 20.0, 100, 2)
    opt, best = oracle.opt(W, 8, 16, want_mask=True)
    out, kept = oracle.safeguard(W, best, new, 8, 16)
    obj_new = oracle.objective(W, new, 8, 16)
    assert kept == int((opt > obj_new).sum())
    np.testing.assert_array_equal(oracle.objective(W, out, 8, 16), np.maximum(opt, obj_new))
    # identical masks: nothing kept, output unchanged
    out2, kept2 = oracle.safeguard(W, new, new, 8, 16)
    assert kept2 == 0 and (out2 == new).all()


def test_safeguard_ignores_invalid_previous_blocks():
    _, W = synth.make_matrix(32, 64, "f32", "normal", 1.0, 4)
    new, _, _ = oracle.mask(W, 4, 8, 20.0, 50, 2)
    allones = np.full_like(new, 0xFFFFFFFF)           # heavier but not N:M
    out, kept = oracle.safeguard(W, allones, new, 4, 8)
    assert kept == 0 and (out == new).all()
