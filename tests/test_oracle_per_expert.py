"""Pins of the per-expert RAC channel sets in the oracle layer
(oracle.moe.layer / down with rac_scope="expert"): S_e is the top-k channel
set by residual score over the rows expert e's GEMM sees (the pages' binary
channel mask, gist.science/it 2.2 B, applied per expert GEMM)."""
import numpy as np

import oracle
from oracle import moe as om


def _bits(a):
    return oracle.f32_to_bf16(np.asarray(a, np.float32))


def _weights(rng, E, H, I):
    w13 = [oracle.quantize(_bits(rng.standard_normal((2 * I, H)) * 0.02)) for _ in range(E)]
    w2 = [oracle.quantize(_bits(rng.standard_normal((H, I)) * 0.02)) for _ in range(E)]
    return w13, w2


def test_routing_to_every_expert_gives_the_shared_x_set():
    # with k_r = E every expert sees every token, so each X set is the tensor's
    rng = np.random.default_rng(0)
    T, H, I, E, k = 40, 128, 64, 3, 9
    x = rng.standard_normal((T, H)).astype(np.float32)
    x[:, [5, 77]] *= 15
    x = _bits(x)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w13, w2 = _weights(rng, E, H, I)
    per = om.layer(x, logits, w13, w2, E, k, 8, rac_scope="expert")
    glob = om.layer(x, logits, w13, w2, E, k, 8)
    for e in range(E):
        assert np.array_equal(per["S_x"][e], glob["S_x"])
        assert np.array_equal(per["rho_x"][e], glob["rho_x"])


def test_one_expert_equals_the_tensor_scope():
    rng = np.random.default_rng(1)
    T, H, I, k = 48, 128, 64, 12
    x = _bits(rng.standard_normal((T, H)) * np.where(rng.random(H) < 0.05, 20.0, 1.0))
    logits = np.zeros((T, 1), np.float32)
    w13, w2 = _weights(rng, 1, H, I)
    per = om.layer(x, logits, w13, w2, 1, k, 10, rac_scope="expert")
    glob = om.layer(x, logits, w13, w2, 1, k, 10)
    assert np.array_equal(per["S_x"][0], glob["S_x"]) and np.array_equal(per["S_h"][0], glob["S_h"])
    assert np.array_equal(per["Y"], glob["Y"])


def test_sets_follow_each_experts_own_rows():
    # tokens 0..19 go to expert 0, 20..39 to expert 1 (top-1); channel 3 is an
    # outlier only in expert 0's tokens, channel 60 only in expert 1's
    rng = np.random.default_rng(2)
    T, H, I = 40, 64, 64
    xf = rng.standard_normal((T, H)).astype(np.float32) * 0.1
    xf[:20, 3] = rng.uniform(3.0, 9.0, 20) * np.sign(rng.standard_normal(20))
    xf[20:, 60] = rng.uniform(3.0, 9.0, 20) * np.sign(rng.standard_normal(20))
    x = _bits(xf)
    logits = np.zeros((T, 2), np.float32)
    logits[:20, 0] = 1.0
    logits[20:, 1] = 1.0
    w13, w2 = _weights(rng, 2, H, I)
    out = om.layer(x, logits, w13, w2, 1, 1, 4, rac_scope="expert")
    assert list(out["S_x"][0]) == [3] and list(out["S_x"][1]) == [60]
    # the expert's set depends only on its own tokens: change expert 1's
    # tokens (keeping the tensor maximum) and expert 0's set and rho stay
    xf2 = xf.copy()
    xf2[20:, 11] = 8.0 * np.sign(rng.standard_normal(20))
    out2 = om.layer(_bits(xf2), logits, w13, w2, 1, 1, 4, rac_scope="expert")
    assert oracle.quantize(_bits(xf2)).s_t == oracle.quantize(x).s_t
    assert np.array_equal(out2["S_x"][0], out["S_x"][0]) and np.array_equal(out2["rho_x"][0], out["rho_x"][0])
    assert list(out2["S_x"][1]) != list(out["S_x"][1])


def test_down_sets_match_scores_over_each_experts_rows():
    # S_h[e] against a full stable sort of the binary64 score over e's rows
    rng = np.random.default_rng(3)
    T, kr, E, I, H, k = 30, 2, 4, 128, 64, 7
    hb = _bits(rng.standard_normal((T * kr, I)) * np.where(rng.random(I) < 0.1, 8.0, 1.0))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    idx, gate = oracle.route(logits, kr)
    w2 = [oracle.quantize(_bits(rng.standard_normal((H, I)) * 0.02)) for _ in range(E)]
    out = om.down(hb, idx, gate, w2, k, rac_scope="expert")
    R = out["hq"].resid.astype(np.float64)
    flat = idx.reshape(-1)
    for e in np.unique(flat):
        rows = np.nonzero(flat == e)[0]
        score = (R[rows] ** 2).sum(axis=0)
        order = sorted(range(I), key=lambda c: (-score[c], c))[:k]
        assert list(out["S_h"][int(e)]) == sorted(order)
