"""Pins of the oracle's routing, W4A4+RAC product and MoE layer against
brute force, library routines and special-case reductions."""
import numpy as np
import pytest
import scipy.special

import oracle
import oracle.moe as omoe


def bf16(a):
    return oracle.f32_to_bf16(np.asarray(a, np.float32))


def test_route_matches_sort_and_softmax():
    rng = np.random.default_rng(0)
    T, E, kr = 200, 16, 4
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[5, [2, 9]] = 3.0                  # a tie: expert 2 must come first
    idx, gate = oracle.route(logits, kr)
    ref_idx = np.argsort(-logits, axis=1, kind="stable")[:, :kr]
    assert np.array_equal(idx, ref_idx)
    assert idx[5, 0] == 2 and idx[5, 1] == 9
    ref_g = scipy.special.softmax(np.take_along_axis(logits, ref_idx, 1).astype(np.float64), axis=1)
    np.testing.assert_allclose(gate, ref_g, rtol=1e-14)


def test_w4a4_rac_matmul_brute_force():
    rng = np.random.default_rng(1)
    M, N, K = 5, 7, 32
    xhat = rng.standard_normal((M, K)).astype(np.float32)
    what = rng.standard_normal((N, K)).astype(np.float32)
    S = np.array([1, 4, 30], np.int32)
    rho = bf16(rng.standard_normal((M, 3)).astype(np.float32) * 0.1)
    s_a = 0.37
    Y = oracle.w4a4_rac_matmul(xhat, s_a, rho, S, what)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(xhat[m, k]) * float(what[n, k])
            for j, c in enumerate(S):
                acc += s_a * float(oracle.bf16_to_f32(rho[m, j:j + 1])[0]) * float(what[n, c])
            assert abs(Y[m, n] - acc) <= 1e-12 * (1 + abs(acc))


def test_rac_special_cases():
    """k = 0 gives the plain W4A4 product; S = every channel recovers X W up to
    the bf16 rounding of the residual."""
    rng = np.random.default_rng(2)
    x = bf16(rng.standard_normal((16, 64)).astype(np.float32))
    w = rng.standard_normal((8, 64)).astype(np.float32) * 0.02
    qx = oracle.quantize(x)
    what = w
    y0 = oracle.w4a4_rac_matmul(qx.xhat, qx.s_t, None, None, what)
    np.testing.assert_allclose(y0, qx.xhat.astype(np.float64) @ what.astype(np.float64).T, rtol=1e-12, atol=1e-12)
    S = np.arange(64, dtype=np.int32)
    rho = oracle.rac_residual(qx.resid, qx.s_t, S)
    yall = oracle.w4a4_rac_matmul(qx.xhat, qx.s_t, rho, S, what)
    xw = oracle.bf16_to_f32(x).astype(np.float64) @ what.astype(np.float64).T
    err_full = np.linalg.norm(yall - xw) / np.linalg.norm(xw)
    err_none = np.linalg.norm(y0 - xw) / np.linalg.norm(xw)
    assert err_full < 2e-3 and err_none > 20 * err_full


def _tiny_layer(rng, T=24, H=64, I=32, E=4, kr=2):
    x = bf16(rng.standard_normal((T, H)).astype(np.float32))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w13 = bf16(rng.standard_normal((E, 2 * I, H)).astype(np.float32) * 0.05)
    w2 = bf16(rng.standard_normal((E, H, I)).astype(np.float32) * 0.05)
    return x, logits, omoe.quantize_weights(w13), omoe.quantize_weights(w2)


def test_moe_layer_per_token_definition():
    """Layer output equals a direct per-(token, slot) evaluation of the
    definition."""
    rng = np.random.default_rng(3)
    x, logits, w13q, w2q = _tiny_layer(rng)
    out = omoe.layer(x, logits, w13q, w2q, kr=2, k_x=8, k_h=4)
    T = x.shape[0]
    I = w13q[0].xhat.shape[0] // 2
    for t in range(T):
        yt = np.zeros(x.shape[1])
        for j in range(2):
            e = out["idx"][t, j]
            y13 = out["xq"].xhat[t].astype(np.float64) @ w13q[e].xhat.astype(np.float64).T
            r = oracle.bf16_to_f32(out["rho_x"][t]).astype(np.float64) * out["xq"].s_t
            y13 += r @ w13q[e].xhat[:, out["S_x"]].astype(np.float64).T
            h = y13[:I] / (1 + np.exp(-y13[:I])) * y13[I:]
            assert np.allclose(h, out["h64"][t * 2 + j], rtol=1e-12, atol=1e-14)
            row = t * 2 + j
            hq = out["hq"]
            y2 = hq.xhat[row].astype(np.float64) @ w2q[e].xhat.astype(np.float64).T
            r2 = oracle.bf16_to_f32(out["rho_h"][row]).astype(np.float64) * hq.s_t
            y2 += r2 @ w2q[e].xhat[:, out["S_h"]].astype(np.float64).T
            yt += out["gate"][t, j] * y2
        assert np.allclose(out["Y"][t], yt, rtol=1e-12, atol=1e-14)


def test_moe_single_expert_top1_is_dense():
    rng = np.random.default_rng(4)
    x, logits, w13q, w2q = _tiny_layer(rng, E=1, kr=1)
    out = omoe.layer(x, logits, w13q, w2q, kr=1, k_x=8, k_h=4)
    assert np.all(out["idx"] == 0) and np.allclose(out["gate"], 1.0)
    I = w13q[0].xhat.shape[0] // 2
    y13 = oracle.w4a4_rac_matmul(out["xq"].xhat, out["xq"].s_t, out["rho_x"], out["S_x"], w13q[0].xhat)
    np.testing.assert_allclose(out["h64"], oracle.swiglu(y13, I), rtol=1e-12)


def test_moe_token_permutation_permutes_rows():
    rng = np.random.default_rng(5)
    x, logits, w13q, w2q = _tiny_layer(rng)
    out = omoe.layer(x, logits, w13q, w2q, kr=2, k_x=8, k_h=4)
    perm = rng.permutation(x.shape[0])
    out_p = omoe.layer(x[perm], logits[perm], w13q, w2q, kr=2, k_x=8, k_h=4)
    np.testing.assert_allclose(out_p["Y"], out["Y"][perm], rtol=1e-9, atol=1e-12)


# ------------------------------------------------------------------ W4A16 layer
# Pins of oracle.moe.layer_w4a16 (gist.science/it 2.2 A: NVFP4 fake-quantized
# weights, BF16 activations) by invariances and by a special case in which the
# fake quantization is the identity.

def _w4a16_inputs(rng, T=6, H=32, I=16, E=3):
    x = bf16(rng.standard_normal((T, H)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w13 = bf16(rng.standard_normal((E, 2 * I, H)) * 0.1)
    w2 = bf16(rng.standard_normal((E, H, I)) * 0.1)
    return x, logits, w13, w2


def test_w4a16_expert_permutation_invariance():
    rng = np.random.default_rng(21)
    x, logits, w13, w2 = _w4a16_inputs(rng)
    perm = np.array([2, 0, 1])
    a = omoe.layer_w4a16(x, logits, w13, w2, 2)["Y"]
    b = omoe.layer_w4a16(x, logits[:, perm], w13[perm], w2[perm], 2)["Y"]
    np.testing.assert_allclose(a, b, rtol=0, atol=0)


def test_w4a16_token_permutation_equivariance():
    rng = np.random.default_rng(22)
    x, logits, w13, w2 = _w4a16_inputs(rng)
    perm = rng.permutation(x.shape[0])
    a = omoe.layer_w4a16(x, logits, w13, w2, 2)["Y"]
    b = omoe.layer_w4a16(x[perm], logits[perm], w13, w2, 2)["Y"]
    np.testing.assert_allclose(a[perm], b, rtol=0, atol=0)


def test_w4a16_down_weight_scaling_is_exact():
    # doubling W2 doubles its tensor scale and leaves its codes and block
    # scales unchanged, so the fake-quantized weight and Y double exactly
    rng = np.random.default_rng(23)
    x, logits, w13, w2 = _w4a16_inputs(rng)
    a = omoe.layer_w4a16(x, logits, w13, w2, 2)["Y"]
    w2x2 = bf16(oracle.bf16_to_f32(w2) * 2.0)
    b = omoe.layer_w4a16(x, logits, w13, w2x2, 2)["Y"]
    np.testing.assert_array_equal(b, 2.0 * a)


def test_w4a16_on_grid_weights_reduce_to_dense_ffn():
    # weights whose every 16-block holds +-6 and E2M1 values with the tensor
    # max 6 * 448 * 2^-12: every block scale is exactly 448 * 2^-12 / s_t
    # representable, so fake quantization returns the weights unchanged and
    # one expert with top-1 routing is the plain SwiGLU FFN
    rng = np.random.default_rng(24)
    T, H, I = 5, 32, 16
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)

    def on_grid(shape):
        v = rng.choice(grid, size=shape) * rng.choice([-1, 1], size=shape)
        v = v.reshape(-1, 16)
        v[:, 0] = 6.0                          # every block's max is 6
        return bf16((v.reshape(shape) * 448.0 * 2.0 ** -12).astype(np.float32))

    w13 = on_grid((1, 2 * I, H))
    w2 = on_grid((1, H, I))
    assert np.array_equal(oracle.qdq(w13[0])[0], w13[0]) and np.array_equal(oracle.qdq(w2[0])[0], w2[0])
    x = bf16(rng.standard_normal((T, H)))
    logits = np.zeros((T, 1), np.float32)
    out = omoe.layer_w4a16(x, logits, w13, w2, 1)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    g = np.einsum("th,nh->tn", xf, oracle.bf16_to_f32(w13[0]).astype(np.float64))
    h = g[:, :I] / (1.0 + np.exp(-g[:, :I])) * g[:, I:]
    hb = oracle.bf16_to_f32(bf16(h.astype(np.float32))).astype(np.float64)
    y = np.einsum("ti,hi->th", hb, oracle.bf16_to_f32(w2[0]).astype(np.float64))
    np.testing.assert_allclose(out["Y"], y, rtol=1e-12, atol=0)


def test_w4a16_router_weights_sum_over_identical_experts():
    # two identical experts, top-2: Y = (g0 + g1) y = y, the one-expert layer
    rng = np.random.default_rng(25)
    x, logits, w13, w2 = _w4a16_inputs(rng, E=1)
    one = omoe.layer_w4a16(x, np.zeros((x.shape[0], 1), np.float32), w13, w2, 1)["Y"]
    two = omoe.layer_w4a16(x, rng.standard_normal((x.shape[0], 2)).astype(np.float32),
                           np.concatenate([w13, w13]), np.concatenate([w2, w2]), 2)["Y"]
    np.testing.assert_allclose(two, one, rtol=1e-13, atol=1e-15)
