"""MoE expert-FFN layer of the QUADS rollout engine, per token -- TEST
INFRASTRUCTURE ONLY (see oracle/__init__.py).

The layer (QUADS pages: gist.science/it sections 1 and 4 -- a routed MoE whose
expert GEMMs run as native W4A4 NVFP4 products; section 2.2 B -- Residual
Activation Compensation on the activations entering each GEMM):

    idx, g   = top-k_r routing of the router logits, softmax over the k_r
    Xq       = NVFP4(X)                       (one s_t over all tokens)
    S_x      = top-k channels of X's residual score
    y13[t,j] = Xhat[t] W13q_e^T + s_x rho_x[t] W13q_e[:, S_x]^T,  e = idx[t,j]
    h[t,j]   = bf16(silu(y13[:, :I]) * y13[:, I:])
    Hq       = NVFP4(h over all routed rows)  (one s_t, one S_h)
    y2[t,j]  = Hhat[t,j] W2q_e^T + s_h rho_h[t,j] W2q_e[:, S_h]^T
    Y[t]     = sum_j g[t,j] y2[t,j]

Weights are quantized per expert tensor, each with its own s_t.  Routed rows
are kept in (token, slot) order, row t*k_r + j; the order is irrelevant to
every quantity above except the binary64 summation order of the h scores.
"""
from __future__ import annotations

import numpy as np

from . import (quantize, select_topk, channel_score, rac_residual, rac_residual_nvfp4, route,
               w4a4_rac_matmul, swiglu, f32_to_bf16, bf16_to_f32)


def _rac_operand(resid, s_t, S, rac_mode):
    """RAC residual operand: bf16 residual (default) or the NVFP4 second pass."""
    if rac_mode == "nvfp4":
        return rac_residual_nvfp4(resid, s_t, S)[0]
    return rac_residual(resid, s_t, S)


def quantize_weights(w: np.ndarray):
    """Per-expert NVFP4 weights: list of oracle.Quantized, one per expert,
    each with its own tensor scale."""
    return [quantize(w[e]) for e in range(w.shape[0])]


def expert_rac(resid, s_t, rows_by_expert, k):
    """Per-expert channel sets: for each expert e, S_e = the k channels of
    largest residual score over e's own rows (rows_by_expert[e], ascending),
    and rho_e = the bf16 residual of those rows on S_e.  READING: the pages
    select one binary channel mask per GEMM input (gist.science/it 2.2 B);
    choosing it per expert applies the same rule to the rows each expert's
    GEMM actually sees.  Returns dict e -> (S_e, rho_e)."""
    out = {}
    for e, rows in rows_by_expert.items():
        S = select_topk(channel_score(resid[rows]), k)
        out[e] = (S, rac_residual(resid[rows], s_t, S))
    return out


def _rows_by_expert(idx):
    """Routed rows (t*kr + j order) of every expert present, ascending."""
    experts = idx.reshape(-1)
    return {int(e): np.nonzero(experts == e)[0] for e in np.unique(experts)}


def gate_up(xq, rho_x, S_x, idx, w13q, inter, per_expert=None):
    """y13 for every routed row (t, j) and h = swiglu(y13); ``per_expert``
    (dict e -> (S_e, rho_e over e's tokens)) replaces the shared (rho_x, S_x).
    Returns (h_f64 [T*kr, I], h_bf16 [T*kr, I])."""
    T, kr = idx.shape
    h = np.zeros((T * kr, inter), np.float64)
    rows_t = np.repeat(np.arange(T), kr)
    experts = idx.reshape(-1)
    for e in np.unique(experts):
        rows = np.nonzero(experts == e)[0]
        toks = rows_t[rows]
        if per_expert is not None:
            S_e, rho_e = per_expert[int(e)]
            y = w4a4_rac_matmul(xq.xhat[toks], xq.s_t, rho_e, S_e, w13q[e].xhat)
        else:
            y = w4a4_rac_matmul(xq.xhat[toks], xq.s_t, None if rho_x is None else rho_x[toks],
                                S_x, w13q[e].xhat)
        h[rows] = swiglu(y, inter)
    return h, f32_to_bf16(h.astype(np.float32))


def down(h_bf16, idx, gate, w2q, k_h, row_valid=None, rac_mode="bf16", rac_scope="tensor"):
    """Quantize the routed h rows as one tensor, select S_h (one set, or one
    per expert with rac_scope "expert"), run the down GEMM with RAC and
    combine with the router weights.
    Returns dict(Y [T, H] f64, hq, S_h, rho_h, y2 [T*kr, H]); per expert,
    S_h and rho_h are dicts e -> S_e and e -> rho_e."""
    T, kr = idx.shape
    hq = quantize(h_bf16)
    H = w2q[0].xhat.shape[0]
    y2 = np.zeros((T * kr, H), np.float64)
    by_e = _rows_by_expert(idx)
    if rac_scope == "expert":
        assert rac_mode == "bf16" and row_valid is None
        per = expert_rac(hq.resid, hq.s_t, by_e, k_h)
        for e, rows in by_e.items():
            S_e, rho_e = per[e]
            y2[rows] = w4a4_rac_matmul(hq.xhat[rows], hq.s_t, rho_e, S_e, w2q[e].xhat)
        S_h = {e: v[0] for e, v in per.items()}
        rho_h = {e: v[1] for e, v in per.items()}
    else:
        S_h = select_topk(channel_score(hq.resid, row_valid), k_h)
        rho_h = _rac_operand(hq.resid, hq.s_t, S_h, rac_mode)
        for e, rows in by_e.items():
            y2[rows] = w4a4_rac_matmul(hq.xhat[rows], hq.s_t, rho_h[rows], S_h, w2q[e].xhat)
    Y = (y2.reshape(T, kr, H) * gate[:, :, None]).sum(axis=1)
    return dict(Y=Y, hq=hq, S_h=S_h, rho_h=rho_h, y2=y2)


def layer(x, logits, w13q, w2q, kr, k_x, k_h, rac_mode="bf16", rac_scope="tensor"):
    """Full layer from bf16 X and router logits; weights already quantized.
    rac_mode "nvfp4" takes the RAC operand from the second NVFP4 pass over
    the selected residual channels (oracle.rac_residual_nvfp4).  rac_scope
    "expert" selects the channel sets per expert, for X over the tokens routed
    to the expert and for h over its routed rows (expert_rac); the tensor
    scales stay per tensor."""
    idx, gate = route(logits, kr)
    xq = quantize(x)
    inter = w13q[0].xhat.shape[0] // 2
    if rac_scope == "expert":
        assert rac_mode == "bf16"
        T = x.shape[0]
        rows_t = np.repeat(np.arange(T), kr)
        toks_by_e = {e: rows_t[rows] for e, rows in _rows_by_expert(idx).items()}
        per = expert_rac(xq.resid, xq.s_t, toks_by_e, k_x)
        h64, hb = gate_up(xq, None, None, idx, w13q, inter, per_expert=per)
        S_x = {e: v[0] for e, v in per.items()}
        rho_x = {e: v[1] for e, v in per.items()}
    else:
        S_x = select_topk(channel_score(xq.resid), k_x)
        rho_x = _rac_operand(xq.resid, xq.s_t, S_x, rac_mode)
        h64, hb = gate_up(xq, rho_x, S_x, idx, w13q, inter)
    out = down(hb, idx, gate, w2q, k_h, rac_mode=rac_mode, rac_scope=rac_scope)
    out.update(idx=idx, gate=gate, xq=xq, S_x=S_x, rho_x=rho_x, h64=h64, h_bf16=hb)
    return out


def layer_w4a16(x, logits, w13, w2, kr, experts=None):
    """Trainer-side W4A16 layer (gist.science/it 2.2 A: NVFP4 fake-quantized
    weights, BF16 activations):

        Wq       = bf16(QDQ(W_e)) per expert tensor (oracle.qdq)
        y13[t,j] = X[t] Wq13_e^T              binary64 of the bf16 values
        h[t,j]   = bf16(silu(y13[:, :I]) * y13[:, I:])
        y2[t,j]  = h[t,j] Wq2_e^T
        Y[t]     = sum_j g[t,j] y2[t,j]

    ``experts``: optional dict e -> (Wq13_e, Wq2_e) bf16 bits, to reuse the
    weight fake-quantization between calls; missing experts are quantized
    here.  Returns dict(Y, h64, h_bf16, idx, gate)."""
    from . import qdq
    idx, gate = route(logits, kr)
    T = x.shape[0]
    inter = w13.shape[1] // 2
    H = w2.shape[1]
    cache = {} if experts is None else experts
    xf = bf16_to_f32(x).astype(np.float64)
    rows_t = np.repeat(np.arange(T), kr)
    flat = idx.reshape(-1)
    h = np.zeros((T * kr, inter), np.float64)
    for e in np.unique(flat):
        if e not in cache:
            cache[e] = (qdq(w13[e])[0], qdq(w2[e])[0])
        rows = np.nonzero(flat == e)[0]
        h[rows] = swiglu(xf[rows_t[rows]] @ bf16_to_f32(cache[e][0]).astype(np.float64).T, inter)
    hb = f32_to_bf16(h.astype(np.float32))
    hf = bf16_to_f32(hb).astype(np.float64)
    y2 = np.zeros((T * kr, H), np.float64)
    for e in np.unique(flat):
        rows = np.nonzero(flat == e)[0]
        y2[rows] = hf[rows] @ bf16_to_f32(cache[e][1]).astype(np.float64).T
    Y = (y2.reshape(T, kr, H) * gate[:, :, None]).sum(axis=1)
    return dict(Y=Y, h64=h, h_bf16=hb, idx=idx, gate=gate)


def tokens_sample(x, logits, tokens):
    """Restrict a layer's token inputs to a subset of tokens (used for the
    large workloads, where the oracle runs on a sample)."""
    return x[tokens], logits[tokens]


__all__ = ["quantize_weights", "gate_up", "down", "layer", "layer_w4a16", "tokens_sample", "bf16_to_f32"]
