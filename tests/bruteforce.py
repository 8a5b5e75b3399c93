"""Independent numpy float64 formulations used to pin the oracle.

Nothing here shares code with the oracle: the block decoders are vectorised
table lookups written from the format definitions, and the layer is computed
with a dense [M, E] gate matrix over ALL experts (``y = sum_e G[:, e] * FFN_e(X)``),
a formulation the oracle does not use.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit, softmax

E2M1_TABLE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_q8_0(blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    b = np.ascontiguousarray(blob, np.uint8).reshape(rows, cols // 32, 34)
    d = b[:, :, 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    q = b[:, :, 2:].view(np.int8).astype(np.float64)
    return (d[..., None] * q).reshape(rows, cols)


def decode_mxfp4(blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    b = np.ascontiguousarray(blob, np.uint8).reshape(rows, cols // 32, 17)
    scale = np.ldexp(1.0, b[:, :, 0].astype(np.int64) - 127)
    qs = b[:, :, 1:]
    codes = np.stack([qs & 15, qs >> 4], axis=-1).reshape(rows, cols // 32, 32)
    return (scale[..., None] * E2M1_TABLE[codes]).reshape(rows, cols)


def decode_int4_affine(blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    b = np.ascontiguousarray(blob, np.uint8).reshape(rows, cols // 32, 20)
    d = b[:, :, 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    m = b[:, :, 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
    qs = b[:, :, 4:]
    q = np.stack([qs & 15, qs >> 4], axis=-1).reshape(rows, cols // 32, 32).astype(np.float64)
    return (d[..., None] * q + m[..., None]).reshape(rows, cols)


def decode(fmt: int, blob, rows, cols):
    return (decode_q8_0, decode_mxfp4, decode_int4_affine)[fmt](blob, rows, cols)


def act_np(kind: int, g, u, alpha=1.702, limit=7.0):
    if kind == 0:
        return g * expit(g) * u
    gc = np.minimum(g, limit)
    uc = np.clip(u, -limit, limit)
    return gc * expit(alpha * gc) * (uc + 1.0)


def topk_bruteforce(lsel_row: np.ndarray, K: int) -> np.ndarray:
    E = lsel_row.shape[0]
    order = np.lexsort((np.arange(E), -lsel_row.astype(np.float64)))
    return order[:K]


def layer_bruteforce(shape, L: dict, x_bits: np.ndarray, resid_bits=None):
    """Returns (logits32, idx, w, y, out) computed with dense matrices."""
    H, I, E, K, S = shape.hidden, shape.moe_inter, shape.num_experts, shape.top_k, shape.shared_inter
    X = bf16_bits_to_f64(x_bits)
    M = X.shape[0]
    s = bf16_bits_to_f64(L["xscale"]) if L.get("xscale") is not None else np.ones(H)
    Wr = decode_q8_0(L["router"], E, H)
    logits = ((X * s) @ Wr.T).astype(np.float32)
    bias = L.get("bias")
    # sigmoid scoring selects on sigmoid(l) (+ the correction bias) instead of l
    base = expit(logits.astype(np.float64)) if shape.score == 2 else logits.astype(np.float64)
    if bias is not None and shape.bias_mode != 0:
        lsel = (base + np.asarray(bias, np.float64)).astype(np.float32)
    else:
        lsel = base.astype(np.float32)
    score = lsel.astype(np.float64) if (shape.bias_mode == 1 and bias is not None) else logits.astype(np.float64)
    idx = np.stack([topk_bruteforce(lsel[m], K) for m in range(M)]).astype(np.int32)
    G = np.zeros((M, E))
    w = np.zeros((M, K))
    for m in range(M):
        if shape.score == 0:
            pw = softmax(score[m, idx[m]])
        elif shape.score == 1:
            pw = softmax(score[m])[idx[m]]
        else:
            sel = base[m, idx[m]]
            pw = sel / sel.sum()
        pes = L.get("pes")
        if pes is not None:
            pw = pw * np.asarray(pes, np.float64)[idx[m]]
        w[m] = pw
        G[m, idx[m]] = pw
    fmt = shape.expert_fmt
    gate = np.asarray(L["gate"]).reshape(E, -1)
    up = np.asarray(L["up"]).reshape(E, -1)
    down = np.asarray(L["down"]).reshape(E, -1)
    Y = np.zeros((M, H))
    for e in range(E):
        Wg = decode(fmt, gate[e], I, H)
        Wu = decode(fmt, up[e], I, H)
        Wd = decode(fmt, down[e], H, I)
        A = act_np(shape.act, X @ Wg.T, X @ Wu.T, shape.act_alpha, shape.act_limit)
        Y += G[:, e:e + 1] * (A @ Wd.T)
    if S:
        Sg = decode_q8_0(L["sh_gate"], S, H)
        Su = decode_q8_0(L["sh_up"], S, H)
        Sd = decode_q8_0(L["sh_down"], H, S)
        Y += act_np(shape.act, X @ Sg.T, X @ Su.T, shape.act_alpha, shape.act_limit) @ Sd.T
    R = bf16_bits_to_f64(resid_bits) if resid_bits is not None else np.zeros_like(Y)
    return logits, idx, w, Y, R + Y
