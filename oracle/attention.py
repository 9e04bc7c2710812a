"""Unbiased inner-product scores and one-pass decode attention over the
compressed cache.

Test infrastructure only (see oracle/__init__.py).

Score of query q against a compressed key (the audit's
``TurboQuantProd.attention_score``, "turboquant/audit_claims.py" AUDIT 3,
AUDIT 5, AUDIT 6; the query is rotated once and the estimate is corrected by
the 1-bit QJL term, "TurboQuant" explainer, troisinh.com, "Ý tưởng cốt lõi"
and "Giới hạn cần biết": the query rotation happens every step):

    q~ = Pi q,  s^ = S q
    score = nk16 * ( <q~, c[idx]> + kappa * rn16 * <s^, 2 sign - 1> ),
    kappa = sqrt(pi/2) / d.

By orthogonality <q~, c> = <q, Pi^T c> and <s^, sigma> = <q, S^T sigma>,
so the score equals <q, k_hat> for the explicit reconstruction.

Decode attention ("03. Results & Benchmarks", turboquant_cutile, "Latency
Benchmarks": score, QJL correction, online softmax and V accumulation in one
pass): for query head hq with KV head h = hq // G (consecutive grouping),
logits = score / sqrt(d) over the len_b cached tokens (no mask), softmax,
out = sum_n p_n v_hat_n with v_hat the group-dequantized values.  Reading: the
output is float32-sized; the oracle works in float64.
"""

from __future__ import annotations

import numpy as np

from .quant import dequantize_keys, dequantize_values, dequantize_values_mse, kappa


def rotate_query(q: np.ndarray, pi: np.ndarray, s: np.ndarray):
    """(Pi q, S q) for q [..., d]."""
    q = np.asarray(q, np.float64)
    return q @ np.asarray(pi, np.float64).T, q @ np.asarray(s, np.float64).T


def qjl_term(sh: np.ndarray, sign, rn, d: int):
    """QJL correction kappa * rn * <S q, 2 sign - 1> for sign bits [..., d]
    and residual norm(s) rn; an unbiased estimate of <q, r>."""
    sigma = 2.0 * np.asarray(sign, np.float64) - 1.0
    return kappa(d) * np.asarray(rn, np.float64) * (sigma @ np.asarray(sh, np.float64))


def score_keys(q: np.ndarray, idx, sign, nk16, rn16, pi, s, centroids) -> np.ndarray:
    """Scores of one query [d] against n compressed keys -> [n]."""
    q = np.asarray(q, np.float64)
    d = q.shape[-1]
    qt, sh = rotate_query(q, pi, s)
    c = np.asarray(centroids, np.float64)[idx]            # [n, d]
    mse = c @ qt
    return np.asarray(nk16, np.float64) * (mse + qjl_term(sh, sign, rn16, d))


def value_rows(rec: dict, h: int, pi, group: int, value_centroids=None) -> np.ndarray:
    """Explicitly dequantized values of KV head h: group-quantized records
    (codes, scale16, zero16) or TurboQuant-MSE records (vidx, nv16)."""
    if "vidx" in rec:
        return dequantize_values_mse(rec["vidx"][:, h], rec["nv16"][:, h], pi, value_centroids)
    return dequantize_values(rec["codes"][:, h], rec["scale16"][:, h], rec["zero16"][:, h], group)


def softmax_average(logits: np.ndarray, vhat: np.ndarray) -> np.ndarray:
    """sum_n softmax(logits)_n vhat_n, max-subtracted, float64."""
    m = np.max(logits)
    p = np.exp(logits - m)
    p = p / np.sum(p)
    return p @ vhat


def decode_one_sequence(q: np.ndarray, rec: dict, pi, s, centroids, group: int,
                        softmax_scale: float | None = None,
                        value_centroids=None) -> np.ndarray:
    """Decode attention for one sequence.

    q   [H_q, d] query
    rec logical cache fields of the sequence's cached tokens, each with a
        leading [N, H_kv] (idx, sign: [N, H_kv, d]; nk16, rn16: [N, H_kv];
        group-quantized values: codes [N, H_kv, d], scale16, zero16
        [N, H_kv, d/group]; TurboQuant-MSE values: vidx [N, H_kv, d], nv16
        [N, H_kv], with value_centroids the values' codebook)
    Returns out [H_q, d] float64.

    TurboQuant-MSE values are accumulated in the rotated space,
    acc = sum_n p_n nv16_n c[vidx_n], and rotated back once per head,
    out = Pi^T acc (the value half of the fused one-pass decode of
    "03. Results & Benchmarks", "Latency Benchmarks", with the value
    reconstruction of the key encoder's MSE stage).
    """
    q = np.asarray(q, np.float64)
    hq, d = q.shape
    n, hkv = rec["nk16"].shape
    if n == 0:
        raise ValueError("decode needs at least one cached token")
    g = hq // hkv
    scale = 1.0 / np.sqrt(d) if softmax_scale is None else softmax_scale
    mse_values = "vidx" in rec
    out = np.zeros((hq, d))
    for h in range(hkv):
        if mse_values:
            vrot = (np.asarray(rec["nv16"][:, h], np.float64)[:, None]
                    * np.asarray(value_centroids, np.float64)[rec["vidx"][:, h]])
        else:
            vhat = dequantize_values(rec["codes"][:, h], rec["scale16"][:, h],
                                     rec["zero16"][:, h], group)
        for j in range(g):
            qh = h * g + j
            sc = score_keys(q[qh], rec["idx"][:, h], rec["sign"][:, h],
                            rec["nk16"][:, h], rec["rn16"][:, h], pi, s, centroids)
            if mse_values:
                acc = softmax_average(sc * scale, vrot)          # rotated space
                out[qh] = acc @ np.asarray(pi, np.float64)       # Pi^T acc, as a row
            else:
                out[qh] = softmax_average(sc * scale, vhat)
    return out


def decode_with_window(q: np.ndarray, rec: dict | None, win_k: np.ndarray, win_v: np.ndarray,
                       pi, s, centroids, group: int,
                       softmax_scale: float | None = None,
                       value_centroids=None) -> np.ndarray:
    """Decode attention over the compressed tokens of one sequence plus a
    window of recent tokens kept exactly ("turboquant/audit_claims.py",
    AUDIT 1: the store keeps the most recent 128 tokens uncompressed in
    bf16 next to the compressed history).  One softmax over both sets:
    compressed tokens score with the estimator (score_keys) and carry the
    group-dequantized values; window tokens score q.k exactly and carry v.

    q      [H_q, d]
    rec    logical cache fields as in decode_one_sequence, or None / N = 0
    win_k, win_v  [W, H_kv, d] exact window keys and values (W may be 0)
    Returns out [H_q, d] float64 (zeros when there is no token at all).
    """
    q = np.asarray(q, np.float64)
    hq, d = q.shape
    win_k = np.asarray(win_k, np.float64)
    win_v = np.asarray(win_v, np.float64)
    w, hkv = win_k.shape[0], win_k.shape[1]
    n = 0 if rec is None else rec["nk16"].shape[0]
    g = hq // hkv
    scale = 1.0 / np.sqrt(d) if softmax_scale is None else softmax_scale
    out = np.zeros((hq, d))
    if n + w == 0:
        return out
    for h in range(hkv):
        vparts = []
        if n:
            vparts.append(value_rows(rec, h, pi, group, value_centroids))
        if w:
            vparts.append(win_v[:, h])
        values = np.concatenate(vparts, axis=0)
        for j in range(g):
            qh = h * g + j
            lparts = []
            if n:
                lparts.append(score_keys(q[qh], rec["idx"][:, h], rec["sign"][:, h],
                                         rec["nk16"][:, h], rec["rn16"][:, h], pi, s,
                                         centroids) * scale)
            if w:
                lparts.append((win_k[:, h] @ q[qh]) * scale)
            out[qh] = softmax_average(np.concatenate(lparts), values)
    return out


def prefill_one_sequence(q: np.ndarray, rec: dict, pi, s, centroids, group: int,
                         softmax_scale: float | None = None,
                         value_centroids=None) -> np.ndarray:
    """Causal attention of a chunk of T query tokens over the compressed cache
    of one sequence whose last T tokens are the chunk itself
    ("turboquant/audit_claims.py", AUDIT 7 and 8: long-context prefill as
    scaled-dot-product attention with a causal mask over the stored cache).
    Query token t (0-based) sees the first N - (T - 1 - t) cached tokens and
    is scored exactly as decode_one_sequence scores a decode query.

    q   [T, H_q, d]
    rec logical cache fields with a leading [N, H_kv] (N >= T)
    Returns out [T, H_q, d] float64; a token that sees no cached token gets
    zeros.
    """
    q = np.asarray(q, np.float64)
    t_chunk = q.shape[0]
    n = rec["nk16"].shape[0]
    out = np.zeros(q.shape)
    for t in range(t_chunk):
        m = n - (t_chunk - 1 - t)
        if m <= 0:
            continue
        sub = {k: v[:m] for k, v in rec.items()}
        out[t] = decode_one_sequence(q[t], sub, pi, s, centroids, group, softmax_scale,
                                     value_centroids)
    return out


def brute_force_one_sequence(q: np.ndarray, rec: dict, pi, s, centroids,
                             group: int, softmax_scale: float | None = None,
                             value_centroids=None) -> np.ndarray:
    """softmax(K_hat q / sqrt d) V_hat over explicitly dequantized K and V
    (the dequantize-then-matmul pattern of the audit's hybrid path, AUDIT 4)."""
    q = np.asarray(q, np.float64)
    hq, d = q.shape
    n, hkv = rec["nk16"].shape
    g = hq // hkv
    scale = 1.0 / np.sqrt(d) if softmax_scale is None else softmax_scale
    out = np.zeros((hq, d))
    for h in range(hkv):
        khat = dequantize_keys(rec["idx"][:, h], rec["sign"][:, h], rec["nk16"][:, h],
                               rec["rn16"][:, h], pi, s, centroids)
        vhat = value_rows(rec, h, pi, group, value_centroids)
        for j in range(g):
            qh = h * g + j
            logits = (khat @ q[qh]) * scale
            w = np.exp(logits - logits.max())
            out[qh] = (w / w.sum()) @ vhat
    return out


def stack_heads(recs: list) -> dict:
    """Combine per-head logical records (each [N, ...]) into [N, H_kv, ...]."""
    return {k: np.stack([r[k] for r in recs], axis=1) for k in recs[0]}
