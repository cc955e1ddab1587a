"""Estimators on the codes: attention logits, MSE dequantisation, decode
attention and top-k search (TEST INFRASTRUCTURE).

* Inner-product estimate ("TurboQuant explainer" (m.163.com), "第二步：QJL"
  and its identity E[<y, Q^-1(Q(x))>] = <y, x>).  For a query q and a key
  stored as (n, idx, gamma, s):

      q_rot = H D q / sqrt(d_pad)            (the rotated query)
      u     = S q_rot                        (the projected query)
      l     = n * ( sum_j q_rot_j c[idx_j]
                    + gamma * sqrt(pi/2) / m * sum_i u_i (2 s_i - 1) )

  The first term is <q, k_mse> because the rotation is orthogonal; the second
  is the QJL correction.  Logits are raw inner products (no 1/sqrt(d) scale).
  GQA: query head h reads KV head h // group.
* MSE-only values ("TurboQuant explainer", "速度" - logits from compressed KV;
  zhidx turboquant_plus article - asymmetric K/V):
      v_hat = n * D o (H c[idx]) / sqrt(d_pad), first d coordinates.
* Product-code reconstruction (the map Q^-1 of "第二步：QJL"):
      x_hat = n * D o (H (c[idx] + sqrt(pi/2)/m * gamma * S^T (2s-1))) / sqrt(d_pad).
* Decode attention: o = sum_j softmax_j(scale * l_j) v_hat_j with the
  maximum subtracted; scale defaults to 1/sqrt(d).  Plain token-by-token
  fp64; the GPU's chunked online softmax is a reassociation of this sum.
* Sparse V (zhidx turboquant_plus article, "Sparse V": skip the value work of
  tokens whose attention weight is negligible): a token with softmax weight
  p_j < v_eps contributes no value; it stays in the normalisation, so
  |o - o_full| <= v_eps * sum over skipped tokens of |v_hat_j|.
* Search ("TurboQuant explainer", "向量搜索"): the k database ids with the
  largest estimate, ties to the lower id.
* Sharded forms (a database or a sequence split across devices): the global
  top-k is the top-k of the union of per-shard top-k lists (ids offset to
  global), and decode attention over a token split is the log-sum-exp merge
  of per-shard partials (m = max score, l = sum exp(score - m),
  o = sum exp(score - m) v_hat).

All arithmetic in fp64; the stored fp16 norms are used as stored.
"""
import numpy as np

from .codec import rotate, unrotate, pad


def prep_queries(q, D, S):
    """Rotated queries q_rot [n_q, d_pad] and projections u [n_q, m] (fp64)."""
    d_pad = D.shape[0]
    q_rot = rotate(pad(np.asarray(q, dtype=np.float64), d_pad), D)
    u = q_rot @ np.asarray(S, dtype=np.float64).T if S is not None else None
    return q_rot, u


def logits_from_codes(q_rot, u, idx, signs, norm_f16, rnorm_f16, centroids, m):
    """Estimates for every (query, key) pair: [n_q, n_keys] fp64.

    q_rot [n_q, d_pad], u [n_q, m] (None for MSE-only codes), idx [n_keys, d_pad],
    signs [n_keys, m] 0/1 (None for MSE-only), norms fp16 [n_keys].
    """
    c = np.asarray(centroids, dtype=np.float64)
    k_mse = c[idx]                                           # [n_keys, d_pad]
    base = q_rot @ k_mse.T
    if signs is not None:
        pm = 2.0 * signs.astype(np.float64) - 1.0            # [n_keys, m]
        corr = (u @ pm.T) * (np.sqrt(np.pi / 2.0) / m) * rnorm_f16.astype(np.float64)[None, :]
        base = base + corr
    return base * norm_f16.astype(np.float64)[None, :]


def logits_gqa(q, D, S, idx, signs, norm_f16, rnorm_f16, centroids, m, n_kv_heads, group, n_keys):
    """tq_logits semantics: q [n_kv_heads*group, d]; keys of head g are rows
    g*n_keys .. (g+1)*n_keys-1 of idx/signs/norms.  Returns [n_q, n_keys]."""
    q_rot, u = prep_queries(q, D, S)
    out = np.zeros((q.shape[0], n_keys), dtype=np.float64)
    for h in range(q.shape[0]):
        g = h // group
        sl = slice(g * n_keys, (g + 1) * n_keys)
        out[h] = logits_from_codes(q_rot[h:h + 1], None if u is None else u[h:h + 1],
                                   idx[sl], None if signs is None else signs[sl],
                                   norm_f16[sl], None if rnorm_f16 is None else rnorm_f16[sl],
                                   centroids, m)[0]
    return out


def dequant_mse(idx, norm_f16, centroids, D, d):
    """v_hat rows [n, d] (fp64) from MSE-only codes."""
    y = np.asarray(centroids, dtype=np.float64)[idx]
    return unrotate(y, D)[:, :d] * norm_f16.astype(np.float64)[:, None]


def dequant_prod(idx, signs, norm_f16, rnorm_f16, centroids, D, S, m, d):
    """x_hat rows [n, d] (fp64) from product codes: the inverse map Q^-1 of
    "TurboQuant explainer" (m.163.com), "第二步：QJL" (the QJL part is
    r_hat = sqrt(pi/2)/m * gamma * S^T sigma with sigma = 2s - 1, so that
    E[<y, Q^-1(Q(x))>] = <y, x>), added to the Lloyd-Max centroids in the
    rotated domain and rotated back:
        x_hat = n * D H (c[idx] + r_hat) / sqrt(d_pad), first d coordinates.
    <q, x_hat> is exactly the logit estimate of `logits_from_codes` (linearity)."""
    y = np.asarray(centroids, dtype=np.float64)[idx]
    sigma = 2.0 * np.asarray(signs, dtype=np.float64) - 1.0                # [n, m]
    r_hat = (np.sqrt(np.pi / 2.0) / m) * rnorm_f16.astype(np.float64)[:, None] * (sigma @ np.asarray(S, dtype=np.float64))
    return unrotate(y + r_hat, D)[:, :d] * norm_f16.astype(np.float64)[:, None]


def softmax_weights(logit_row, scale):
    """p = softmax(scale * logit_row), maximum subtracted."""
    s = scale * np.asarray(logit_row, dtype=np.float64)
    s = s - np.max(s)
    p = np.exp(s)
    return p / np.sum(p)


def softmax_attend(logit_row, values, scale, v_eps=0.0):
    """o = sum_j p_j values_j with p = softmax(scale * logit_row); with v_eps > 0
    the tokens with p_j < v_eps add nothing (Sparse V), their weight stays in
    the normalisation."""
    p = softmax_weights(logit_row, scale)
    if v_eps > 0.0:
        p = np.where(p < v_eps, 0.0, p)
    return p @ values


def decode_attention(q, kD, kS, k_idx, k_signs, k_norm, k_rnorm, k_cent, km,
                     vD, v_idx, v_norm, v_cent, d, seq_lens, Hq, Hkv, max_tokens,
                     scale=0.0, pairs=None, v_eps=0.0, bound=None):
    """tq_decode_attn semantics (v_eps > 0: Sparse V, as softmax_attend).

    q [B, Hq, d]; key/value vector index = (b*Hkv + g)*max_tokens + t.
    Returns out [B, Hq, d] (fp64); rows not in `pairs` (list of (b, h)) are NaN
    when `pairs` is given.  If `bound` is an array [B, Hq] it receives
    v_eps * sum_{p_j < v_eps} |v_hat_j|, the largest change Sparse V can make.
    """
    B = q.shape[0]
    group = Hq // Hkv
    if scale == 0.0:
        scale = 1.0 / np.sqrt(d)
    out = np.full((B, Hq, d), np.nan)
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hq)]
    cache = {}
    for (b, h) in todo:
        g = h // group
        L = int(seq_lens[b])
        if L == 0:
            out[b, h] = 0.0
            continue
        base = (b * Hkv + g) * max_tokens
        sl = slice(base, base + L)
        q_rot, u = prep_queries(q[b, h][None, :], kD, kS)
        lg = logits_from_codes(q_rot, u, k_idx[sl], k_signs[sl], k_norm[sl], k_rnorm[sl], k_cent, km)[0]
        key = (b, g)
        if key not in cache:
            cache[key] = dequant_mse(v_idx[sl], v_norm[sl], v_cent, vD, d)
        out[b, h] = softmax_attend(lg, cache[key], scale, v_eps)
        if bound is not None:
            p = softmax_weights(lg, scale)
            bound[b, h] = v_eps * np.sum(np.linalg.norm(cache[key][p < v_eps], axis=1))
    return out


def topk(scores, k):
    """Top-k column ids per row by descending score, ties to the lower id."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[1]
    ids = np.broadcast_to(np.arange(n), scores.shape)
    order = np.lexsort((ids, -scores), axis=1)   # primary: -score, secondary: id
    top = order[:, :k]
    return top.astype(np.int64), np.take_along_axis(scores, top, axis=1)


def recall_at_k(found, truth):
    """Mean over rows of |found_row ∩ truth_row| / k."""
    k = truth.shape[1]
    return float(np.mean([len(set(f) & set(t)) / k for f, t in zip(found, truth)]))


def decode_partial(q, kD, kS, k_idx, k_signs, k_norm, k_rnorm, k_cent, km,
                   vD, v_idx, v_norm, v_cent, d, seq_lens, Hq, Hkv, max_tokens, scale=0.0):
    """Unnormalised decode attention over the tokens given (one shard of every sequence),
    same arguments and indexing as decode_attention.  Per (b, h): m = max_t scale*l_t,
    l = sum_t exp(scale*l_t - m), o = sum_t exp(scale*l_t - m) v_hat_t.  A row without
    tokens has m = -inf, l = 0, o = 0.  Returns (m [B, Hq], l [B, Hq], o [B, Hq, d])."""
    B = q.shape[0]
    group = Hq // Hkv
    if scale == 0.0:
        scale = 1.0 / np.sqrt(d)
    m = np.full((B, Hq), -np.inf)
    lsum = np.zeros((B, Hq))
    o = np.zeros((B, Hq, d))
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        for h in range(Hq):
            g = h // group
            base = (b * Hkv + g) * max_tokens
            sl = slice(base, base + L)
            q_rot, u = prep_queries(q[b, h][None, :], kD, kS)
            s = scale * logits_from_codes(q_rot, u, k_idx[sl], k_signs[sl], k_norm[sl], k_rnorm[sl], k_cent, km)[0]
            m[b, h] = np.max(s)
            w = np.exp(s - m[b, h])
            lsum[b, h] = np.sum(w)
            o[b, h] = w @ dequant_mse(v_idx[sl], v_norm[sl], v_cent, vD, d)
    return m, lsum, o


def merge_partials(parts):
    """Log-sum-exp merge of decode partials [(m, l, o), ...]: with M = max_k m_k and
    w_k = exp(m_k - M) (0 for an empty part), out = sum_k w_k o_k / sum_k w_k l_k;
    rows that are empty in every part are 0."""
    M = np.max(np.stack([p[0] for p in parts]), axis=0)
    num = np.zeros_like(parts[0][2])
    den = np.zeros_like(parts[0][1])
    for m, lsum, o in parts:
        w = np.where(np.isfinite(m), np.exp(np.where(np.isfinite(m), m - np.where(np.isfinite(M), M, 0.0), 0.0)),
                     0.0)
        num += w[..., None] * o
        den += w * lsum
    safe = np.where(den > 0, den, 1.0)
    return np.where(den[..., None] > 0, num / safe[..., None], 0.0)


def merge_topk(ids_parts, score_parts, offsets, k):
    """Global top-k from per-shard top-k lists: ids_parts[p] [n_q, k_p] shard-local ids
    (an id < 0 marks an empty slot), score_parts[p] their estimates, offsets[p] the first
    global id of shard p.  Ties go to the lower global id.  Returns (ids, scores) [n_q, k]."""
    ids = np.concatenate([np.where(np.asarray(i) >= 0, np.asarray(i, dtype=np.int64) + int(o), -1)
                          for i, o in zip(ids_parts, offsets)], axis=1)
    sc = np.concatenate([np.asarray(s, dtype=np.float64) for s in score_parts], axis=1)
    sc = np.where(ids >= 0, sc, -np.inf)
    big = np.where(ids >= 0, ids, np.iinfo(np.int64).max)
    order = np.lexsort((big, -sc), axis=1)[:, :k]
    out_i = np.take_along_axis(ids, order, axis=1)
    out_s = np.take_along_axis(sc, order, axis=1)
    return out_i, out_s
