"""fp64 reference for the sparse-attention layers' decode step: a lightweight indexer scores
every past position of a sequence, the top-k positions are kept, and the core attention of
the query's heads runs over those positions only.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only tests/, the smoke entry
point and the benchmark's CPU-baseline leg may import it.

The pages (Zhidx article "280B Total Parameters, 14B Activated ...", section "1.
Latent-Gated Sparse Attention", DSA paragraph; wiki summary "Key claims": full-context MLA
layers use DeepSeek-style DSA, a lightweight indexer scores past positions and core attention
is only over the top-k; model-card page: MLA layers use 256-dim query, key and value) leave
the forms open.  This module's readings, the same in the kernels:
  - indexer: H_I indexer heads of dimension d_I per query, one indexer key of dimension d_I
    per position shared by the heads, and a weight per query and head:
        I(t, s) = sum_j w[t, j] * max(0, q_I[t, j] . k_I[s])
    (the ReLU-gated, head-weighted sum of the DeepSeek-style indexer);
  - selection: the k positions s <= t with the largest I(t, s); equal scores are taken in
    increasing position order; with at most k visible positions all are kept;
  - core attention: the query's Hq heads of dimension d attend, in one softmax per head, to
    the selected positions' keys and values (one key and one value row of dimension d per
    position, shared by all heads), logits scale * q . k.
Everything is fp64 on the given (bf16-valued) inputs.
"""
import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def index_scores(q_idx, w_idx, k_idx, seqlens):
    """Indexer scores of the decode query of each sequence (position L_b - 1) over positions
    0 .. L_b - 1.  q_idx [B, H_I, d_I], w_idx [B, H_I], k_idx [B, Lmax, d_I], seqlens [B].
    Returns [B, Lmax] with -inf past each sequence's length."""
    q, w, k = _f64(q_idx), _f64(w_idx), _f64(k_idx)
    B, Lmax = k.shape[0], k.shape[1]
    out = np.full((B, Lmax), -np.inf)
    for b in range(B):
        L = int(seqlens[b])
        dots = k[b, :L] @ q[b].T                      # [L, H_I]
        out[b, :L] = np.maximum(dots, 0.0) @ w[b]     # sum_j w_j relu(q_j . k_s)
    return out


def select_topk(scores, seqlens, k):
    """Positions of the k largest scores of each sequence among 0 .. L_b - 1, equal scores in
    increasing position order; returned in increasing position order, padded with -1 when a
    sequence has fewer than k positions.  [B, k] int32."""
    B = scores.shape[0]
    out = np.full((B, k), -1, dtype=np.int32)
    for b in range(B):
        L = int(seqlens[b])
        s = np.asarray(scores[b, :L], dtype=np.float64)
        # sort by (score descending, position ascending): lexsort's last key is primary
        order = np.lexsort((np.arange(L), -s))
        keep = np.sort(order[:min(k, L)])
        out[b, :len(keep)] = keep
    return out


def sparse_attend(q, kk, vv, idx, scale):
    """Core attention of each sequence's Hq query heads over its selected positions.
    q [B, Hq, d], kk / vv [B, Lmax, d], idx [B, k] (-1 = none).  Returns [B, Hq, d]."""
    q, kk, vv = _f64(q), _f64(kk), _f64(vv)
    B, Hq, d = q.shape
    out = np.zeros((B, Hq, vv.shape[2]))
    for b in range(B):
        sel = idx[b][idx[b] >= 0]
        logits = scale * (q[b] @ kk[b, sel].T)        # [Hq, n]
        logits -= logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p /= p.sum(axis=1, keepdims=True)
        out[b] = p @ vv[b, sel]
    return out


def decode(q_idx, w_idx, k_idx, q, kk, vv, seqlens, k, scale):
    """The whole step: scores, selection, attention.  Returns (out, idx, scores)."""
    sc = index_scores(q_idx, w_idx, k_idx, seqlens)
    idx = select_topk(sc, seqlens, k)
    return sparse_attend(q, kk, vv, idx, scale), idx, sc
