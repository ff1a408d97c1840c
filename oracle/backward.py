"""fp64 reference for the HCA backward pass (training): the gradients of the layer's output
with respect to the queries, the raw keys and values, and the pooling weights.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only tests/, the smoke entry
point and the benchmark's CPU-baseline leg may import it.

The forward it differentiates is the one the rest of the oracle computes, in fp64 and
without the bf16 rounding of the pooled cache.  Rounding has no gradient: in training the
stored cache is taken at its exact value.
  - Pooling (official blog "ERNIE 5.5 Flash Base . ERNIE", section 2.1: every 128 tokens
    become one cached entry; the softmax-weighted form is this library's reading of the
    compressor): alpha = softmax of the block's weights, Kc[j] = sum_i alpha_i K[blk*j + i],
    Vc likewise; one weight per position, shared by K, V and every KV head.
  - Attention of query t over the visible entries j < n_c(t) = max(0, floor((t-W+1)/blk))
    and the raw window [t-W+1, t], with one softmax over both segments; query head h reads
    KV head h*Hkv // Hq.
Everything here is written densely: a [T, Nc + T] visibility mask per sequence, the masked
softmax, and the textbook attention backward dS = P * (dP - rowsum(dO * O)).  All
arguments are float arrays (any float dtype, taken as fp64).
"""
import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def pool_f64(k, v, w, blk):
    """Softmax-weighted pooling of every complete block.

    k [B,T,Hkv,d], v [B,T,Hkv,dv], w [B,T] or None (zero weights: the mean).
    Returns kc [B,Nc,Hkv,d], vc [B,Nc,Hkv,dv] and alpha [B,Nc,blk], Nc = T // blk.
    """
    k, v = _f64(k), _f64(v)
    B, T = k.shape[:2]
    Nc = T // blk
    wb = np.zeros((B, Nc, blk)) if w is None else _f64(w)[:, :Nc * blk].reshape(B, Nc, blk)
    a = np.exp(wb - wb.max(axis=2, keepdims=True)) if Nc else np.zeros((B, 0, blk))
    a = a / a.sum(axis=2, keepdims=True) if Nc else a
    kb = k[:, :Nc * blk].reshape(B, Nc, blk, *k.shape[2:])
    vb = v[:, :Nc * blk].reshape(B, Nc, blk, *v.shape[2:])
    kc = np.einsum("bji,bjigc->bjgc", a, kb)
    vc = np.einsum("bji,bjigc->bjgc", a, vb)
    return kc, vc, a


def visibility(T, Nc, blk, W):
    """Keys visible to each query: mask [T, Nc + T], column j < Nc is entry j, column Nc + u
    is raw token u.  Entry j is visible iff j < n_c(t); raw u iff t - W + 1 <= u <= t."""
    t = np.arange(T)[:, None]
    n_c = np.maximum(0, (t - W + 1) // blk)
    ent = np.arange(Nc)[None, :] < n_c
    u = np.arange(T)[None, :]
    raw = (u <= t) & (u >= t - W + 1)
    return np.concatenate([ent, raw], axis=1)


def _keys(k, v, kc, vc, b, g):
    return np.concatenate([kc[b, :, g], k[b, :, g]]), np.concatenate([vc[b, :, g], v[b, :, g]])


def _probs(qh, keys, mask, scale):
    s = scale * (qh @ keys.T)
    s = np.where(mask, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=1, keepdims=True)


def attend_f64(q, k, v, kc, vc, blk, W, scale):
    """The attention output out [B,T,Hq,dv] for the given entries (taken as they are)."""
    q, k, v, kc, vc = map(_f64, (q, k, v, kc, vc))
    B, T, Hq, _ = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    mask = visibility(T, kc.shape[1], blk, W)
    out = np.zeros((B, T, Hq, dv))
    for b in range(B):
        for h in range(Hq):
            keys, vals = _keys(k, v, kc, vc, b, h * Hkv // Hq)
            out[b, :, h] = _probs(q[b, :, h], keys, mask, scale) @ vals
    return out


def attend_backward_f64(q, k, v, kc, vc, blk, W, scale, dout):
    """Gradients of sum(dout * out) for attend_f64, entries held fixed.

    Returns dq [B,T,Hq,d], dk [B,T,Hkv,d] and dv [B,T,Hkv,dv] through the raw window, and
    dkc [B,Nc,Hkv,d], dvc [B,Nc,Hkv,dv] for the entries.
    """
    q, k, v, kc, vc, dout = map(_f64, (q, k, v, kc, vc, dout))
    B, T, Hq, _ = q.shape
    Hkv = k.shape[2]
    Nc = kc.shape[1]
    mask = visibility(T, Nc, blk, W)
    dq = np.zeros_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    dkc, dvc = np.zeros_like(kc), np.zeros_like(vc)
    for b in range(B):
        for h in range(Hq):
            g = h * Hkv // Hq
            keys, vals = _keys(k, v, kc, vc, b, g)
            qh, do = q[b, :, h], dout[b, :, h]
            p = _probs(qh, keys, mask, scale)
            o = p @ vals
            dp = do @ vals.T
            ds = p * (dp - (do * o).sum(axis=1, keepdims=True))
            dq[b, :, h] = scale * (ds @ keys)
            dkeys = scale * (ds.T @ qh)
            dvals = p.T @ do
            dkc[b, :, g] += dkeys[:Nc]
            dk[b, :, g] += dkeys[Nc:]
            dvc[b, :, g] += dvals[:Nc]
            dv[b, :, g] += dvals[Nc:]
    return dq, dk, dv, dkc, dvc


def pool_backward_f64(k, v, w, blk, dkc, dvc):
    """Gradients of sum(dkc * kc + dvc * vc) for pool_f64: dk, dv (rows past the last
    complete block get zero) and dw [B,T].  The softmax over a block's weights gives
    dw_i = alpha_i (dalpha_i - sum_i' alpha_i' dalpha_i'), with
    dalpha_i = sum over KV heads of (K_i . dKc + V_i . dVc)."""
    k, v, dkc, dvc = map(_f64, (k, v, dkc, dvc))
    B, T = k.shape[:2]
    Nc = T // blk
    _, _, a = pool_f64(k, v, w, blk)
    kb = k[:, :Nc * blk].reshape(B, Nc, blk, *k.shape[2:])
    vb = v[:, :Nc * blk].reshape(B, Nc, blk, *v.shape[2:])
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    dk[:, :Nc * blk] = np.einsum("bji,bjgc->bjigc", a, dkc).reshape(B, Nc * blk, *k.shape[2:])
    dv[:, :Nc * blk] = np.einsum("bji,bjgc->bjigc", a, dvc).reshape(B, Nc * blk, *v.shape[2:])
    dal = np.einsum("bjigc,bjgc->bji", kb, dkc) + np.einsum("bjigc,bjgc->bji", vb, dvc)
    dwb = a * (dal - (a * dal).sum(axis=2, keepdims=True))
    dw = np.zeros((B, T))
    dw[:, :Nc * blk] = dwb.reshape(B, Nc * blk)
    return dk, dv, dw


def forward(q, k, v, w, blk, W, scale):
    """The layer's output [B,T,Hq,dv] in fp64: pooling, then attention."""
    kc, vc, _ = pool_f64(k, v, w, blk)
    return attend_f64(q, k, v, kc, vc, blk, W, scale)


def backward(q, k, v, w, blk, W, scale, dout):
    """The layer's gradients of sum(dout * out): dq, dk, dv (raw window path plus pooling
    path) and dw [B,T]."""
    kc, vc, _ = pool_f64(k, v, w, blk)
    dq, dk_raw, dv_raw, dkc, dvc = attend_backward_f64(q, k, v, kc, vc, blk, W, scale, dout)
    dk_pool, dv_pool, dw = pool_backward_f64(k, v, w, blk, dkc, dvc)
    return dq, dk_raw + dk_pool, dv_raw + dv_pool, dw


def _row_keys(t, T, Nc, blk, W):
    """Indices of the keys query t sees: entries j < n_c(t) and raw positions [t-W+1, t]."""
    n_c = max(0, (t - W + 1) // blk)
    return np.arange(min(n_c, Nc)), np.arange(max(0, t - W + 1), t + 1)


def backward_sampled(q, k, v, w, blk, W, scale, dout, b, rows=(), raw=(), entries=()):
    """Selected gradients of sequence b without the dense [T, Nc + T] matrices, for checks at
    lengths where the dense form does not fit.

    rows: query positions t -> dq[t] [Hq, d] (each needs only its own softmax row).
    raw: positions u -> the total dk[u], dv[u] [Hkv, d|dv] (window path from the W queries
    t in [u, u+W-1], plus the pooling path through u's block when it is complete) and dw[u].
    entries: blocks j -> dkc[j], dvc[j] (from the queries t >= blk(j+1) + W - 1).
    The cost is that of the queries involved: cheap for entries near the end of the
    sequence. Returns a dict of dicts keyed by position / block.
    """
    # q and dout are read row by row (widened to fp64 per row), so that full-size inputs need
    # no fp64 copy; sequence b's K and V are widened once
    T, Hq = q.shape[1], q.shape[2]
    Hkv = k.shape[2]
    k, v = _f64(k[b:b + 1]), _f64(v[b:b + 1])
    b_in, b = b, 0
    kc, vc, a = pool_f64(k, v, None if w is None else _f64(w)[b_in:b_in + 1], blk)
    kc, vc, a = kc[0], vc[0], a[0]
    Nc = kc.shape[0]
    blocks = sorted(set(entries) | {u // blk for u in raw if u // blk < Nc})
    # the queries whose softmax rows are needed
    need = set(rows)
    for u in raw:
        need.update(range(u, min(T, u + W)))
    for j in blocks:
        need.update(range(blk * (j + 1) + W - 1, T))
    dq = {t: np.zeros((Hq, q.shape[3])) for t in rows}
    dk_win = {u: np.zeros((Hkv, k.shape[3])) for u in raw}
    dv_win = {u: np.zeros((Hkv, v.shape[3])) for u in raw}
    dkc = {j: np.zeros((Hkv, kc.shape[2])) for j in blocks}
    dvc = {j: np.zeros((Hkv, vc.shape[2])) for j in blocks}
    for t in sorted(need):
        ej, ru = _row_keys(t, T, Nc, blk, W)
        for h in range(Hq):
            g = h * Hkv // Hq
            keys = np.concatenate([kc[ej, g], k[b, ru, g]])
            vals = np.concatenate([vc[ej, g], v[b, ru, g]])
            qh = _f64(q[b_in, t, h])
            s = scale * (keys @ qh)
            p = np.exp(s - s.max())
            p /= p.sum()
            do = _f64(dout[b_in, t, h])
            dp = vals @ do
            ds = p * (dp - do @ (p @ vals))
            if t in dq:
                dq[t][h] = scale * (ds @ keys)
            for i, j in enumerate(ej):
                if j in dkc:
                    dkc[j][g] += scale * ds[i] * qh
                    dvc[j][g] += p[i] * do
            for i, u in enumerate(ru):
                if u in dk_win:
                    dk_win[u][g] += scale * ds[len(ej) + i] * qh
                    dv_win[u][g] += p[len(ej) + i] * do
    # pooling path of the requested raw positions, and their weight gradients
    dk, dv, dw = {}, {}, {}
    for u in raw:
        j, i = divmod(u, blk)
        dk[u], dv[u], dw[u] = dk_win[u].copy(), dv_win[u].copy(), 0.0
        if j < Nc:
            dk[u] += a[j, i] * dkc[j]
            dv[u] += a[j, i] * dvc[j]
            kb, vb = k[b, blk * j:blk * (j + 1)], v[b, blk * j:blk * (j + 1)]
            dal = np.einsum("igc,gc->i", kb, dkc[j]) + np.einsum("igc,gc->i", vb, dvc[j])
            dw[u] = float(a[j, i] * (dal[i] - (a[j] * dal).sum()))
    return {"dq": dq, "dk": dk, "dv": dv, "dw": dw,
            "dkc": {j: dkc[j] for j in entries}, "dvc": {j: dvc[j] for j in entries}}
