"""Independent dense brute force for small HCA problems (test-only, numpy fp64).

It does not follow the oracle's loop structure: it builds the explicit key list
[compressed entries ; raw tokens] and a dense boolean visibility matrix from the
semantic description of the layer (official blog, section 2.1: each query sees the
compressed entries plus a short window of recent raw tokens), then runs one dense
masked softmax.

Visibility, stated without the closed-form entry count:
  * raw token u is visible to query t iff t - W + 1 <= u <= t (the window);
  * compressed entry j (raw positions blk*j .. blk*j+blk-1) is visible iff the whole
    block lies strictly before the window start, i.e. blk*j + blk - 1 < t - W + 1.
"""
import numpy as np
import torch


def bits_to_f64(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def pool_numpy(k, w, blk):
    """k [B,T,H,d] fp64, w [B,T] -> [B,T//blk,H,d] softmax-weighted block means (fp64)."""
    B, T, H, d = k.shape
    Nc = T // blk
    kb = k[:, :Nc * blk].reshape(B, Nc, blk, H, d)
    wb = w[:, :Nc * blk].reshape(B, Nc, blk).astype(np.float64)
    e = np.exp(wb - wb.max(axis=2, keepdims=True))
    a = e / e.sum(axis=2, keepdims=True)
    return np.einsum("bni,bnihd->bnhd", a, kb)


def to_bf16_f64(x):
    """Round fp64 -> bf16 through torch (fp64 -> fp32 -> bf16) and widen back."""
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def visibility(T, W, blk):
    """Dense mask [T, Nc + T] over the key list [entries ; raw tokens]."""
    Nc = T // blk
    t = np.arange(T)[:, None]
    j = np.arange(Nc)[None, :]
    u = np.arange(T)[None, :]
    ent = (blk * j + blk - 1) < (t - W + 1)
    raw = (u >= t - W + 1) & (u <= t)
    return np.concatenate([ent, raw], axis=1)


def attention_dense(q, keys, vals, mask, scale, Hkv):
    """q [T,Hq,d]; keys [N,Hkv,d]; vals [N,Hkv,dv]; mask [T,N] -> out [T,Hq,dv], lse [T,Hq]."""
    T, Hq, d = q.shape
    grp = Hq // Hkv
    out = np.zeros((T, Hq, vals.shape[2]))
    lse = np.zeros((T, Hq))
    for h in range(Hq):
        g = h // grp
        z = scale * q[:, h, :] @ keys[:, g, :].T
        z = np.where(mask, z, -np.inf)
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        s = p.sum(axis=1, keepdims=True)
        out[:, h, :] = (p @ vals[:, g, :]) / s
        lse[:, h] = (m + np.log(s))[:, 0]
    return out, lse


def hca_prefill_bruteforce(q, k, v, w, blk, W, scale):
    """All arrays fp64 numpy (exact bf16 values); B handled one by one."""
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    outs, lses = [], []
    kc = to_bf16_f64(pool_numpy(k, w, blk))
    vc = to_bf16_f64(pool_numpy(v, w, blk))
    mask = visibility(T, W, blk)
    for b in range(B):
        keys = np.concatenate([kc[b], k[b]], axis=0)
        vals = np.concatenate([vc[b], v[b]], axis=0)
        o, l = attention_dense(q[b], keys, vals, mask, scale, Hkv)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)
