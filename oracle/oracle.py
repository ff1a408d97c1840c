"""ctypes wrapper around the fp64 C oracle (test infrastructure only).

bf16 tensors travel as ``uint16`` numpy arrays holding the bf16 bit patterns;
fp32 tensors as ``float32``; results come back as ``float64``.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


def _bind(path):
    """Load an oracle shared object and declare its C signatures."""
    lib = ctypes.CDLL(path)
    _declare(lib)
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(_build.build())
    return _lib


def _declare(lib):
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_visible_entries.restype = _i64
    lib.oracle_visible_entries.argtypes = [_i64, _i64, _i64]
    lib.oracle_round_bf16.argtypes = [_f64p, _u16p, _i64]
    lib.oracle_compress.restype = ctypes.c_int
    lib.oracle_compress.argtypes = [_u16p, _u16p, _vp] + [_i64] * 6 + [_f64p, _f64p]
    lib.oracle_prefill_rows.restype = ctypes.c_int
    lib.oracle_prefill_rows.argtypes = ([_u16p] * 5 + [_i64] * 8 + [ctypes.c_double, _i64p, _i64,
                                        ctypes.c_int, _f64p, _vp])
    lib.oracle_decode.restype = ctypes.c_int
    lib.oracle_decode.argtypes = ([_u16p, _u16p, _u16p, _vp, _i64, _i64, _u16p, _u16p, _i32p,
                                   _vp, _vp, ctypes.c_double, _vp] + [_i64] * 8
                                  + [ctypes.c_double, _f64p, _vp])


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())


def bf16_bits(x):
    """bf16 bit patterns (uint16 numpy) of a torch bf16 tensor (any device)."""
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16))


def bits_to_f64(bits):
    """Exact fp64 values of bf16 bit patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def visible_entries(t: int, W: int, blk: int) -> int:
    """n_c(t) = max(0, floor((t - W + 1) / blk))."""
    return int(_load().oracle_visible_entries(int(t), int(W), int(blk)))


def round_bf16(x):
    """Round fp64 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_round_bf16(x.reshape(-1), y.reshape(-1), x.size)
    return y


def compress(k, v, w, blk):
    """Pool each complete block of blk raw rows into one entry.

    k: [B,T,Hkv,d] uint16 (bf16 bits), v: [B,T,Hkv,dv], w: [B,T] float32 or None.
    Returns (kc, vc) fp64 of shape [B, T//blk, Hkv, d|dv].
    """
    B, T, Hkv, d = k.shape
    dv = v.shape[3]
    assert v.shape[:3] == (B, T, Hkv)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    if w is not None:
        w = np.ascontiguousarray(w, dtype=np.float32)
        assert w.shape == (B, T)
    Nc = T // blk
    kc = np.zeros((B, Nc, Hkv, d), dtype=np.float64)
    vc = np.zeros((B, Nc, Hkv, dv), dtype=np.float64)
    rc = _load().oracle_compress(k, v, _ptr(w), B, T, Hkv, d, dv, blk, kc, vc)
    if rc:
        raise ValueError("oracle_compress rejected its arguments (%d)" % rc)
    return kc, vc


def prefill_rows(q, k, v, kc, vc, blk, W, scale, rows, want_lse=False, q_rows=False):
    """Attention output of prefill rows.

    q [B,T,Hq,d] (or [n_rows,Hq,d] with q_rows=True), k [B,T,Hkv,d], v [B,T,Hkv,dv],
    kc [B,Nc,Hkv,d], vc [B,Nc,Hkv,dv]: uint16 bf16 bits.
    rows: iterable of (b, t).  Returns out [n_rows, Hq, dv] fp64 (and lse [n_rows, Hq]).
    """
    B, T, Hkv, _ = k.shape
    Hq, d = q.shape[-2], q.shape[-1]
    dv = v.shape[3]
    Nc = T // blk
    assert kc.shape == (B, Nc, Hkv, d) and vc.shape == (B, Nc, Hkv, dv)
    rows = np.ascontiguousarray(np.asarray(list(rows), dtype=np.int64).reshape(-1, 2))
    n = rows.shape[0]
    out = np.zeros((n, Hq, dv), dtype=np.float64)
    lse = np.zeros((n, Hq), dtype=np.float64) if want_lse else None
    args = [np.ascontiguousarray(a, dtype=np.uint16) for a in (q, k, v, kc, vc)]
    if q_rows:
        assert q.shape[0] == n
    else:
        assert q.shape[:2] == (B, T)
    rc = _load().oracle_prefill_rows(*args, B, T, Hq, Hkv, d, dv, blk, W, float(scale), rows, n,
                                     1 if q_rows else 0, out, _ptr(lse))
    if rc:
        raise ValueError("oracle_prefill_rows rejected its arguments (%d)" % rc)
    return (out, lse) if want_lse else out


def decode(q, kc, vc, kw, vw, seqlens, blk, W, scale, page_table=None, page_size=0,
           gq=None, gk=None, eps=1e-6, gate=None, want_lse=False):
    """One decode query per sequence at position seqlens[b]-1.

    q [B,Hq,d]; kc/vc contiguous [B,Nmax,Hkv,d|dv] or a page pool [P,page,Hkv,d|dv] with
    page_table [B,max_pages] int32; kw/vw [B,W,Hkv,d|dv]; seqlens [B] int32;
    gq/gk [d] float32 or None; gate [B,Hq,dv] bf16 bits or None.
    Returns out [B,Hq,dv] fp64 (and lse [B,Hq]).
    """
    B, Hq, d = q.shape
    Hkv = kc.shape[2]
    dv = vc.shape[3]
    Nmax = kc.shape[1]
    assert kw.shape == (B, W, Hkv, d) and vw.shape == (B, W, Hkv, dv)
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    if page_table is not None:
        page_table = np.ascontiguousarray(page_table, dtype=np.int32)
        max_pages = page_table.shape[1]
        assert page_size == kc.shape[1]
    else:
        max_pages = 0
    if gq is not None:
        gq = np.ascontiguousarray(gq, dtype=np.float32)
        gk = np.ascontiguousarray(gk, dtype=np.float32)
    if gate is not None:
        gate = np.ascontiguousarray(gate, dtype=np.uint16)
    out = np.zeros((B, Hq, dv), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64) if want_lse else None
    a = [np.ascontiguousarray(x, dtype=np.uint16) for x in (q, kc, vc, kw, vw)]
    rc = _load().oracle_decode(a[0], a[1], a[2], _ptr(page_table), int(page_size), int(max_pages),
                               a[3], a[4], seqlens, _ptr(gq), _ptr(gk), float(eps), _ptr(gate),
                               B, Hq, Hkv, d, dv, blk, W, Nmax, float(scale), out, _ptr(lse))
    if rc:
        raise ValueError("oracle_decode rejected its arguments (%d)" % rc)
    return (out, lse) if want_lse else out


def vha(out, U, V):
    """Virtual Head Attention, the reading of the pages' "cross-head low-rank mixing with an
    identity skip" (official blog, section 2.1; Zhidx article, section "1. Latent-Gated
    Sparse Attention"): per token and per channel c, o'[:, c] = (I + U V^T) o[:, c] over the
    token's Hq heads, with U, V of shape [Hq, r].  Applied to the final attention output.

    out [n, Hq, dv] (any float), U, V [Hq, r] float32.  Returns fp64 [n, Hq, dv].
    Plain numpy in fp64: t = V^T o (r values per channel), then o + U t.
    """
    o = np.asarray(out, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    assert o.ndim == 3 and U.shape == V.shape and U.shape[0] == o.shape[1]
    t = np.einsum("hk,nhc->nkc", V, o)
    return o + np.einsum("hk,nkc->nhc", U, t)


def gate_logits(cq, Wg):
    """Low-Rank Gated Attention, the reading of the pages' gate (Zhidx article, section "1.
    Latent-Gated Sparse Attention"; official blog, section 2.1): the output gate's logits come
    from the attention layer's own query latent instead of the hidden state.  The latent is a
    quarter of the hidden size, so the gate projection has a quarter of the weights.

    cq [n, r_q] query latents, Wg [r_q, Hq, dv] gate projection.  Returns the logits
    g[n, h, c] = sum_k cq[n, k] Wg[k, h, c] in fp64; the attention output is then scaled by
    sigmoid(g), element-wise (the decode gate).  A plain contraction, written out with einsum.
    """
    cq = np.asarray(cq, dtype=np.float64)
    Wg = np.asarray(Wg, dtype=np.float64)
    assert cq.ndim == 2 and Wg.ndim == 3 and cq.shape[1] == Wg.shape[0]
    return np.einsum("nk,khc->nhc", cq, Wg)
