"""compressed_long_context_b200 -- Heavily Compressed Attention (HCA) on B200.

A thin PyTorch-facing binding over the C ABI of ``libhca.so`` (include/hca.h).
Every step of the computation runs in the library's CUDA kernels; this module only
checks dtypes/devices, allocates outputs with PyTorch and passes raw device pointers
and the current CUDA stream.  If the library is missing, calls fail loudly.

The layer (web pages on ERNIE 5.5 Flash Base: official blog, section 2.1; Zhidx
article, section "1. Latent-Gated Sparse Attention"): every 128 tokens of K/V are
pooled into one cached entry, and each query attends, in one causal softmax, to all
completed entries plus a window of the W most recent raw tokens.
"""
import torch

from . import _lib
from ._lib import (HCA_OUT_F32, HCA_OUT_GATE, HCA_PAGED, HCA_QK_NORM,  # noqa: F401
                   HCA_WINDOW_RING, HCA_WRITE_LSE)

__all__ = ["HCAError", "compress", "prefill", "decode", "decode_workspace_size", "append", "append_state_size",
           "vha", "gate_logits", "prefill_backward", "dsa_index", "dsa_topk", "dsa_attend", "dsa_decode",
           "get_device_error", "status_string"]


class HCAError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__("%s: %s" % (where, status_string(code)))


def status_string(code: int) -> str:
    return _lib.load().hca_status_string(int(code)).decode()


def _check(code, where):
    if code != _lib.HCA_OK:
        raise HCAError(code, where)


def _p(t):
    return None if t is None else t.data_ptr()


def _stream(device):
    return torch.cuda.current_stream(device).cuda_stream


def _need(t, dtype, name, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _room(t, n, name):
    """The kernels address a buffer from the sizes they are given: refuse one that holds fewer
    elements than that footprint (it would be read or written out of bounds)."""
    if t is not None and t.numel() < n:
        raise ValueError("%s holds %d elements, the call addresses %d" % (name, t.numel(), n))


def get_device_error(device=None) -> None:
    """Synchronise the current stream and raise if a kernel recorded a device-side error."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    _check(_lib.load().hca_get_device_error(_stream(device)), "device")


def compress(k, v, w=None, blk=128, kc=None, vc=None):
    """Pool every complete block of ``blk`` raw rows into one cache entry.

    k [B,T,Hkv,d], v [B,T,Hkv,dv] bf16; w [B,T] fp32 or None (mean pooling).
    Returns (kc, vc) of shape [B, T // blk, Hkv, d|dv] bf16.
    """
    _need(k, torch.bfloat16, "k")
    _need(v, torch.bfloat16, "v", k.device)
    B, T, Hkv, d = k.shape
    dv = v.shape[3]
    if w is not None:
        _need(w, torch.float32, "w", k.device)
    Nc = T // blk
    if kc is None:
        kc = torch.empty((B, Nc, Hkv, d), dtype=torch.bfloat16, device=k.device)
    if vc is None:
        vc = torch.empty((B, Nc, Hkv, dv), dtype=torch.bfloat16, device=k.device)
    _need(kc, torch.bfloat16, "kc", k.device)
    _need(vc, torch.bfloat16, "vc", k.device)
    _room(v, B * T * Hkv * dv, "v")
    _room(w, B * T, "w")
    _room(kc, B * Nc * Hkv * d, "kc")
    _room(vc, B * Nc * Hkv * dv, "vc")
    rc = _lib.load().hca_compress(_p(k), _p(v), _p(w), _p(kc), _p(vc), B, T, Hkv, d, dv, blk, _stream(k.device))
    _check(rc, "hca_compress")
    return kc, vc


def prefill(q, k, v, kc, vc, blk, W, scale, out=None, want_lse=False, out_f32=False):
    """Causal HCA attention for every position.  Returns out [B,T,Hq,dv] (and lse [B,Hq,T])."""
    _need(q, torch.bfloat16, "q")
    for name, t in (("k", k), ("v", v), ("kc", kc), ("vc", vc)):
        _need(t, torch.bfloat16, name, q.device)
    B, T, Hq, d = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    if out is None:
        out = torch.empty((B, T, Hq, dv), dtype=torch.float32 if out_f32 else torch.bfloat16, device=q.device)
    _need(out, torch.float32 if out_f32 else torch.bfloat16, "out", q.device)
    Nc = T // blk if blk > 0 else 0
    _room(k, B * T * Hkv * d, "k")
    _room(v, B * T * Hkv * dv, "v")
    _room(kc, B * Nc * Hkv * d, "kc")
    _room(vc, B * Nc * Hkv * dv, "vc")
    _room(out, B * T * Hq * dv, "out")
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device) if want_lse else None
    flags = (HCA_WRITE_LSE if want_lse else 0) | (HCA_OUT_F32 if out_f32 else 0)
    rc = _lib.load().hca_prefill(_p(q), _p(k), _p(v), _p(kc), _p(vc), _p(out), _p(lse), B, T, Hq, Hkv, d, dv,
                                 blk, W, float(scale), flags, _stream(q.device))
    _check(rc, "hca_prefill")
    return (out, lse) if want_lse else out


def prefill_backward(q, k, v, w, kc, vc, out, lse, dout, blk, W, scale, want_dw=True):
    """Gradients of sum(dout * out) for the layer (compress + prefill): dq [B,T,Hq,d],
    dk [B,T,Hkv,d], dv [B,T,Hkv,dv] (window path plus pooling path) and dw [B,T] (None if
    not wanted), all fp32.  ``out`` (bf16 or fp32) and ``lse`` [B,Hq,T] are the forward's
    (prefill with want_lse=True); kc, vc the compressed cache it read."""
    _need(q, torch.bfloat16, "q")
    for name, t in (("k", k), ("v", v), ("kc", kc), ("vc", vc), ("dout", dout)):
        _need(t, torch.bfloat16, name, q.device)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be bf16 or fp32")
    _need(out, out.dtype, "out", q.device)
    _need(lse, torch.float32, "lse", q.device)
    if w is not None:
        _need(w, torch.float32, "w", q.device)
    B, T, Hq, d = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    Nc = T // blk if blk > 0 else 0
    for name, t, n in (("k", k, B * T * Hkv * d), ("v", v, B * T * Hkv * dv), ("kc", kc, B * Nc * Hkv * d),
                       ("vc", vc, B * Nc * Hkv * dv), ("out", out, B * T * Hq * dv), ("lse", lse, B * Hq * T),
                       ("dout", dout, B * T * Hq * dv), ("w", w, B * T)):
        _room(t, n, name)
    dq = torch.empty((B, T, Hq, d), dtype=torch.float32, device=q.device)
    dk = torch.empty((B, T, Hkv, d), dtype=torch.float32, device=q.device)
    dvv = torch.empty((B, T, Hkv, dv), dtype=torch.float32, device=q.device)
    dw = torch.empty((B, T), dtype=torch.float32, device=q.device) if want_dw else None
    lib = _lib.load()
    nbytes = int(lib.hca_prefill_backward_workspace_size(B, T, Hq, Hkv, dv, blk, W))
    if nbytes == 0:
        raise HCAError(_lib.HCA_ERR_UNSUPPORTED, "hca_prefill_backward_workspace_size")
    ws = torch.empty((nbytes,), dtype=torch.uint8, device=q.device)
    flags = HCA_OUT_F32 if out.dtype == torch.float32 else 0
    rc = lib.hca_prefill_backward(_p(q), _p(k), _p(v), _p(w), _p(kc), _p(vc), _p(out), _p(lse), _p(dout), _p(dq),
                                  _p(dk), _p(dvv), _p(dw), _p(ws), nbytes, B, T, Hq, Hkv, d, dv, blk, W,
                                  float(scale), flags, _stream(q.device))
    _check(rc, "hca_prefill_backward")
    return dq, dk, dvv, dw


def dsa_index(q_idx, w_idx, k_idx, seqlens, scores=None):
    """Indexer scores of the sparse-attention decode step: q_idx [B,H_I,64] bf16, w_idx [B,H_I]
    fp32, k_idx [B,Lmax,64] bf16, seqlens [B] int32.  Returns scores [B,Lmax] fp32."""
    _need(q_idx, torch.bfloat16, "q_idx")
    dev = q_idx.device
    _need(w_idx, torch.float32, "w_idx", dev)
    _need(k_idx, torch.bfloat16, "k_idx", dev)
    _need(seqlens, torch.int32, "seqlens", dev)
    B, HI, dI = q_idx.shape
    Lmax = k_idx.shape[1]
    if scores is None:
        scores = torch.empty((B, Lmax), dtype=torch.float32, device=dev)
    _need(scores, torch.float32, "scores", dev)
    for name, t, n in (("w_idx", w_idx, B * HI), ("k_idx", k_idx, B * Lmax * dI), ("seqlens", seqlens, B),
                       ("scores", scores, B * Lmax)):
        _room(t, n, name)
    _check(_lib.load().hca_dsa_index(_p(q_idx), _p(w_idx), _p(k_idx), _p(seqlens), _p(scores), B, HI, dI, Lmax,
                                     _stream(dev)), "hca_dsa_index")
    return scores


def dsa_topk(scores, seqlens, k, idx=None):
    """Positions of the k largest scores per sequence (ascending, -1 padded): [B,k] int32."""
    _need(scores, torch.float32, "scores")
    dev = scores.device
    _need(seqlens, torch.int32, "seqlens", dev)
    B, Lmax = scores.shape
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=dev)
    _need(idx, torch.int32, "idx", dev)
    _room(idx, B * k, "idx")
    _room(seqlens, B, "seqlens")
    _check(_lib.load().hca_dsa_topk(_p(scores), _p(seqlens), _p(idx), B, Lmax, int(k), _stream(dev)), "hca_dsa_topk")
    return idx


def dsa_attend(q, k, v, idx, seqlens, scale, out=None):
    """Core attention over the kept positions: q [B,Hq,256], k / v [B,Lmax,256] bf16,
    idx [B,kmax] int32.  Returns out [B,Hq,256] fp32."""
    _need(q, torch.bfloat16, "q")
    dev = q.device
    for name, t in (("k", k), ("v", v)):
        _need(t, torch.bfloat16, name, dev)
    _need(idx, torch.int32, "idx", dev)
    _need(seqlens, torch.int32, "seqlens", dev)
    B, Hq, d = q.shape
    Lmax, kmax = k.shape[1], idx.shape[1]
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    _need(out, torch.float32, "out", dev)
    for name, t, n in (("k", k, B * Lmax * d), ("v", v, B * Lmax * d), ("seqlens", seqlens, B),
                       ("out", out, B * Hq * d)):
        _room(t, n, name)
    _check(_lib.load().hca_dsa_attend(_p(q), _p(k), _p(v), _p(idx), _p(seqlens), _p(out), B, Hq, d, Lmax, kmax,
                                      float(scale), _stream(dev)), "hca_dsa_attend")
    return out


def dsa_decode(q_idx, w_idx, k_idx, q, k, v, seqlens, topk, scale):
    """The whole sparse-attention decode step: scores, selection, attention.  Returns
    (out, idx, scores)."""
    scores = dsa_index(q_idx, w_idx, k_idx, seqlens)
    idx = dsa_topk(scores, seqlens, topk)
    return dsa_attend(q, k, v, idx, seqlens, scale), idx, scores


def decode_workspace_size(B, Hq, Hkv, dv) -> int:
    """Bytes of scratch ``decode`` needs on the current device."""
    return int(_lib.load().hca_decode_workspace_size(B, Hq, Hkv, dv))


def decode(q, kc, vc, kw, vw, seqlens, blk, W, scale, page_table=None, page_size=0,
           gq=None, gk=None, eps=1e-6, gate=None, out=None, workspace=None, window_ring=False,
           vha_u=None, vha_v=None):
    """One query per sequence at position seqlens[b]-1 over its compressed cache + raw window.

    q [B,Hq,d] bf16; kc/vc contiguous [B,Nmax,Hkv,d|dv] or page pools [P,page_size,Hkv,d|dv]
    with page_table [B,max_pages] int32; kw/vw [B,W,Hkv,d|dv] bf16; seqlens [B] int32;
    gq/gk [d] fp32 for QK RMSNorm; gate [B,Hq,dv] bf16 logits; vha_u/vha_v [Hq,r] fp32 Virtual
    Head Attention factors (mixing fused into the merge, hca_decode_vha).  Returns out [B,Hq,dv]
    fp32.
    """
    _need(q, torch.bfloat16, "q")
    dev = q.device
    for name, t in (("kc", kc), ("vc", vc), ("kw", kw), ("vw", vw)):
        _need(t, torch.bfloat16, name, dev)
    _need(seqlens, torch.int32, "seqlens", dev)
    B, Hq, d = q.shape
    Hkv, dv = kc.shape[2], vc.shape[3]
    flags = 0
    max_pages = num_pages = 0
    Nmax = kc.shape[1]
    if page_table is not None:
        _need(page_table, torch.int32, "page_table", dev)
        flags |= HCA_PAGED
        max_pages = page_table.shape[1]
        num_pages = kc.shape[0]
        page_size = kc.shape[1]
        Nmax = 0
    if gq is not None or gk is not None:
        _need(gq, torch.float32, "gq", dev)
        _need(gk, torch.float32, "gk", dev)
        flags |= HCA_QK_NORM
    if gate is not None:
        _need(gate, torch.bfloat16, "gate", dev)
        flags |= HCA_OUT_GATE
    if window_ring:
        flags |= HCA_WINDOW_RING
    if out is None:
        out = torch.empty((B, Hq, dv), dtype=torch.float32, device=dev)
    _need(out, torch.float32, "out", dev)
    rows = num_pages * page_size if page_table is not None else B * Nmax
    _room(kc, rows * Hkv * d, "kc")
    _room(vc, rows * Hkv * dv, "vc")
    _room(page_table, B * max_pages, "page_table")
    _room(kw, B * W * Hkv * d, "kw")
    _room(vw, B * W * Hkv * dv, "vw")
    _room(seqlens, B, "seqlens")
    _room(gq, d, "gq")
    _room(gk, d, "gk")
    _room(gate, B * Hq * dv, "gate")
    _room(out, B * Hq * dv, "out")
    ws_bytes = decode_workspace_size(B, Hq, Hkv, dv)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    _need(workspace, torch.uint8, "workspace", dev)
    if vha_u is not None or vha_v is not None:
        _need(vha_u, torch.float32, "vha_u", dev)
        _need(vha_v, torch.float32, "vha_v", dev)
        r = vha_u.shape[1]
        if vha_u.shape != (Hq, r) or vha_v.shape != (Hq, r):
            raise ValueError("vha_u and vha_v must both be [Hq, r]")
        rc = _lib.load().hca_decode_vha(_p(q), _p(kc), _p(vc), _p(page_table), int(page_size), int(max_pages),
                                        int(num_pages), _p(kw), _p(vw), _p(seqlens), _p(gq), _p(gk), float(eps),
                                        _p(gate), _p(vha_u), _p(vha_v), int(r), _p(out), _p(workspace),
                                        workspace.numel(), B, Hq, Hkv, d, dv, blk, W, Nmax, float(scale), flags,
                                        _stream(dev))
        _check(rc, "hca_decode_vha")
        return out
    rc = _lib.load().hca_decode(_p(q), _p(kc), _p(vc), _p(page_table), int(page_size), int(max_pages),
                                int(num_pages), _p(kw), _p(vw), _p(seqlens), _p(gq), _p(gk), float(eps), _p(gate), _p(out),
                                _p(workspace), workspace.numel(), B, Hq, Hkv, d, dv, blk, W, Nmax,
                                float(scale), flags, _stream(dev))
    _check(rc, "hca_decode")
    return out


def append_state_size(B, Hkv, d, dv) -> int:
    """Bytes of pooling state ``append`` keeps for a batch (zero it before a sequence starts)."""
    return int(_lib.load().hca_append_state_size(B, Hkv, d, dv))


def append(k_new, v_new, w_new, seqlens, kw, vw, kc, vc, state, blk, page_table=None):
    """One decode step's cache update: the newest token of each sequence enters the window
    ring (slot (L-1) % W), and a block it completes is pooled into the compressed cache.

    k_new [B,Hkv,d], v_new [B,Hkv,dv] bf16; w_new [B] fp32 or None; seqlens [B] int32 (length
    including the new token); kw/vw [B,W,Hkv,d|dv] bf16 rings; kc/vc contiguous
    [B,Nmax,Hkv,d|dv] or page pools with page_table [B,max_pages] int32; state: a uint8 or
    float32 tensor of ``append_state_size`` bytes, zero for an empty block.
    """
    _need(k_new, torch.bfloat16, "k_new")
    dev = k_new.device
    _need(v_new, torch.bfloat16, "v_new", dev)
    for name, t in (("kw", kw), ("vw", vw), ("kc", kc), ("vc", vc)):
        _need(t, torch.bfloat16, name, dev)
    _need(seqlens, torch.int32, "seqlens", dev)
    if w_new is not None:
        _need(w_new, torch.float32, "w_new", dev)
    if not isinstance(state, torch.Tensor) or state.dtype not in (torch.uint8, torch.float32):
        raise TypeError("state must be a uint8 or float32 torch.Tensor")
    _need(state, state.dtype, "state", dev)
    B, Hkv, d = k_new.shape
    dv = v_new.shape[2]
    W = kw.shape[1]
    if state.numel() * state.element_size() < append_state_size(B, Hkv, d, dv):
        raise ValueError("state is smaller than append_state_size()")
    flags = 0
    max_pages = num_pages = page_size = 0
    Nmax = kc.shape[1]
    if page_table is not None:
        _need(page_table, torch.int32, "page_table", dev)
        flags |= HCA_PAGED
        max_pages = page_table.shape[1]
        num_pages = kc.shape[0]
        page_size = kc.shape[1]
        Nmax = 0
    rows = num_pages * page_size if page_table is not None else B * Nmax
    _room(v_new, B * Hkv * dv, "v_new")
    _room(w_new, B, "w_new")
    _room(seqlens, B, "seqlens")
    _room(kw, B * W * Hkv * d, "kw")
    _room(vw, B * W * Hkv * dv, "vw")
    _room(kc, rows * Hkv * d, "kc")
    _room(vc, rows * Hkv * dv, "vc")
    _room(page_table, B * max_pages, "page_table")
    rc = _lib.load().hca_append(_p(k_new), _p(v_new), _p(w_new), _p(seqlens), _p(kw), _p(vw), _p(kc), _p(vc),
                                _p(page_table), int(page_size), int(max_pages), int(num_pages), _p(state),
                                B, Hkv, d, dv, int(blk), int(W), int(Nmax), flags, _stream(dev))
    _check(rc, "hca_append")


def vha(out, U, V):
    """Virtual Head Attention in place on an attention output ``out`` [..., Hq, dv] (bf16 or
    fp32): per token and channel, out[:, c] <- (I + U V^T) out[:, c] over the heads.
    U, V [Hq, r] fp32.  Returns ``out``."""
    if not isinstance(out, torch.Tensor) or out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be a bf16 or fp32 torch.Tensor")
    _need(out, out.dtype, "out")
    dev = out.device
    _need(U, torch.float32, "U", dev)
    _need(V, torch.float32, "V", dev)
    Hq, dv = out.shape[-2], out.shape[-1]
    n = out.numel() // (Hq * dv)
    r = U.shape[1]
    if U.shape != (Hq, r) or V.shape != (Hq, r):
        raise ValueError("U and V must both be [Hq, r]")
    flags = HCA_OUT_F32 if out.dtype == torch.float32 else 0
    _check(_lib.load().hca_vha(_p(out), _p(U), _p(V), int(n), Hq, dv, r, flags, _stream(dev)), "hca_vha")
    return out



def gate_logits(cq, wg, out=None):
    """Low-Rank Gated Attention's gate projection: gate[i, h, c] = sum_k cq[i, k] wg[k, h, c].
    cq [n, rq] bf16 query latents, wg [rq, Hq, dv] bf16.  Returns gate logits [n, Hq, dv] bf16,
    the ``gate`` argument of ``decode``."""
    _need(cq, torch.bfloat16, "cq")
    _need(wg, torch.bfloat16, "wg", cq.device)
    n, rq = cq.shape
    if wg.dim() != 3 or wg.shape[0] != rq:
        raise ValueError("wg must be [rq, Hq, dv] with rq = cq.shape[1]")
    Hq, dv = wg.shape[1], wg.shape[2]
    if out is None:
        out = torch.empty((n, Hq, dv), dtype=torch.bfloat16, device=cq.device)
    _need(out, torch.bfloat16, "gate", cq.device)
    _room(out, n * Hq * dv, "gate")
    _check(_lib.load().hca_gate_logits(_p(cq), _p(wg), _p(out), n, rq, Hq, dv, _stream(cq.device)), "hca_gate_logits")
    return out
