"""Host-side checks of the Python binding, on CPU: the footprint checks refuse a buffer that
is smaller than what the C call would address, before anything reaches the library, and
accept the shapes the library's own tests use.  The library is replaced by a stub that
records the calls (no kernel runs; the dtype checks stay, the CUDA-device check is lifted)."""
import pytest
import torch

import compressed_long_context_b200 as hca


class StubLib:
    def __init__(self):
        self.calls = []

    def hca_append_state_size(self, B, Hkv, d, dv):
        return B * Hkv * (4 + d + dv) * 4

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return 0
        return fn


@pytest.fixture
def stub(monkeypatch):
    lib = StubLib()
    monkeypatch.setattr(hca._lib, "load", lambda: lib)
    monkeypatch.setattr(hca, "_stream", lambda device: 0)

    def need(t, dtype, name, device=None):
        if not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_contiguous():
            raise TypeError(name)
    monkeypatch.setattr(hca, "_need", need)
    return lib


bf = torch.bfloat16


def z(*shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


def test_room_helper():
    hca._room(z(4), 4, "x")
    hca._room(None, 10, "x")
    with pytest.raises(ValueError, match="x holds 3 elements, the call addresses 4"):
        hca._room(z(3), 4, "x")


def test_compress_footprints(stub):
    k, v, w = z(2, 300, 1, 64), z(2, 300, 1, 32), z(2, 300, dtype=torch.float32)
    kc, vc = hca.compress(k, v, w, 128)
    assert kc.shape == (2, 2, 1, 64) and vc.shape == (2, 2, 1, 32)
    assert stub.calls == ["hca_compress"]
    with pytest.raises(ValueError, match="kc"):
        hca.compress(k, v, w, 128, kc=z(2, 1, 1, 64), vc=vc)
    with pytest.raises(ValueError, match="w"):
        hca.compress(k, v, z(2, 299, dtype=torch.float32), 128)
    with pytest.raises(ValueError, match="v"):
        hca.compress(k, v[:1].contiguous(), w, 128)
    assert stub.calls == ["hca_compress"]


def test_prefill_footprints(stub):
    q, k, v = z(1, 400, 8, 64), z(1, 400, 1, 64), z(1, 400, 1, 64)
    kc, vc = z(1, 3, 1, 64), z(1, 3, 1, 64)
    out = hca.prefill(q, k, v, kc, vc, 128, 128, 0.125)
    assert out.shape == (1, 400, 8, 64)
    hca.prefill(q, k, v, kc, vc, 128, 128, 0.125, out_f32=True, want_lse=True)
    with pytest.raises(ValueError, match="kc"):
        hca.prefill(q, k, v, z(1, 2, 1, 64), vc, 128, 128, 0.125)
    with pytest.raises(ValueError, match="out"):
        hca.prefill(q, k, v, kc, vc, 128, 128, 0.125, out=z(1, 400, 8, 63))
    assert stub.calls == ["hca_prefill"] * 2


def test_decode_footprints(stub):
    B, Hq, d, W = 3, 64, 512, 128
    q = z(B, Hq, d)
    kc, vc = z(B, 160, 1, d), z(B, 160, 1, d)
    kw, vw = z(B, W, 1, d), z(B, W, 1, d)
    seq = z(B, dtype=torch.int32)
    gq, gk = z(d, dtype=torch.float32), z(d, dtype=torch.float32)
    gate = z(B, Hq, d)
    hca.decode(q, kc, vc, kw, vw, seq, 128, W, 0.05, gq=gq, gk=gk, gate=gate, window_ring=True)
    # paged: pools [P, 64, Hkv, d] with a [B, max_pages] table
    table = z(B, 3, dtype=torch.int32)
    hca.decode(q, z(9, 64, 1, d), z(9, 64, 1, d), kw, vw, seq, 128, W, 0.05, page_table=table, page_size=64)
    n = len(stub.calls)
    for kwargs, name in ((dict(kw=z(B, W - 1, 1, d)), "kw"), (dict(vw=z(B - 1, W, 1, d)), "vw"),
                         (dict(seqlens=z(B - 1, dtype=torch.int32)), "seqlens"),
                         (dict(gate=z(B, Hq - 1, d)), "gate"), (dict(gq=z(d - 1, dtype=torch.float32)), "gq"),
                         (dict(out=z(B, Hq, d - 1, dtype=torch.float32)), "out")):
        args = dict(kw=kw, vw=vw, seqlens=seq, gate=gate, gq=gq, gk=gk)
        args.update(kwargs)
        with pytest.raises(ValueError, match=name):
            hca.decode(q, kc, vc, args["kw"], args["vw"], args["seqlens"], 128, W, 0.05, gq=args["gq"],
                       gk=args["gk"], gate=args["gate"], out=args.get("out"))
    with pytest.raises(ValueError, match="kc"):
        hca.decode(q, kc[:2].contiguous(), vc[:2].contiguous(), kw, vw, seq, 128, W, 0.05)
    assert len(stub.calls) == n


def test_append_footprints(stub):
    B, Hkv, d, W = 2, 2, 512, 200
    kn, vn = z(B, Hkv, d), z(B, Hkv, d)
    seq = z(B, dtype=torch.int32)
    kw, vw = z(B, W, Hkv, d), z(B, W, Hkv, d)
    st = torch.zeros(B * Hkv * (4 + 2 * d), dtype=torch.float32)
    hca.append(kn, vn, None, seq, kw, vw, z(B, 6, Hkv, d), z(B, 6, Hkv, d), st, 128)
    table = z(B, 5, dtype=torch.int32)
    hca.append(kn, vn, z(B, dtype=torch.float32), seq, kw, vw, z(13, 64, Hkv, d), z(13, 64, Hkv, d), st, 128,
               page_table=table)
    n = len(stub.calls)
    with pytest.raises(ValueError, match="kw"):
        hca.append(kn, vn, None, seq, z(1, W, Hkv, d), vw, z(B, 6, Hkv, d), z(B, 6, Hkv, d), st, 128)
    with pytest.raises(ValueError, match="v_new"):
        hca.append(kn, z(B, 1, d), None, seq, kw, vw, z(B, 6, Hkv, d), z(B, 6, Hkv, d), st, 128)
    with pytest.raises(ValueError, match="vc"):
        hca.append(kn, vn, None, seq, kw, vw, z(B, 6, Hkv, d), z(1, 6, Hkv, d), st, 128)
    with pytest.raises(ValueError, match="state"):
        hca.append(kn, vn, None, seq, kw, vw, z(B, 6, Hkv, d), z(B, 6, Hkv, d), st[:-1], 128)
    assert len(stub.calls) == n


def test_vha_shapes(stub):
    out = z(5, 16, 128)
    hca.vha(out, z(16, 3, dtype=torch.float32), z(16, 3, dtype=torch.float32))
    with pytest.raises(ValueError):
        hca.vha(out, z(16, 3, dtype=torch.float32), z(16, 2, dtype=torch.float32))
