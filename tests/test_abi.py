"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/sdpa.h declares, and rejects bad arguments before
queuing any work (those calls return before touching CUDA)."""
import ctypes
import os
import re

import pytest
import torch

from scaled_dot_product_bwd_b200 import binding
from scaled_dot_product_bwd_b200.build import LIB_PATH, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdpa.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sdpa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "sdpa_fwd" in names and "sdpa_bwd" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding.EXPORTED)


def test_library_is_in_tree():
    build()
    assert os.path.dirname(LIB_PATH) == os.path.join(ROOT, "scaled_dot_product_bwd_b200")
    assert os.path.exists(LIB_PATH)


def test_status_strings(lib):
    for code in range(6):
        assert binding.sdpa_status_string(code)
    assert binding.sdpa_status_string(5) == "in-kernel wait timed out"


def _shape(**kw):
    base = dict(B=1, L=128, Hq=4, Hkv=2, d=64, sq_b=128 * 4 * 64, sq_l=4 * 64, sq_h=64,
                skv_b=128 * 2 * 64, skv_l=2 * 64, skv_h=64, Lk=0)
    base.update(kw)
    return binding.Shape(*[base[n] for n, _ in binding.Shape._fields_])


FAKE = ctypes.c_void_p(0x10000)   # aligned, never dereferenced: validation fails first


def _fwd(lib, shape, mask=None, bias=None, scale=0.125, ptr=FAKE, lse=FAKE):
    mask = mask or binding.MaskSpec(1, -1, -1)
    return lib.sdpa_fwd(ctypes.byref(shape), ptr, ptr, ptr,
                        ctypes.byref(bias) if bias is not None else None,
                        ctypes.byref(mask), scale, ptr, lse, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), 2), (dict(d=32), 2), (dict(Hq=3, Hkv=2), 1), (dict(L=0), 1),
    (dict(B=0), 1), (dict(sq_l=4 * 64 + 4), 1), (dict(skv_h=0), 1), (dict(Hkv=0), 1),
])
def test_fwd_rejects_bad_shapes(lib, kw, code):
    assert _fwd(lib, _shape(**kw)) == code


def test_fwd_rejects_null_and_misaligned(lib):
    assert _fwd(lib, _shape(), ptr=ctypes.c_void_p(0)) == 1
    assert _fwd(lib, _shape(), ptr=ctypes.c_void_p(0x10008)) == 1
    assert lib.sdpa_fwd(None, FAKE, FAKE, FAKE, None, None, 0.1, FAKE, FAKE, None) == 1
    assert _fwd(lib, _shape(), scale=float("nan")) == 1


def test_fwd_rejects_bad_bias(lib):
    bad = [binding.BiasDesc(7, 0x10000, 0, 0, 0, 0, 0, 0),           # unknown kind
           binding.BiasDesc(1, 0, 0, 0, 128, 0, 0, 0),               # dense, null
           binding.BiasDesc(1, 0x10004, 0, 0, 128, 0, 0, 0),         # dense, misaligned
           binding.BiasDesc(1, 0x10000, 0, 0, 130, 0, 0, 0),         # dense, stride_i % 4
           binding.BiasDesc(1, 0x10000, 0, 2, 128, 0, 0, 0),         # dense, stride_h % 4
           binding.BiasDesc(1, 0x10000, 6, 0, 128, 0, 0, 0),         # dense, stride_b % 4
           binding.BiasDesc(2, 0x10000, 0, 0, 0, 31, 128, 1),        # T5, odd buckets (bidir)
           binding.BiasDesc(2, 0x10000, 0, 0, 0, 256, 128, 1),       # T5, too many buckets
           binding.BiasDesc(2, 0x10000, 0, 0, 0, 32, 8, 1),          # T5, max_distance <= max_exact
           binding.BiasDesc(2, 0, 0, 0, 0, 32, 128, 1),              # T5, null table
           binding.BiasDesc(3, 0, 0, 0, 0, 0, 0, 0)]                 # ALiBi, null slopes
    for b in bad:
        assert _fwd(lib, _shape(), bias=b) == 1, (b.kind, b.num_buckets)


def test_bwd_rejects_bad_args(lib):
    s = _shape()
    m = binding.MaskSpec(1, -1, -1)
    ws = lib.sdpa_bwd_workspace_size(ctypes.byref(s), 1)
    assert ws >= 128 * 4 * 4 and ws % 256 == 0

    def call(det=1, wsp=FAKE, wsb=ws, shape=s):
        return lib.sdpa_bwd(ctypes.byref(shape), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                            ctypes.byref(m), 0.125, FAKE, FAKE, FAKE, det, wsp, wsb, None)
    assert call(det=0) == 2                               # only deterministic mode is built
    assert call(wsp=ctypes.c_void_p(0)) == 3
    assert call(wsp=ctypes.c_void_p(0x10010)) == 3        # not 256-byte aligned
    assert call(wsb=ws - 1) == 3
    assert call(shape=_shape(d=80)) == 2
    assert lib.sdpa_bwd_workspace_size(None, 1) == 0


def test_bwd_workspace_layout(lib):
    # D, one float per LSE entry, rounded up to 256 bytes.
    r256 = lambda x: (x + 255) // 256 * 256
    for B, L, Hq, d, Lk in ((1, 128, 4, 64, 0), (2, 300, 4, 128, 0), (3, 37, 2, 64, 1000)):
        s = _shape(B=B, L=L, Hq=Hq, d=d, Lk=Lk)
        want = r256(B * Hq * L * 4)
        assert lib.sdpa_bwd_workspace_size(ctypes.byref(s), 1) == want
    assert lib.sdpa_bwd_workspace_size(ctypes.byref(_shape(Lk=-1)), 1) == 0


def test_bwd_phases_rejects_bad_bits(lib):
    s = _shape()
    m = binding.MaskSpec(1, -1, -1)
    ws = lib.sdpa_bwd_workspace_size(ctypes.byref(s), 1)
    for ph in (0, 8, 9, 16, 0x80000007):
        assert lib.sdpa_bwd_phases(ph, ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                   ctypes.byref(m), 0.125, FAKE, FAKE, FAKE, 1, FAKE, ws,
                                   None) == 1


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    m = binding.MaskSpec(1, -1, -1)
    L = 1 << 20  # B * Hq * L = 8M LSE entries: 32 MiB of D
    big = _shape(B=1, L=L, Hq=8, d=64, sq_b=L * 8 * 64, sq_l=8 * 64, sq_h=64,
                 skv_b=L * 2 * 64, skv_l=2 * 64, skv_h=64)
    assert lib.sdpa_bwd_workspace_size(ctypes.byref(big), 1) > binding.NOALLOC_SCRATCH_BYTES
    assert lib.sdpa_bwd_noalloc(ctypes.byref(big), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                ctypes.byref(m), 0.1, FAKE, FAKE, FAKE, 1, None) == 3


def _varlen(**kw):
    base = dict(cu_seqlens_q=0x20000, cu_seqlens_k=0x20100, max_seqlen_q=300, max_seqlen_k=300,
                total_q=1000, total_k=1000)
    base.update(kw)
    return binding.Varlen(*[base[n] for n, _ in binding.Varlen._fields_])


def test_varlen_rejects_bad_args(lib):
    s = binding.Shape(3, 0, 4, 2, 64, 0, 4 * 64, 64, 0, 2 * 64, 64, 0)
    m = binding.MaskSpec(1, -1, -1)

    def fwd(vl, bias=None, shape=s):
        return lib.sdpa_fwd_varlen(ctypes.byref(shape), ctypes.byref(vl) if vl else None, FAKE,
                                   FAKE, FAKE, ctypes.byref(bias) if bias else None,
                                   ctypes.byref(m), 0.125, FAKE, FAKE, None)
    assert fwd(None) == 1
    for bad in (dict(cu_seqlens_q=0), dict(cu_seqlens_k=0x20102), dict(max_seqlen_q=0),
                dict(max_seqlen_k=-3), dict(total_q=0), dict(total_k=0)):
        assert fwd(_varlen(**bad)) == 1, bad
    assert fwd(_varlen(total_q=1 << 30)) == 2
    assert fwd(_varlen(), bias=_dense(0, 0, 300)) == 2       # no packed form of a dense bias
    assert fwd(_varlen(), shape=binding.Shape(3, 0, 4, 2, 96, 0, 4 * 96, 96, 0, 2 * 96, 96, 0)) == 2
    assert lib.sdpa_bwd_varlen_workspace_size(ctypes.byref(s), None) == 0
    # D, one float per LSE row: Hq * total_q rows
    want = (4 * 1000 * 4 + 255) // 256 * 256
    assert lib.sdpa_bwd_varlen_workspace_size(ctypes.byref(s), ctypes.byref(_varlen())) == want


def _dense(sb, sh, si, ptr=0x10000):
    return binding.BiasDesc(1, ptr, sb, sh, si, 0, 0, 0)


def test_bias_grad_workspace_size(lib):
    B, L, Hq = 2, 128, 4
    s = _shape(B=B, sq_b=128 * 4 * 64, skv_b=128 * 2 * 64)
    ws = lambda bias: lib.sdpa_bwd_bias_grad_workspace_size(ctypes.byref(s), ctypes.byref(bias))
    d_bytes = lib.sdpa_bwd_workspace_size(ctypes.byref(s), 1)
    ds_bytes = B * Hq * L * L * 4
    # full-shape dense bias: dS goes straight into dbias, only D is staged
    assert ws(_dense(Hq * L * L, L * L, L)) == d_bytes
    # a padded full-shape bias needs no more
    assert ws(_dense(Hq * L * (L + 4), L * (L + 4), L + 4)) == d_bytes
    # broadcast over heads, over batch, over both: dS is staged and reduced
    for b in (_dense(L * L, 0, L), _dense(0, L * L, L), _dense(0, 0, L)):
        n = ws(b)
        assert n >= d_bytes + ds_bytes and n % 256 == 0
    # T5: no dS; per (batch, head, query tile) 8 warps x 32 per-bucket sums
    r256 = lambda x: (x + 255) // 256 * 256
    nt = (L + 127) // 128
    tiles = B * Hq * nt * nt
    t5 = binding.BiasDesc(2, 0x10000, 0, 0, 0, 32, 128, 1)
    assert ws(t5) == d_bytes + r256(B * Hq * nt * 8 * 32 * 4)
    # REL: no dS; per (batch, head, query tile, key tile) 1024 per-warp
    # diagonal sums and 256 tile diagonals, per (batch, head, tile offset)
    # 256 band sums, per head 2L - 1 totals
    want = (d_bytes + r256(tiles * 1024 * 4) + r256(tiles * 256 * 4) +
            r256(B * Hq * (2 * nt - 1) * 256 * 4) + r256(Hq * (2 * L - 1) * 4))
    rel = binding.BiasDesc(4, 0x10000, 0, 0, 0, 0, 0, 0)
    assert ws(rel) == want
    # ALiBi: per (batch, head, query tile, key tile) 8 per-warp sums of |j - i| dS
    alibi = binding.BiasDesc(3, 0x10000, 0, 0, 0, 0, 0, 0)
    assert ws(alibi) == d_bytes + r256(tiles * 8 * 4)
    assert ws(binding.BiasDesc(0, None, 0, 0, 0, 0, 0, 0)) == 0       # nothing to differentiate
    assert ws(_dense(L * L, L * L, L)) == 0                          # heads overlap batches
    assert ws(_dense(Hq * L * L, L * L, 0)) == 0                      # one row for all queries
    assert lib.sdpa_bwd_bias_grad_workspace_size(None, ctypes.byref(t5)) == 0


def test_bias_grad_rejects_bad_args(lib):
    B, L, Hq = 2, 128, 4
    s = _shape(B=B)
    m = binding.MaskSpec(1, -1, -1)
    full = _dense(Hq * L * L, L * L, L)
    need = lib.sdpa_bwd_bias_grad_workspace_size(ctypes.byref(s), ctypes.byref(full))

    def call(bias=full, dbias=FAKE, det=1, wsb=need, wsp=FAKE):
        return lib.sdpa_bwd_bias_grad(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                      ctypes.byref(bias) if bias is not None else None,
                                      ctypes.byref(m), 0.125, FAKE, FAKE, FAKE, dbias, det, wsp,
                                      wsb, None)
    assert call(bias=None) == 2                                      # no bias
    assert call(bias=binding.BiasDesc(0, None, 0, 0, 0, 0, 0, 0)) == 2
    assert call(bias=_dense(Hq * L * L, L * L, 0)) == 2              # row-broadcast bias
    assert call(bias=_dense(L * L, L * L, L)) == 2                   # overlapping layout
    assert call(dbias=ctypes.c_void_p(0)) == 1
    assert call(dbias=ctypes.c_void_p(0x10008)) == 1                 # not 16-byte aligned
    assert call(det=0) == 2
    assert call(wsb=need - 1) == 3
    assert call(wsp=ctypes.c_void_p(0x10040)) == 3                   # not 256-byte aligned


def test_binding_checks_bias_shapes():
    import torch
    ok = torch.zeros(1, 4, 16, 16)
    binding.make_bias(ok, None, 32, 128, True, (2, 4, 16))
    for bad in (torch.zeros(2, 4, 1, 16), torch.zeros(3, 4, 16, 16), torch.zeros(1, 2, 16, 16),
                torch.zeros(1, 4, 16, 8)):
        with pytest.raises(ValueError):
            binding.make_bias(bad, None, 32, 128, True, (2, 4, 16))
    with pytest.raises(ValueError):
        binding.make_bias(None, torch.zeros(32, 3), 32, 128, True, (2, 4, 16))
    binding.make_bias(None, None, 32, 128, True, (2, 4, 16), torch.zeros(4))
    with pytest.raises(ValueError):                                   # one slope per head
        binding.make_bias(None, None, 32, 128, True, (2, 4, 16), torch.zeros(3))
    with pytest.raises(ValueError):                                   # one bias at a time
        binding.make_bias(ok, None, 32, 128, True, (2, 4, 16), torch.zeros(4))


def test_binding_entry_points_share_the_bias_keywords():
    import inspect
    keys = {"causal", "window_left", "window_right", "bias", "t5_table", "t5_num_buckets",
            "t5_max_distance", "t5_bidirectional", "alibi_slopes", "scale"}
    for fn in (binding.sdpa_fwd, binding.sdpa_bwd, binding.sdpa_bwd_noalloc,
               binding.sdpa_bwd_bias_grad):
        missing = keys - set(inspect.signature(fn).parameters)
        assert not missing, (fn.__name__, missing)
    for fn in (binding.sdpa_fwd_varlen, binding.sdpa_bwd_varlen):   # no dense bias when packed
        missing = (keys - {"bias"}) - set(inspect.signature(fn).parameters)
        assert not missing, (fn.__name__, missing)


def test_t5_bucket_rejects_bad_args(lib):
    assert lib.sdpa_t5_bucket(FAKE, FAKE, -1, 32, 128, 1, None) == 1
    assert lib.sdpa_t5_bucket(None, None, 5, 32, 128, 1, None) == 1
    assert lib.sdpa_t5_bucket(FAKE, FAKE, 4, 33, 128, 1, None) == 1
    assert lib.sdpa_t5_bucket(FAKE, FAKE, 0, 32, 128, 1, None) == 0   # nothing to do


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError):
        binding.load_library(str(tmp_path / "missing.so"))


def test_fire_rejects_bad_args(lib):
    def fire(**kw):
        base = dict(w1=0x10000, b1=0x10000, w2=0x10000, b2=0x10000, c=0.5, threshold=300.0,
                    width=32, heads=4)
        base.update(kw)
        return binding.Fire(*[base[n] for n, _ in binding.Fire._fields_])

    def table(f, Lq=200, Lk=150, out=FAKE):
        return lib.sdpa_fire_table(ctypes.byref(f) if f else None, Lq, Lk, out, None)
    assert table(None) == 1
    assert table(fire(w2=0)) == 1
    assert table(fire(b1=0x10002)) == 1                   # not 4-byte aligned
    for bad in (dict(width=0), dict(width=1025), dict(heads=0), dict(c=0.0), dict(c=-1.0),
                dict(c=float("nan")), dict(threshold=float("inf"))):
        assert table(fire(**bad)) == 1, bad
    assert table(fire(), Lq=0) == 1
    assert table(fire(), out=None) == 1
    assert table(fire(threshold=198.0)) == 2             # below the last query position
    # workspace: hidden activations and their gradients [R, W], then x, dx/dc, dx/dT [R]
    r256 = lambda x: (x + 255) // 256 * 256
    R = 200 + 150 - 1
    want = 2 * r256(R * 32 * 4) + 3 * r256(R * 4)
    assert lib.sdpa_fire_backward_workspace_size(ctypes.byref(fire()), 200, 150) == want
    assert lib.sdpa_fire_backward_workspace_size(ctypes.byref(fire(threshold=10.0)), 200, 150) == 0
    args = [FAKE] * 6
    assert lib.sdpa_fire_backward(ctypes.byref(fire()), 200, 150, *args, FAKE, want - 1, None) == 3
    assert lib.sdpa_fire_backward(ctypes.byref(fire()), 200, 150, *args, None, want, None) == 3
    assert lib.sdpa_fire_backward(ctypes.byref(fire()), 200, 150, None, *args[1:], FAKE, want,
                                  None) == 1


def test_rel_table_bias_checks(lib):
    s = _shape()
    rel = binding.BiasDesc(4, None, 0, 0, 0, 0, 0, 0)
    assert _fwd(lib, s, bias=rel) == 1                       # no table
    with pytest.raises(ValueError):
        binding.make_bias(None, None, 32, 128, True, (1, 4, 128), None,
                          torch.zeros(200, 4))               # rows != L + Lk - 1
