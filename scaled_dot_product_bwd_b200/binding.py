"""ctypes binding of the C ABI in include/sdpa.h (argument marshalling only).

Every function here converts torch tensors into pointers, sizes and strides,
calls the entry point of the same name in libsdpa_b200.so on the current CUDA
stream, and turns a non-OK status into an exception.  All arithmetic runs in
the library's kernels; there is no fallback: if the library is missing or
cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsdpa_b200.so")

SDPA_OK = 0
STATUS_NAMES = {0: "SDPA_OK", 1: "SDPA_ERR_INVALID_ARG", 2: "SDPA_ERR_UNSUPPORTED",
                3: "SDPA_ERR_WORKSPACE", 4: "SDPA_ERR_CUDA", 5: "SDPA_ERR_TIMEOUT"}
BIAS_NONE, BIAS_DENSE, BIAS_T5, BIAS_ALIBI, BIAS_REL = 0, 1, 2, 3, 4

BWD_PREPROCESS, BWD_DQ, BWD_DKDV, BWD_ALL = 1, 2, 4, 7

NOALLOC_SCRATCH_BYTES = 16 << 20

EXPORTED = ("sdpa_fwd", "sdpa_fwd_varlen", "sdpa_bwd", "sdpa_bwd_phases", "sdpa_bwd_varlen",
            "sdpa_bwd_noalloc", "sdpa_bwd_workspace_size", "sdpa_bwd_varlen_workspace_size",
            "sdpa_bwd_bias_grad", "sdpa_bwd_bias_grad_workspace_size", "sdpa_t5_bucket",
            "sdpa_exp2_fma", "sdpa_read_device_status", "sdpa_set_wait_limit_ns",
            "sdpa_debug_wait_timeout", "sdpa_status_string", "sdpa_fire_table",
            "sdpa_fire_backward_workspace_size", "sdpa_fire_backward")


class SdpaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class MaskSpec(ctypes.Structure):
    _fields_ = [("causal", ctypes.c_int32), ("window_left", ctypes.c_int64),
                ("window_right", ctypes.c_int64)]


class BiasDesc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("ptr", ctypes.c_void_p),
                ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64),
                ("stride_i", ctypes.c_int64), ("num_buckets", ctypes.c_int32),
                ("max_distance", ctypes.c_int32), ("bidirectional", ctypes.c_int32)]


class Fire(ctypes.Structure):
    _fields_ = [("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                ("b2", ctypes.c_void_p), ("c", ctypes.c_float), ("threshold", ctypes.c_float),
                ("width", ctypes.c_int32), ("heads", ctypes.c_int32)]


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("B", "L", "Hq", "Hkv", "d", "sq_b", "sq_l", "sq_h", "skv_b", "skv_l", "skv_h",
                 "Lk")]


class Varlen(ctypes.Structure):
    _fields_ = [("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
                ("max_seqlen_q", ctypes.c_int64), ("max_seqlen_k", ctypes.c_int64),
                ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64)]


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libsdpa_b200.so once and declare the signatures.  Raises if absent."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"CUDA library not built: {p} (run scaled_dot_product_bwd_b200.build)")
    lib = ctypes.CDLL(p)
    vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
    sp, bp, mp = ctypes.POINTER(Shape), ctypes.POINTER(BiasDesc), ctypes.POINTER(MaskSpec)
    vlp = ctypes.POINTER(Varlen)
    lib.sdpa_fwd.argtypes = [sp, vp, vp, vp, bp, mp, f32, vp, vp, vp]
    lib.sdpa_fwd.restype = i32
    lib.sdpa_fwd_varlen.argtypes = [sp, vlp, vp, vp, vp, bp, mp, f32, vp, vp, vp]
    lib.sdpa_fwd_varlen.restype = i32
    lib.sdpa_bwd.argtypes = [sp, vp, vp, vp, vp, vp, vp, bp, mp, f32, vp, vp, vp, i32, vp, sz, vp]
    lib.sdpa_bwd.restype = i32
    lib.sdpa_bwd_varlen.argtypes = [sp, vlp] + lib.sdpa_bwd.argtypes[1:]
    lib.sdpa_bwd_varlen.restype = i32
    lib.sdpa_bwd_varlen_workspace_size.argtypes = [sp, vlp]
    lib.sdpa_bwd_varlen_workspace_size.restype = sz
    lib.sdpa_bwd_phases.argtypes = [ctypes.c_uint32] + lib.sdpa_bwd.argtypes
    lib.sdpa_bwd_phases.restype = i32
    lib.sdpa_bwd_noalloc.argtypes = [sp, vp, vp, vp, vp, vp, vp, bp, mp, f32, vp, vp, vp, i32, vp]
    lib.sdpa_bwd_noalloc.restype = i32
    lib.sdpa_bwd_workspace_size.argtypes = [sp, i32]
    lib.sdpa_bwd_workspace_size.restype = sz
    lib.sdpa_bwd_bias_grad.argtypes = [sp, vp, vp, vp, vp, vp, vp, bp, mp, f32, vp, vp, vp, vp,
                                       i32, vp, sz, vp]
    lib.sdpa_bwd_bias_grad.restype = i32
    lib.sdpa_bwd_bias_grad_workspace_size.argtypes = [sp, bp]
    lib.sdpa_bwd_bias_grad_workspace_size.restype = sz
    lib.sdpa_t5_bucket.argtypes = [vp, vp, i64, i32, i32, i32, vp]
    lib.sdpa_t5_bucket.restype = i32
    lib.sdpa_exp2_fma.argtypes = [vp, vp, i64, vp]
    lib.sdpa_exp2_fma.restype = i32
    lib.sdpa_read_device_status.argtypes = [vp]
    lib.sdpa_read_device_status.restype = i32
    lib.sdpa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.sdpa_set_wait_limit_ns.restype = None
    lib.sdpa_debug_wait_timeout.argtypes = [vp]
    lib.sdpa_debug_wait_timeout.restype = i32
    fp = ctypes.POINTER(Fire)
    lib.sdpa_fire_table.argtypes = [fp, i64, i64, vp, vp]
    lib.sdpa_fire_table.restype = i32
    lib.sdpa_fire_backward_workspace_size.argtypes = [fp, i64, i64]
    lib.sdpa_fire_backward_workspace_size.restype = sz
    lib.sdpa_fire_backward.argtypes = [fp, i64, i64, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.sdpa_fire_backward.restype = i32
    lib.sdpa_status_string.argtypes = [i32]
    lib.sdpa_status_string.restype = ctypes.c_char_p
    if path is None:
        _lib = lib
    return lib


def _check(status: int, where: str):
    if status != SDPA_OK:
        raise SdpaError(status, where)


def _stream(t: torch.Tensor | None = None):
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def make_shape(q: torch.Tensor, k: torch.Tensor) -> Shape:
    """Shape of q [B, L, Hq, d] against k [B, Lk, Hkv, d] (Lk may differ from L)."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, L, H, d]")
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape[0] != B or k.shape[3] != d:
        raise ValueError(f"k shape {tuple(k.shape)} does not match q {tuple(q.shape)}")
    if q.stride(-1) != 1 or k.stride(-1) != 1:
        raise ValueError("head_dim must be contiguous")
    return Shape(B, L, Hq, Hkv, d, q.stride(0), q.stride(1), q.stride(2),
                 k.stride(0), k.stride(1), k.stride(2), k.shape[1])


def make_varlen_shape(q: torch.Tensor, k: torch.Tensor, batch: int) -> Shape:
    """Shape of packed q [total_q, Hq, d] and k [total_k, Hkv, d] with `batch` sequences."""
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("packed q and k must be [total, H, d]")
    if q.shape[2] != k.shape[2]:
        raise ValueError("q and k head dims differ")
    if q.stride(-1) != 1 or k.stride(-1) != 1:
        raise ValueError("head_dim must be contiguous")
    return Shape(int(batch), 0, q.shape[1], k.shape[1], q.shape[2], 0, q.stride(0), q.stride(1),
                 0, k.stride(0), k.stride(1), 0)


def make_varlen(cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor, max_seqlen_q: int,
                max_seqlen_k: int, total_q: int, total_k: int) -> Varlen:
    for t, n in ((cu_seqlens_q, "cu_seqlens_q"), (cu_seqlens_k, "cu_seqlens_k")):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.dim() != 1:
            raise ValueError(f"{n} must be a contiguous int32 CUDA vector")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel():
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 entries")
    return Varlen(cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), int(max_seqlen_q),
                  int(max_seqlen_k), int(total_q), int(total_k))


def make_mask(causal: bool, window_left: int, window_right: int) -> MaskSpec:
    return MaskSpec(1 if causal else 0, int(window_left), int(window_right))


def make_bias(bias: torch.Tensor | None, t5_table: torch.Tensor | None, num_buckets: int,
              max_distance: int, bidirectional: bool, dims: tuple | None = None,
              alibi_slopes: torch.Tensor | None = None,
              rel_table: torch.Tensor | None = None) -> BiasDesc:
    """Bias descriptor; ``dims`` = (B, Hq, L) of the attention checks the shapes."""
    if sum(x is not None for x in (bias, t5_table, alibi_slopes, rel_table)) > 1:
        raise ValueError("give one of a dense bias, a T5 table, ALiBi slopes or a relative table")
    if rel_table is not None:
        if (rel_table.dtype != torch.float32 or rel_table.dim() != 2
                or not rel_table.is_contiguous()):
            raise ValueError("relative table must be contiguous float32 [Lq + Lk - 1, Hq]")
        if dims is not None:
            if rel_table.shape[1] != dims[1]:
                raise ValueError("relative table columns must equal the query heads")
            if len(dims) > 2 and dims[2] > 0:
                Lk = dims[3] if len(dims) > 3 else dims[2]
                if rel_table.shape[0] != dims[2] + Lk - 1:
                    raise ValueError("relative table must have Lq + Lk - 1 rows")
        return BiasDesc(BIAS_REL, rel_table.data_ptr(), 0, 0, 0, 0, 0, 0)
    if alibi_slopes is not None:
        if (alibi_slopes.dtype != torch.float32 or alibi_slopes.dim() != 1
                or not alibi_slopes.is_contiguous()):
            raise ValueError("ALiBi slopes must be a contiguous float32 [Hq] vector")
        if dims is not None and alibi_slopes.shape[0] != dims[1]:
            raise ValueError("ALiBi slopes must have one entry per query head")
        return BiasDesc(BIAS_ALIBI, alibi_slopes.data_ptr(), 0, 0, 0, 0, 0, 0)
    if bias is not None:
        if bias.dtype != torch.float32 or bias.dim() != 4 or bias.stride(-1) != 1:
            raise ValueError("dense bias must be float32 [B|1, H|1, L, L] with j contiguous")
        if dims is not None:
            B, Hq, L = dims[:3]
            Lk = dims[3] if len(dims) > 3 else L
            if (bias.shape[0] not in (1, B) or bias.shape[1] not in (1, Hq)
                    or tuple(bias.shape[2:]) != (L, Lk)):
                raise ValueError(f"dense bias shape {tuple(bias.shape)} is not "
                                 f"[{B}|1, {Hq}|1, {L}, {Lk}]")
        sb = bias.stride(0) if bias.shape[0] > 1 else 0
        sh = bias.stride(1) if bias.shape[1] > 1 else 0
        return BiasDesc(BIAS_DENSE, bias.data_ptr(), sb, sh, bias.stride(2), 0, 0, 0)
    if t5_table is not None:
        if t5_table.dtype != torch.float32 or not t5_table.is_contiguous():
            raise ValueError("T5 table must be contiguous float32 [num_buckets, Hq]")
        if t5_table.dim() != 2 or t5_table.shape[0] != num_buckets:
            raise ValueError("T5 table must be [num_buckets, Hq]")
        if dims is not None and t5_table.shape[1] != dims[1]:
            raise ValueError("T5 table columns must equal the query heads")
        return BiasDesc(BIAS_T5, t5_table.data_ptr(), 0, 0, 0, int(num_buckets),
                        int(max_distance), 1 if bidirectional else 0)
    return BiasDesc(BIAS_NONE, None, 0, 0, 0, 0, 0, 0)


def _same_layout(a: torch.Tensor, ref: torch.Tensor, name: str):
    if a.shape != ref.shape or a.stride() != ref.stride() or a.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bf16 with the shape and strides of its partner")


def sdpa_fwd(q, k, v, *, causal=False, window_left=-1, window_right=-1, bias=None,
             t5_table=None, t5_num_buckets=32, t5_max_distance=128, t5_bidirectional=True,
             alibi_slopes=None, rel_table=None, scale=None, out=None, lse=None):
    """O, LSE = attention forward (see sdpa_fwd in include/sdpa.h)."""
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise ValueError(f"{n} must be a bf16 CUDA tensor")
    shape = make_shape(q, k)
    _same_layout(v, k, "v")
    B, L, Hq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _same_layout(out, q, "out")
    if lse is None:
        lse = torch.empty(B, Hq, L, device=q.device, dtype=torch.float32)
    if lse.shape != (B, Hq, L) or not lse.is_contiguous() or lse.dtype != torch.float32:
        raise ValueError("lse must be contiguous float32 [B, Hq, L]")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    bd = make_bias(bias, t5_table, t5_num_buckets, t5_max_distance, t5_bidirectional,
                   (B, Hq, L, k.shape[1]), alibi_slopes, rel_table)
    m = make_mask(causal, window_left, window_right)
    st = lib.sdpa_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(bd),
                      ctypes.byref(m), sc, _ptr(out), _ptr(lse), _stream(q))
    _check(st, "sdpa_fwd")
    return out, lse


def sdpa_bwd_workspace_size(q, k, deterministic: bool = True) -> int:
    lib = load_library()
    shape = make_shape(q, k)
    return int(lib.sdpa_bwd_workspace_size(ctypes.byref(shape), 1 if deterministic else 0))


def sdpa_bwd(q, k, v, o, do, lse, *, causal=False, window_left=-1, window_right=-1,
             bias=None, t5_table=None, t5_num_buckets=32, t5_max_distance=128,
             t5_bidirectional=True, alibi_slopes=None, rel_table=None,
             scale=None, dq=None, dk=None, dv=None,
             workspace=None, deterministic=True, phases=BWD_ALL):
    """dQ, dK, dV = attention backward (see sdpa_bwd / sdpa_bwd_phases in include/sdpa.h).

    ``phases`` selects launches (BWD_PREPROCESS | BWD_DQ | BWD_DKDV); the
    default runs all three in order.  DQ and DKDV read D from the workspace
    of an earlier PREPROCESS call on the same O and dO.
    """
    lib = load_library()
    shape = make_shape(q, k)
    _same_layout(v, k, "v")
    _same_layout(o, q, "o")
    _same_layout(do, q, "do")
    d = q.shape[-1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _same_layout(dq, q, "dq")
    _same_layout(dk, k, "dk")
    _same_layout(dv, k, "dv")
    need = int(lib.sdpa_bwd_workspace_size(ctypes.byref(shape), 1))
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    bd = make_bias(bias, t5_table, t5_num_buckets, t5_max_distance, t5_bidirectional,
                   (q.shape[0], q.shape[2], q.shape[1], k.shape[1]), alibi_slopes, rel_table)
    m = make_mask(causal, window_left, window_right)
    args = (ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
            ctypes.byref(bd), ctypes.byref(m), sc, _ptr(dq), _ptr(dk), _ptr(dv),
            1 if deterministic else 0, _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(q))
    if phases == BWD_ALL:
        _check(lib.sdpa_bwd(*args), "sdpa_bwd")
    else:
        _check(lib.sdpa_bwd_phases(int(phases), *args), "sdpa_bwd_phases")
    return dq, dk, dv


def sdpa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, *, causal=False, window_left=-1,
                     window_right=-1, bias=None, t5_table=None, t5_num_buckets=32,
                     t5_max_distance=128, t5_bidirectional=True, alibi_slopes=None, rel_table=None,
                     scale=None):
    """Backward into caller-given dQ, dK, dV with no workspace and no allocation.

    For callers that cannot allocate device memory: the library's built-in
    scratch array (NOALLOC_SCRATCH_BYTES) stands in for the workspace, so the
    shape's sdpa_bwd_workspace_size must fit in it.  Calls that overlap on
    the GPU race on that array.
    """
    lib = load_library()
    shape = make_shape(q, k)
    for t, ref, n in ((v, k, "v"), (o, q, "o"), (do, q, "do"), (dq, q, "dq"), (dk, k, "dk"),
                      (dv, k, "dv")):
        _same_layout(t, ref, n)
    sc = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    bd = make_bias(bias, t5_table, t5_num_buckets, t5_max_distance, t5_bidirectional,
                   (q.shape[0], q.shape[2], q.shape[1], k.shape[1]), alibi_slopes, rel_table)
    m = make_mask(causal, window_left, window_right)
    st = lib.sdpa_bwd_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do),
                              _ptr(lse), ctypes.byref(bd), ctypes.byref(m), sc, _ptr(dq),
                              _ptr(dk), _ptr(dv), 1, _stream(q))
    _check(st, "sdpa_bwd_noalloc")
    return dq, dk, dv


def sdpa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, *,
                    causal=False, window_left=-1, window_right=-1, t5_table=None,
                    t5_num_buckets=32, t5_max_distance=128, t5_bidirectional=True,
                    alibi_slopes=None, rel_table=None, scale=None, out=None, lse=None):
    """O [total_q, Hq, d], LSE [Hq, total_q] of a packed batch (sdpa_fwd_varlen)."""
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise ValueError(f"{n} must be a bf16 CUDA tensor")
    _same_layout(v, k, "v")
    B = cu_seqlens_q.numel() - 1
    shape = make_varlen_shape(q, k, B)
    vl = make_varlen(cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, q.shape[0],
                     k.shape[0])
    total_q, Hq, d = q.shape
    out = torch.empty_like(q) if out is None else out
    _same_layout(out, q, "out")
    if lse is None:
        lse = torch.empty(Hq, total_q, device=q.device, dtype=torch.float32)
    if lse.shape != (Hq, total_q) or not lse.is_contiguous() or lse.dtype != torch.float32:
        raise ValueError("lse must be contiguous float32 [Hq, total_q]")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    bd = make_bias(None, t5_table, t5_num_buckets, t5_max_distance, t5_bidirectional,
                   (B, q.shape[1], 0, 0), alibi_slopes, rel_table)
    m = make_mask(causal, window_left, window_right)
    st = lib.sdpa_fwd_varlen(ctypes.byref(shape), ctypes.byref(vl), _ptr(q), _ptr(k), _ptr(v),
                             ctypes.byref(bd), ctypes.byref(m), sc, _ptr(out), _ptr(lse),
                             _stream(q))
    _check(st, "sdpa_fwd_varlen")
    return out, lse


def sdpa_bwd_varlen(q, k, v, o, do, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                    max_seqlen_k, *, causal=False, window_left=-1, window_right=-1,
                    t5_table=None, t5_num_buckets=32, t5_max_distance=128,
                    t5_bidirectional=True, alibi_slopes=None, rel_table=None,
                    scale=None, dq=None, dk=None,
                    dv=None, workspace=None):
    """dQ, dK, dV of a packed batch (sdpa_bwd_varlen)."""
    lib = load_library()
    _same_layout(v, k, "v")
    _same_layout(o, q, "o")
    _same_layout(do, q, "do")
    B = cu_seqlens_q.numel() - 1
    shape = make_varlen_shape(q, k, B)
    vl = make_varlen(cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, q.shape[0],
                     k.shape[0])
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _same_layout(dq, q, "dq")
    _same_layout(dk, k, "dk")
    _same_layout(dv, k, "dv")
    need = int(lib.sdpa_bwd_varlen_workspace_size(ctypes.byref(shape), ctypes.byref(vl)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    sc = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    bd = make_bias(None, t5_table, t5_num_buckets, t5_max_distance, t5_bidirectional,
                   (B, q.shape[1], 0, 0), alibi_slopes, rel_table)
    m = make_mask(causal, window_left, window_right)
    st = lib.sdpa_bwd_varlen(ctypes.byref(shape), ctypes.byref(vl), _ptr(q), _ptr(k), _ptr(v),
                             _ptr(o), _ptr(do), _ptr(lse), ctypes.byref(bd), ctypes.byref(m), sc,
                             _ptr(dq), _ptr(dk), _ptr(dv), 1, _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(q))
    _check(st, "sdpa_bwd_varlen")
    return dq, dk, dv


def sdpa_bwd_bias_grad_workspace_size(q, k, *, bias=None, t5_table=None, t5_num_buckets=32,
                                      t5_max_distance=128, t5_bidirectional=True,
                                      alibi_slopes=None, rel_table=None) -> int:
    lib = load_library()
    shape = make_shape(q, k)
    bd = make_bias(bias, t5_table, t5_num_buckets, t5_max_distance, t5_bidirectional,
                   (q.shape[0], q.shape[2], q.shape[1], k.shape[1]), alibi_slopes, rel_table)
    return int(lib.sdpa_bwd_bias_grad_workspace_size(ctypes.byref(shape), ctypes.byref(bd)))


def sdpa_bwd_bias_grad(q, k, v, o, do, lse, *, causal=False, window_left=-1, window_right=-1,
                       bias=None, t5_table=None, t5_num_buckets=32, t5_max_distance=128,
                       t5_bidirectional=True, alibi_slopes=None, rel_table=None,
                       scale=None, dq=None, dk=None,
                       dv=None, dbias=None, workspace=None):
    """dQ, dK, dV and the bias gradient (see sdpa_bwd_bias_grad in include/sdpa.h).

    The bias gradient has the dense bias's shape and strides, the T5 table's
    [num_buckets, Hq] shape, or the ALiBi slopes' [Hq] shape.
    """
    lib = load_library()
    shape = make_shape(q, k)
    _same_layout(v, k, "v")
    _same_layout(o, q, "o")
    _same_layout(do, q, "do")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _same_layout(dq, q, "dq")
    _same_layout(dk, k, "dk")
    _same_layout(dv, k, "dv")
    bd = make_bias(bias, t5_table, t5_num_buckets, t5_max_distance, t5_bidirectional,
                   (q.shape[0], q.shape[2], q.shape[1], k.shape[1]), alibi_slopes, rel_table)
    ref = next((x for x in (bias, t5_table, alibi_slopes, rel_table) if x is not None), None)
    if ref is None:
        raise ValueError("a bias gradient needs a dense bias, a T5 table or ALiBi slopes")
    if dbias is None:
        dbias = torch.empty_strided(ref.shape, ref.stride(), device=q.device,
                                    dtype=torch.float32)
    if (dbias.shape != ref.shape or dbias.stride() != ref.stride()
            or dbias.dtype != torch.float32):
        raise ValueError("dbias must be float32 with the shape and strides of the bias")
    need = int(lib.sdpa_bwd_bias_grad_workspace_size(ctypes.byref(shape), ctypes.byref(bd)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    sc = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    m = make_mask(causal, window_left, window_right)
    st = lib.sdpa_bwd_bias_grad(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                _ptr(do), _ptr(lse), ctypes.byref(bd), ctypes.byref(m), sc,
                                _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbias), 1, _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(q))
    _check(st, "sdpa_bwd_bias_grad")
    return dq, dk, dv, dbias


def sdpa_t5_bucket(rel: torch.Tensor, num_buckets=32, max_distance=128, bidirectional=True):
    """Bucket ids of int32 signed distances (device tensor) by the kernels' own function."""
    lib = load_library()
    if rel.dtype != torch.int32 or not rel.is_cuda or not rel.is_contiguous():
        raise ValueError("rel must be a contiguous int32 CUDA tensor")
    out = torch.empty_like(rel)
    st = lib.sdpa_t5_bucket(_ptr(rel), _ptr(out), rel.numel(), int(num_buckets),
                            int(max_distance), 1 if bidirectional else 0, _stream(rel))
    _check(st, "sdpa_t5_bucket")
    return out


def sdpa_exp2_fma(x: torch.Tensor) -> torch.Tensor:
    """2^x by the kernels' FMA-pipe exponential (float32 CUDA tensor)."""
    lib = load_library()
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    _check(lib.sdpa_exp2_fma(_ptr(x), _ptr(y), x.numel(), _stream(x)), "sdpa_exp2_fma")
    return y


def sdpa_read_device_status() -> int:
    """Synchronise the current stream; return (and clear) the device status code."""
    return int(load_library().sdpa_read_device_status(_stream()))


def sdpa_set_wait_limit_ns(ns: int):
    load_library().sdpa_set_wait_limit_ns(int(ns))


def sdpa_debug_wait_timeout():
    _check(load_library().sdpa_debug_wait_timeout(_stream()), "sdpa_debug_wait_timeout")


def _fire_desc(w1, b1, w2, b2, c, threshold):
    for t, n in ((w1, "w1"), (b1, "b1"), (w2, "w2"), (b2, "b2")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"FIRE {n} must be a contiguous float32 CUDA tensor")
    W = w1.shape[0]
    if w1.dim() != 1 or b1.shape != (W,) or w2.dim() != 2 or w2.shape[1] != W or \
            b2.shape != (w2.shape[0],):
        raise ValueError("FIRE weights must be w1 [W], b1 [W], w2 [H, W], b2 [H]")
    return Fire(w1.data_ptr(), b1.data_ptr(), w2.data_ptr(), b2.data_ptr(), float(c),
                float(threshold), int(W), int(w2.shape[0]))


def sdpa_fire_table(w1, b1, w2, b2, c, threshold, Lq, Lk, out=None):
    """FIRE bias as a relative-position table [Lq + Lk - 1, H] (see sdpa_fire_table in
    include/sdpa.h); pass it as ``rel_table``."""
    f = _fire_desc(w1, b1, w2, b2, c, threshold)
    if out is None:
        out = torch.empty(Lq + Lk - 1, f.heads, device=w1.device, dtype=torch.float32)
    _check(load_library().sdpa_fire_table(ctypes.byref(f), int(Lq), int(Lk), _ptr(out),
                                          _stream(w1)), "sdpa_fire_table")
    return out


def sdpa_fire_backward(w1, b1, w2, b2, c, threshold, Lq, Lk, d_table):
    """Gradients of FIRE's parameters from its table's gradient: a dict with w1, b1, w2,
    b2 and c_threshold (d/dc, d/dthreshold)."""
    lib = load_library()
    f = _fire_desc(w1, b1, w2, b2, c, threshold)
    if d_table.dtype != torch.float32 or not d_table.is_contiguous() or \
            tuple(d_table.shape) != (Lq + Lk - 1, f.heads):
        raise ValueError("d_table must be contiguous float32 [Lq + Lk - 1, H]")
    need = int(lib.sdpa_fire_backward_workspace_size(ctypes.byref(f), int(Lq), int(Lk)))
    ws = torch.empty(max(need, 256), device=w1.device, dtype=torch.uint8)
    g = {n: torch.empty_like(t) for n, t in (("w1", w1), ("b1", b1), ("w2", w2), ("b2", b2))}
    g["c_threshold"] = torch.empty(2, device=w1.device, dtype=torch.float32)
    _check(lib.sdpa_fire_backward(ctypes.byref(f), int(Lq), int(Lk), _ptr(d_table), _ptr(g["w1"]),
                                  _ptr(g["b1"]), _ptr(g["w2"]), _ptr(g["b2"]),
                                  _ptr(g["c_threshold"]), _ptr(ws), ws.numel(), _stream(w1)),
           "sdpa_fire_backward")
    return g


def sdpa_status_string(status: int) -> str:
    return load_library().sdpa_status_string(int(status)).decode()
