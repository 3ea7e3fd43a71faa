"""qk_rmsnorm_rope_qknr_b200 -- fused Q/K RMSNorm + RoPE (+ V copy, FP8 out) for B200.

A thin ctypes binding over libqknr.so (C ABI in include/qknr.h). Every step of
the transform runs in the library's CUDA kernels; this module only turns torch
tensors into pointers, sizes and a stream. There is no CPU or eager fallback:
if libqknr.so is missing or cannot load, every call raises.

Low-level names mirror the C entry points:
  qknr_rope_table(...)     table-driven per-head form
  qknr_rope_3d(...)        packed-QKV across-heads 3D form
  qknr_ucpe_cam_prep(...)  UCPE camera prep (ReLU, K scale, ray projection, RoPE)
  Rope3DCall(**params)     qknr_rope_3d prepared once, for repeated small calls
  RopeTableCall(...)       qknr_rope_table prepared once, likewise
Page-shaped wrappers allocate missing outputs and return them:
  fused_qk_norm_rope(q, k, q_weight, k_weight, rope_table, eps, *, head_dim=None,
                     rotary_dim=None, interleaved=False) -> (q, k)
      ("vllm_omni.diffusion.layers.fused_qk_norm_rope", fused_qk_norm_rope)
  fused_qk_rmsnorm_rope(qkv, q_weight, k_weight, *, ppf, pph, ppw, ...,
                        q_out=None, k_out=None, v_out=None) -> (q, k, v)
      ("flashinfer.norm.fused_qk_rmsnorm_rope", Parameters / Returns)
  cam_prep_func(q_normed, k_normed, v_raw, *, proj_q, proj_kv, rope_cos, rope_sin,
                k_scale) -> (q_trans, k_trans, v_trans, inflation_sq)
      ("vllm_omni.diffusion.models.sana_wm.ucpe", cam_prep_func)
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqknr.so")

QKNR_OK, QKNR_ERR_NULL, QKNR_ERR_SHAPE, QKNR_ERR_UNSUPPORTED = 0, 1, 2, 3
QKNR_ERR_ALIGN, QKNR_ERR_ALIAS, QKNR_ERR_POINTER, QKNR_ERR_CUDA = 4, 5, 6, 7
QKNR_DT_BF16, QKNR_DT_F32, QKNR_DT_E4M3, QKNR_DT_F16 = 0, 1, 2, 3
ABI_VERSION = 4  # QKNR_ABI_VERSION the argument lists below are written for

EXPORTS = ("qknr_rope_table", "qknr_rope_3d", "qknr_rope_3d_partial_ssq", "qknr_rope_3d_with_ssq",
           "qknr_ucpe_cam_prep", "qknr_device_status", "qknr_test_set_wait_fault", "qknr_status_string",
           "qknr_last_error_detail", "qknr_abi_version")


class QknrError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"qknr status {status}: {detail}")
        self.status = status


class QknrValueError(QknrError, ValueError):
    """Shape, parameter, alignment or aliasing errors (the pages raise ValueError)."""


class Rope3DParams(C.Structure):
    _fields_ = [("struct_size", C.c_size_t), ("qkv", C.c_void_p), ("q_weight", C.c_void_p),
                ("k_weight", C.c_void_p), ("q_out", C.c_void_p), ("k_out", C.c_void_p),
                ("v_out", C.c_void_p), ("num_tokens", C.c_int64), ("pos_offset", C.c_int64),
                ("ppf", C.c_int32), ("pph", C.c_int32), ("ppw", C.c_int32),
                ("num_frame_channels", C.c_int32), ("num_height_channels", C.c_int32),
                ("num_width_channels", C.c_int32), ("num_heads_q", C.c_int32),
                ("num_heads_k", C.c_int32), ("num_heads_v", C.c_int32), ("head_dim", C.c_int32),
                ("eps", C.c_float), ("base", C.c_double), ("interleave", C.c_int32),
                ("factor", C.c_float), ("low", C.c_float), ("high", C.c_float),
                ("attention_factor", C.c_float), ("is_qk_norm", C.c_int32),
                ("output_fp8", C.c_int32), ("output_quant_scale", C.c_float),
                ("v_quant_scale", C.c_float), ("sequence_shard", C.c_int32),
                ("neox_per_axis", C.c_int32)]


_lib = None


def lib() -> C.CDLL:
    """The loaded libqknr.so; raises if it is missing (build it with build())."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libqknr.so not built at {LIB_PATH}; run "
                              "qk_rmsnorm_rope_qknr_b200.build.build()")
        L = C.CDLL(LIB_PATH)
        vp, i32, i64 = C.c_void_p, C.c_int32, C.c_int64
        L.qknr_rope_table.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i64, i32, i32, i32,
                                      i32, i64, i64, i64, i64, C.c_float, i32, vp]
        L.qknr_rope_table.restype = C.c_int
        L.qknr_rope_3d.argtypes = [C.POINTER(Rope3DParams), vp]
        L.qknr_rope_3d.restype = C.c_int
        L.qknr_rope_3d_partial_ssq.argtypes = [C.POINTER(Rope3DParams), vp, vp]
        L.qknr_rope_3d_partial_ssq.restype = C.c_int
        L.qknr_rope_3d_with_ssq.argtypes = [C.POINTER(Rope3DParams), vp, i32, i32, vp]
        L.qknr_rope_3d_with_ssq.restype = C.c_int
        L.qknr_ucpe_cam_prep.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64,
                                         i64, i32, i32, C.c_float, vp]
        L.qknr_ucpe_cam_prep.restype = C.c_int
        L.qknr_status_string.argtypes = [C.c_int]
        L.qknr_status_string.restype = C.c_char_p
        L.qknr_last_error_detail.restype = C.c_char_p
        L.qknr_abi_version.restype = C.c_int
        if L.qknr_abi_version() != ABI_VERSION:
            raise ImportError(f"libqknr.so has ABI version {L.qknr_abi_version()}, this binding "
                              f"expects {ABI_VERSION}; rebuild it")
        L.qknr_device_status.argtypes = [vp, C.POINTER(C.c_uint32), i32]
        L.qknr_device_status.restype = C.c_int
        L.qknr_test_set_wait_fault.argtypes = [C.c_uint32, C.c_uint64]
        L.qknr_test_set_wait_fault.restype = C.c_int
        _lib = L
    return _lib


def build(force: bool = False) -> str:
    """Compile libqknr.so in-tree (nvcc, sm_100a) if it is missing or stale."""
    import importlib

    return importlib.import_module(__name__ + ".build").build(force=force)


def _check(status: int) -> None:
    if status == QKNR_OK:
        return
    L = lib()
    detail = (L.qknr_last_error_detail() or b"").decode() or L.qknr_status_string(status).decode()
    if status in (QKNR_ERR_NULL, QKNR_ERR_SHAPE, QKNR_ERR_UNSUPPORTED, QKNR_ERR_ALIGN,
                  QKNR_ERR_ALIAS, QKNR_ERR_POINTER):
        raise QknrValueError(status, detail)
    raise QknrError(status, detail)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream, *tensors) -> Optional[int]:
    if stream is not None:
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    for t in tensors:
        if t is not None and t.is_cuda:
            return torch.cuda.current_stream(t.device).cuda_stream
    return None


_ACT_DTYPES = {torch.bfloat16: QKNR_DT_BF16, torch.float16: QKNR_DT_F16}


def _act_dtype(q: torch.Tensor) -> int:
    if q.dtype not in _ACT_DTYPES:
        raise QknrValueError(QKNR_ERR_SHAPE, f"q dtype {q.dtype} is not bfloat16/float16")
    return _ACT_DTYPES[q.dtype]


def _table_dtype(t: torch.Tensor, act: torch.dtype) -> int:
    if t.dtype == torch.float32:
        return QKNR_DT_F32
    if t.dtype == act:
        return _ACT_DTYPES[act]
    raise QknrValueError(QKNR_ERR_SHAPE,
                         f"rope_table dtype {t.dtype} is neither float32 nor {act}")


def _token_stride(t: torch.Tensor, name: str, heads: int, head_dim: int,
                  dtype: torch.dtype = torch.bfloat16) -> int:
    sh = t.shape  # (one shape and one stride tuple: this runs on every call)
    if len(sh) != 3 or sh[1] != heads or sh[2] != head_dim:
        raise QknrValueError(QKNR_ERR_SHAPE, f"{name} must be [tokens, {heads}, {head_dim}]")
    if t.dtype != dtype:
        raise QknrValueError(QKNR_ERR_SHAPE, f"{name} must be {dtype}")
    st = t.stride()
    if sh[0] > 0 and heads > 0 and (st[2] != 1 or (heads > 1 and st[1] != head_dim)):
        raise QknrValueError(QKNR_ERR_SHAPE, f"{name}: heads must be dense inside a token")
    return st[0]


# --------------------------------------------------------------- C-ABI names --
def qknr_rope_table(q, k, q_out, k_out, q_weight, k_weight, rope_table, *, eps: float,
                    rotary_dim: int = 0, interleaved: bool = False, stream=None) -> None:
    """Table form through the C ABI (destination passing; see include/qknr.h).
    q/k/q_out/k_out are [tokens, heads, head_dim] with dense heads, all bf16 or
    all float16 (the activation dtype, taken from q); the weights have the
    activation dtype, the table float32 or the activation dtype."""
    if q.dim() != 3:
        raise QknrValueError(QKNR_ERR_SHAPE, "q must be [tokens, heads, head_dim]")
    act = _act_dtype(q)
    T, Hq, D = q.shape
    Hk = k.shape[1] if k.dim() == 3 else -1
    qs = _token_stride(q, "q", Hq, D, q.dtype)
    ks = _token_stride(k, "k", Hk, D, q.dtype)
    qos = _token_stride(q_out, "q_out", Hq, D, q.dtype)
    kos = _token_stride(k_out, "k_out", Hk, D, q.dtype)
    if k.shape[0] != T or q_out.shape[0] != T or k_out.shape[0] != T:
        raise QknrValueError(QKNR_ERR_SHAPE, "q, k and outputs differ in token count")
    R = rotary_dim or D
    if rope_table.dim() != 2 or tuple(rope_table.shape) != (T, R) or not rope_table.is_contiguous():
        raise QknrValueError(QKNR_ERR_SHAPE, f"rope_table must be a dense [{T}, {R}] tensor")
    for n, w in (("q_weight", q_weight), ("k_weight", k_weight)):
        if w.dtype != q.dtype or w.numel() != D or not w.is_contiguous():
            raise QknrValueError(QKNR_ERR_SHAPE, f"{n} must be a dense {q.dtype} [{D}] tensor")
    st = _stream(stream, q, k, q_out, k_out)
    _check(lib().qknr_rope_table(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _ptr(q_weight),
                                 _ptr(k_weight), _ptr(rope_table),
                                 _table_dtype(rope_table, q.dtype), act, T, Hq,
                                 Hk, D, R, qs, ks, qos, kos, float(eps), int(bool(interleaved)),
                                 st))


class RopeTableCall:
    """The table form prepared once for repeated use: head counts, head_dim,
    rotary_dim, eps, the pair layout and the dtypes are fixed here. Each call
    checks the tensors' shapes, dtypes and head density, takes their token
    strides and launches (about two thirds of qknr_rope_table's Python cost). Pass
    the stream (a torch stream or its handle) to skip the current-stream
    lookup."""

    def __init__(self, *, heads_q: int, heads_k: int, head_dim: int, eps: float,
                 rotary_dim: int = 0, interleaved: bool = False,
                 act_dtype: torch.dtype = torch.bfloat16,
                 table_dtype: torch.dtype = torch.float32):
        if act_dtype not in _ACT_DTYPES:
            raise QknrValueError(QKNR_ERR_SHAPE, f"act_dtype {act_dtype} is not bfloat16/float16")
        self._tcode = _table_dtype(torch.empty(0, dtype=table_dtype), act_dtype)
        self._acode = _ACT_DTYPES[act_dtype]
        self._act, self._tdt = act_dtype, table_dtype
        self._hq, self._hk, self._d = int(heads_q), int(heads_k), int(head_dim)
        self._r = int(rotary_dim) or self._d
        self._eps, self._il = float(eps), int(bool(interleaved))
        self._fn = lib().qknr_rope_table

    def _stride(self, t, heads, T):
        sh = t.shape
        if len(sh) != 3 or sh[0] != T or sh[1] != heads or sh[2] != self._d or \
                t.dtype is not self._act:
            raise QknrValueError(QKNR_ERR_SHAPE,
                                 f"expected {self._act} [{T}, {heads}, {self._d}] tensors")
        st = t.stride()
        if T > 0 and heads > 0 and (st[2] != 1 or (heads > 1 and st[1] != self._d)):
            raise QknrValueError(QKNR_ERR_SHAPE, "heads must be dense inside a token")
        return st[0]

    def __call__(self, q, k, q_out, k_out, q_weight, k_weight, rope_table, stream=None) -> None:
        T = q.shape[0] if q.dim() == 3 else -1
        qs = self._stride(q, self._hq, T)
        ks = self._stride(k, self._hk, T)
        qos = self._stride(q_out, self._hq, T)
        kos = self._stride(k_out, self._hk, T)
        if rope_table.dtype is not self._tdt or tuple(rope_table.shape) != (T, self._r) or \
                not rope_table.is_contiguous():
            raise QknrValueError(QKNR_ERR_SHAPE,
                                 f"rope_table must be a dense {self._tdt} [{T}, {self._r}]")
        for w in (q_weight, k_weight):
            if w.dtype is not self._act or w.numel() != self._d or not w.is_contiguous():
                raise QknrValueError(QKNR_ERR_SHAPE, f"weights must be dense {self._act} [{self._d}]")
        if stream is None:
            st = torch.cuda.current_stream(q.device).cuda_stream
        else:
            st = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        status = self._fn(q.data_ptr(), k.data_ptr(), q_out.data_ptr(), k_out.data_ptr(),
                          q_weight.data_ptr(), k_weight.data_ptr(), rope_table.data_ptr(),
                          self._tcode, self._acode, T, self._hq, self._hk, self._d, self._r, qs,
                          ks, qos, kos, self._eps, self._il, st)
        if status:
            _check(status)


def make_3d_params(qkv, q_weight, k_weight, q_out, k_out, v_out, *, ppf, pph, ppw,
                   num_frame_channels, num_height_channels, num_width_channels, num_heads_q,
                   num_heads_k, num_heads_v, head_dim, eps=1e-6, base=10000.0, interleave=True,
                   factor=1.0, low=0.0, high=0.0, attention_factor=1.0, is_qk_norm=True,
                   output_fp8=False, output_quant_scale=1.0, v_quant_scale=1.0,
                   pos_offset: Optional[int] = None, num_tokens=None,
                   neox_per_axis=False) -> Rope3DParams:
    """C parameter block. pos_offset=None is a whole call (num_tokens must be a
    multiple of ppf*pph*ppw); an integer marks a sequence shard whose first
    token sits at that patch position (any token count). neox_per_axis picks
    the NeoX pairs inside each axis group (see include/qknr.h)."""
    row = (num_heads_q + num_heads_k + num_heads_v) * head_dim
    if num_tokens is None:
        if qkv.dtype != torch.bfloat16 or qkv.shape[-1] != row or not qkv.is_contiguous():
            raise QknrValueError(QKNR_ERR_SHAPE,
                                 f"qkv must be a contiguous bf16 tensor [..., {row}]")
        num_tokens = qkv.numel() // row
    p = Rope3DParams()
    p.struct_size = C.sizeof(Rope3DParams)
    p.qkv, p.q_weight, p.k_weight = _ptr(qkv), _ptr(q_weight), _ptr(k_weight)
    p.q_out, p.k_out, p.v_out = _ptr(q_out), _ptr(k_out), _ptr(v_out)
    p.num_tokens = int(num_tokens)
    p.pos_offset = 0 if pos_offset is None else int(pos_offset)
    p.sequence_shard = 0 if pos_offset is None else 1
    p.ppf, p.pph, p.ppw = ppf, pph, ppw
    p.num_frame_channels, p.num_height_channels = num_frame_channels, num_height_channels
    p.num_width_channels = num_width_channels
    p.num_heads_q, p.num_heads_k, p.num_heads_v = num_heads_q, num_heads_k, num_heads_v
    p.head_dim = head_dim
    p.eps, p.base, p.interleave = eps, base, int(bool(interleave))
    p.factor, p.low, p.high, p.attention_factor = factor, low, high, attention_factor
    p.is_qk_norm, p.output_fp8 = int(bool(is_qk_norm)), int(bool(output_fp8))
    p.output_quant_scale, p.v_quant_scale = output_quant_scale, v_quant_scale
    p.neox_per_axis = int(bool(neox_per_axis))
    return p


def qknr_rope_3d(qkv, q_weight, k_weight, q_out, k_out, v_out, *, stream=None, **params) -> None:
    """3D form through the C ABI (destination passing; see include/qknr.h).
    params are the page's keyword arguments plus pos_offset (an integer marks
    a sequence shard; see make_3d_params)."""
    p = make_3d_params(qkv, q_weight, k_weight, q_out, k_out, v_out, **params)
    odt = torch.float8_e4m3fn if params.get("output_fp8") else torch.bfloat16
    for n, o, h in (("q_out", q_out, p.num_heads_q), ("k_out", k_out, p.num_heads_k),
                    ("v_out", v_out, p.num_heads_v)):
        if h and o is not None:
            if o.dtype not in (odt, torch.uint8) or not o.is_contiguous() or \
                    o.numel() != p.num_tokens * h * p.head_dim:
                raise QknrValueError(QKNR_ERR_SHAPE,
                                     f"{n} must be a dense {odt} tensor of {p.num_tokens}x{h}x"
                                     f"{p.head_dim} elements")
    for n, w, h in (("q_weight", q_weight, p.num_heads_q), ("k_weight", k_weight, p.num_heads_k)):
        if p.is_qk_norm and h and w is not None and (w.dtype != torch.bfloat16 or
                                                      w.numel() != h * p.head_dim):
            raise QknrValueError(QKNR_ERR_SHAPE, f"{n} must be bf16 [{h * p.head_dim}]")
    st = _stream(stream, qkv, q_out)
    _check(lib().qknr_rope_3d(C.byref(p), st))


class Rope3DCall:
    """A 3D-form call prepared once for repeated use: the page's keyword
    arguments (as for qknr_rope_3d) are fixed here and the C parameter block is
    built once. Each call checks only what changes between calls (the tensors'
    dtype, density and element counts, which the kernel trusts), fills in the
    six pointers and the token count, and launches: about a third of
    qknr_rope_3d's Python cost. Pass the stream (a torch stream or its handle)
    to skip the current-stream lookup. One instance is not for concurrent use
    from several threads (the parameter block is reused)."""

    def __init__(self, **params):
        self._p = make_3d_params(None, None, None, None, None, None, num_tokens=0, **params)
        p = self._p
        self._row = (p.num_heads_q + p.num_heads_k + p.num_heads_v) * p.head_dim
        self._sizes = (p.num_heads_q * p.head_dim, p.num_heads_k * p.head_dim,
                       p.num_heads_v * p.head_dim)
        self._odt = torch.float8_e4m3fn if p.output_fp8 else torch.bfloat16
        self._norm = bool(p.is_qk_norm)
        self._fn = lib().qknr_rope_3d
        self._byref = C.byref(p)

    def __call__(self, qkv, q_weight, k_weight, q_out, k_out, v_out, stream=None) -> None:
        p = self._p
        n = qkv.numel()
        if qkv.dtype is not torch.bfloat16 or n % self._row or not qkv.is_contiguous():
            raise QknrValueError(QKNR_ERR_SHAPE,
                                 f"qkv must be a contiguous bf16 tensor [..., {self._row}]")
        T = n // self._row
        odt = self._odt
        for o, sz in ((q_out, self._sizes[0]), (k_out, self._sizes[1]), (v_out, self._sizes[2])):
            if sz and (o is None or o.numel() != T * sz or
                       (o.dtype is not odt and o.dtype is not torch.uint8) or
                       not o.is_contiguous()):
                raise QknrValueError(QKNR_ERR_SHAPE,
                                     f"outputs must be dense {odt} tensors of {T} tokens")
        if self._norm:
            for w, sz in ((q_weight, self._sizes[0]), (k_weight, self._sizes[1])):
                if sz and (w is None or w.numel() != sz or w.dtype is not torch.bfloat16):
                    raise QknrValueError(QKNR_ERR_SHAPE, f"weights must be bf16 [{sz}]")
        p.qkv = qkv.data_ptr()
        p.q_weight, p.k_weight = _ptr(q_weight), _ptr(k_weight)
        p.q_out, p.k_out, p.v_out = _ptr(q_out), _ptr(k_out), _ptr(v_out)
        p.num_tokens = T
        if stream is None:
            st = torch.cuda.current_stream(qkv.device).cuda_stream
        else:
            st = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        status = self._fn(self._byref, st)
        if status:
            _check(status)


def qknr_rope_3d_partial_ssq(qkv, ssq_out, *, stream=None, **params) -> None:
    """Tensor-parallel pass 1 through the C ABI: per-token sums of x^2 over this
    call's Q and K heads into ssq_out (fp32 [tokens, 2])."""
    p = make_3d_params(qkv, None, None, None, None, None, **params)
    if ssq_out.dtype != torch.float32 or tuple(ssq_out.shape) != (p.num_tokens, 2) or \
            not ssq_out.is_contiguous():
        raise QknrValueError(QKNR_ERR_SHAPE, f"ssq_out must be a dense fp32 [{p.num_tokens}, 2]")
    _check(lib().qknr_rope_3d_partial_ssq(C.byref(p), _ptr(ssq_out), _stream(stream, qkv)))


def qknr_rope_3d_with_ssq(qkv, q_weight, k_weight, q_out, k_out, v_out, ssq, *, heads_q_total,
                          heads_k_total, stream=None, **params) -> None:
    """Tensor-parallel pass 3 through the C ABI: the 3D transform of this call's
    heads with the all-reduced sums ssq (fp32 [tokens, 2]) over heads_q_total /
    heads_k_total heads."""
    p = make_3d_params(qkv, q_weight, k_weight, q_out, k_out, v_out, **params)
    if ssq.dtype != torch.float32 or tuple(ssq.shape) != (p.num_tokens, 2) or \
            not ssq.is_contiguous():
        raise QknrValueError(QKNR_ERR_SHAPE, f"ssq must be a dense fp32 [{p.num_tokens}, 2]")
    _check(lib().qknr_rope_3d_with_ssq(C.byref(p), _ptr(ssq), int(heads_q_total),
                                       int(heads_k_total), _stream(stream, qkv, q_out)))


def qknr_ucpe_cam_prep(q_normed, k_normed, v_raw, proj_q, proj_kv, rope_cos, rope_sin, q_trans,
                       k_trans, v_trans, inflation_sq, *, k_scale: float, stream=None) -> None:
    """UCPE camera prep through the C ABI (destination passing; see
    include/qknr.h). q_normed/k_normed/v_raw dense [B, N, H, D] bf16 or float16;
    proj_q/proj_kv dense fp32 [B, N, 4, 4]; rope_cos/rope_sin dense fp32
    [N, D/2]; outputs dense [B, H, D, N] of the activation dtype; inflation_sq
    dense fp32 [B, H, N] or None."""
    if q_normed.dim() != 4:
        raise QknrValueError(QKNR_ERR_SHAPE, "q_normed must be [B, N, H, D]")
    act = _act_dtype(q_normed)
    B, N, H, D = q_normed.shape
    for n, t in (("k_normed", k_normed), ("v_raw", v_raw)):
        if tuple(t.shape) != (B, N, H, D) or t.dtype != q_normed.dtype:
            raise QknrValueError(QKNR_ERR_SHAPE, f"{n} must match q_normed's shape and dtype")
    for n, t, shape, dt in (("q_normed", q_normed, (B, N, H, D), q_normed.dtype),
                            ("k_normed", k_normed, (B, N, H, D), q_normed.dtype),
                            ("v_raw", v_raw, (B, N, H, D), q_normed.dtype),
                            ("proj_q", proj_q, (B, N, 4, 4), torch.float32),
                            ("proj_kv", proj_kv, (B, N, 4, 4), torch.float32),
                            ("rope_cos", rope_cos, (N, D // 2), torch.float32),
                            ("rope_sin", rope_sin, (N, D // 2), torch.float32),
                            ("q_trans", q_trans, (B, H, D, N), q_normed.dtype),
                            ("k_trans", k_trans, (B, H, D, N), q_normed.dtype),
                            ("v_trans", v_trans, (B, H, D, N), q_normed.dtype),
                            ("inflation_sq", inflation_sq, (B, H, N), torch.float32)):
        if t is None and n == "inflation_sq":
            continue
        if tuple(t.shape) != shape or t.dtype != dt or not t.is_contiguous():
            raise QknrValueError(QKNR_ERR_SHAPE, f"{n} must be a dense {dt} tensor {list(shape)}")
    st = _stream(stream, q_normed, q_trans)
    _check(lib().qknr_ucpe_cam_prep(_ptr(q_normed), _ptr(k_normed), _ptr(v_raw), _ptr(proj_q),
                                    _ptr(proj_kv), _ptr(rope_cos), _ptr(rope_sin),
                                    _ptr(q_trans), _ptr(k_trans), _ptr(v_trans),
                                    _ptr(inflation_sq), act, B, N, H, D, float(k_scale), st))


def qknr_device_status(clear: bool = False, stream=None, device=None) -> int:
    """Device status word (bit 0: a kernel gave up waiting on its own bulk
    copy and left its outputs incomplete). Synchronises the stream."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    out = C.c_uint32(0)
    _check(lib().qknr_device_status(_stream(stream), C.byref(out), int(bool(clear))))
    return out.value


# ------------------------------------------------------- page-shaped wrappers --
def fused_qk_norm_rope(q: torch.Tensor, k: torch.Tensor, q_weight: torch.Tensor,
                       k_weight: torch.Tensor, rope_table: torch.Tensor, eps: float, *,
                       head_dim: Optional[int] = None, rotary_dim: Optional[int] = None,
                       interleaved: bool = False, q_out: Optional[torch.Tensor] = None,
                       k_out: Optional[torch.Tensor] = None, stream=None
                       ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Q/K RMSNorm + packed RoPE, table form. q and k are bf16 or float16 (the
    weights too; the table float32 or the same 16-bit type). Returns new
    (q, k) unless outputs are given (pass q_out=q, k_out=k to work in place)."""
    D = head_dim or q.shape[-1]
    if q.shape[-1] != D or k.shape[-1] != D:
        raise QknrValueError(QKNR_ERR_SHAPE, f"last dim of q/k must be head_dim={D}")
    if q_out is None:
        q_out = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    if k_out is None:
        k_out = torch.empty(k.shape, dtype=k.dtype, device=k.device)
    qknr_rope_table(q, k, q_out, k_out, q_weight, k_weight, rope_table, eps=eps,
                    rotary_dim=rotary_dim or D, interleaved=interleaved, stream=stream)
    return q_out, k_out


def fused_qk_rmsnorm_rope(qkv: torch.Tensor, q_weight: torch.Tensor, k_weight: torch.Tensor, *,
                          ppf: int, pph: int, ppw: int, num_frame_channels: int,
                          num_height_channels: int, num_width_channels: int, num_heads_q: int,
                          num_heads_k: int, num_heads_v: int, head_dim: int, eps: float = 1e-6,
                          base: float = 10000.0, interleave: bool = True, factor: float = 1.0,
                          low: float = 0.0, high: float = 0.0, attention_factor: float = 1.0,
                          is_qk_norm: bool = True, output_fp8: bool = False,
                          output_quant_scale: float = 1.0, v_quant_scale: float = 1.0,
                          q_out: Optional[torch.Tensor] = None,
                          k_out: Optional[torch.Tensor] = None,
                          v_out: Optional[torch.Tensor] = None,
                          pos_offset: Optional[int] = None, neox_per_axis: bool = False,
                          stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Across-heads Q/K RMSNorm + 3D RoPE + V copy (+ FP8). Outputs are
    [B, S, H, D] for a 3D qkv and [T, H, D] for a 2D one. neox_per_axis (with
    interleave=False) takes the NeoX halves inside each axis group instead of
    across the whole head; the page does not say which is meant."""
    lead = tuple(qkv.shape[:-1])
    odt = torch.float8_e4m3fn if output_fp8 else torch.bfloat16
    outs = []
    for o, h in ((q_out, num_heads_q), (k_out, num_heads_k), (v_out, num_heads_v)):
        outs.append(o if o is not None else torch.empty(lead + (h, head_dim), dtype=odt,
                                                        device=qkv.device))
    qknr_rope_3d(qkv, q_weight, k_weight, *outs, stream=stream, ppf=ppf, pph=pph, ppw=ppw,
                 num_frame_channels=num_frame_channels, num_height_channels=num_height_channels,
                 num_width_channels=num_width_channels, num_heads_q=num_heads_q,
                 num_heads_k=num_heads_k, num_heads_v=num_heads_v, head_dim=head_dim, eps=eps,
                 base=base, interleave=interleave, factor=factor, low=low, high=high,
                 attention_factor=attention_factor, is_qk_norm=is_qk_norm,
                 output_fp8=output_fp8, output_quant_scale=output_quant_scale,
                 v_quant_scale=v_quant_scale, pos_offset=pos_offset,
                 neox_per_axis=neox_per_axis)
    return tuple(outs)


def cam_prep_func(q_normed: torch.Tensor, k_normed: torch.Tensor, v_raw: torch.Tensor, *,
                  proj_q: torch.Tensor, proj_kv: torch.Tensor, rope_cos: torch.Tensor,
                  rope_sin: torch.Tensor, k_scale: float, stream=None
                  ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """UCPE camera prep: ReLU, the K scale, the 4x4 ray projections and
    adjacent-pair RoPE of camera Q/K (projection only for V), from [B, N, H, D]
    inputs. Returns q_trans, k_trans, v_trans [B, H, D, N] (the inputs' dtype)
    and inflation_sq [B, H, N] float32, the squared-norm gain of each key under
    its projection."""
    B, N, H, D = q_normed.shape
    outs = [torch.empty((B, H, D, N), dtype=q_normed.dtype, device=q_normed.device)
            for _ in range(3)]
    infl = torch.empty((B, H, N), dtype=torch.float32, device=q_normed.device)
    qknr_ucpe_cam_prep(q_normed, k_normed, v_raw, proj_q, proj_kv, rope_cos, rope_sin, *outs,
                       infl, k_scale=k_scale, stream=stream)
    return outs[0], outs[1], outs[2], infl


__all__ = ["qknr_rope_table", "qknr_rope_3d", "qknr_rope_3d_partial_ssq", "qknr_rope_3d_with_ssq",
           "qknr_ucpe_cam_prep", "cam_prep_func",
           "qknr_device_status", "fused_qk_norm_rope", "fused_qk_rmsnorm_rope",
           "QknrError", "QknrValueError", "lib", "build", "make_3d_params", "Rope3DParams",
           "Rope3DCall", "RopeTableCall",
           "EXPORTS", "LIB_PATH"]
