"""fp64 CPU oracle for the fused Q/K RMSNorm + RoPE transform -- TEST INFRASTRUCTURE.

Only tests/, the smoke check in __graft_entry__ and the CPU-baseline leg of
bench.py may import this package. The product library never imports it and
shares no code with it (the C source is compiled on its own by oracle/build.py).

Everything here is numpy-in / numpy-out marshalling around the C functions in
qknr_oracle.c; the arithmetic, and the readings R1..R13 and U1..U6 of the pages, are
stated there. bf16 and binary16 values travel as uint16 bit patterns, E4M3 as
uint8.

Parity status: every function is pinned by tests/test_oracle_pins.py except
three readings the pages cannot decide -- the 3D NeoX pair layout (whole-head
pairs vs per-axis-group pairs, R8), the direction of the FP8 scale (R9) and
the definition of the camera prep's inflation_sq output (U6): "parity
unpinned" for those three choices.
"""
import ctypes as C

import numpy as np

from . import build as _build

_lib = None


def use_library(path=None):
    """Load the oracle from `path` (default: the built oracle/liboracle_qknr.so).
    The mutation tests point this at copies of the oracle with a planted mistake."""
    global _lib
    _lib = None
    return lib(path)


def lib(path=None):
    global _lib
    if _lib is None:
        path = path or _build.build()
        L = C.CDLL(path)
        i32, i64, f64, vp = C.c_int32, C.c_int64, C.c_double, C.c_void_p
        L.qknr_oracle_bf16_to_double.argtypes = [C.c_uint16]
        L.qknr_oracle_bf16_to_double.restype = f64
        L.qknr_oracle_bf16_from_double.argtypes = [f64]
        L.qknr_oracle_bf16_from_double.restype = C.c_uint16
        L.qknr_oracle_e4m3_to_double.argtypes = [C.c_uint8]
        L.qknr_oracle_e4m3_to_double.restype = f64
        L.qknr_oracle_e4m3_from_double.argtypes = [f64]
        L.qknr_oracle_e4m3_from_double.restype = C.c_uint8
        L.qknr_oracle_bf16_from_double_array.argtypes = [vp, vp, i64]
        L.qknr_oracle_f16_from_double_array.argtypes = [vp, vp, i64]
        L.qknr_oracle_f16_to_double.argtypes = [C.c_uint16]
        L.qknr_oracle_f16_to_double.restype = f64
        L.qknr_oracle_rope_table_exact_act.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32,
                                                       i32, i32, i32, f64, i32, vp, vp]
        L.qknr_oracle_rope_table_act.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32, i32,
                                                 i32, i32, f64, i32, vp, vp]
        L.qknr_oracle_e4m3_from_double_array.argtypes = [vp, vp, i64]
        L.qknr_oracle_rmsnorm.argtypes = [vp, i64, vp, f64, vp]
        L.qknr_oracle_rotate.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
        L.qknr_oracle_pairs_table.argtypes = [i32, i32, vp, vp]
        L.qknr_oracle_pairs_3d.argtypes = [i32, i32, i32, i32, i32, vp, vp]
        L.qknr_oracle_position_3d.argtypes = [i64, i64, i32, i32, i32, vp, vp, vp]
        L.qknr_oracle_angles_3d.argtypes = [i64, i64, i64, i32, i32, i32, f64, vp]
        L.qknr_oracle_rope_table_exact.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                                   i32, f64, i32, vp, vp]
        L.qknr_oracle_rope_table.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                             f64, i32, vp, vp]
        L.qknr_oracle_rope_3d_exact.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, i32, i32,
                                                i32, i32, i32, i32, i32, f64, f64, i32, i32, i32,
                                                vp, vp, vp]
        L.qknr_oracle_rope_3d.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, i32, i32, i32,
                                          i32, i32, i32, i32, f64, f64, i32, i32, i32, i32, f64,
                                          f64, vp, vp, vp]
        L.qknr_oracle_relu.argtypes = [vp, i64, vp]
        L.qknr_oracle_ray_project.argtypes = [vp, vp, i64, vp]
        L.qknr_oracle_ucpe_exact.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i64, i32,
                                             i32, f64, vp, vp, vp, vp]
        L.qknr_oracle_ucpe.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i64, i32, i32, f64,
                                       vp, vp, vp, vp]
        L.qknr_oracle_threads.restype = C.c_int
        L.qknr_oracle_set_threads.argtypes = [C.c_int]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


# ---------------------------------------------------------------- formats --
def bf16_to_f64(bits):
    """bfloat16 bit patterns (uint16 array) -> exact float64 values."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_from_f64(x):
    """One RNE rounding of float64 values to bfloat16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().qknr_oracle_bf16_from_double_array(_p(x), _p(out), x.size)
    return out


def f16_from_f64(x):
    """One RNE rounding of float64 values to IEEE binary16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().qknr_oracle_f16_from_double_array(_p(x), _p(out), x.size)
    return out


def f16_to_f64(bits):
    """binary16 bit patterns -> exact float64 values."""
    return np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def e4m3_from_f64(x):
    """One RNE rounding of float64 values to E4M3FN bit patterns, saturating."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint8)
    lib().qknr_oracle_e4m3_from_double_array(_p(x), _p(out), x.size)
    return out


def e4m3_to_f64(bits):
    L = lib()
    b = np.asarray(bits, dtype=np.uint8)
    table = np.array([L.qknr_oracle_e4m3_to_double(i) for i in range(256)])
    return table[b]


# ------------------------------------------------------------------ steps --
def rmsnorm(x, weight, eps):
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = None if weight is None else np.ascontiguousarray(weight, dtype=np.float64)
    y = np.empty_like(x)
    lib().qknr_oracle_rmsnorm(_p(x), x.size, _p(w), float(eps), _p(y))
    return y


def pairs_table(rotary_dim, interleaved):
    pa = np.empty(rotary_dim // 2, np.int32)
    pb = np.empty(rotary_dim // 2, np.int32)
    lib().qknr_oracle_pairs_table(rotary_dim, int(interleaved), _p(pa), _p(pb))
    return pa, pb


def pairs_3d(cf, ch, cw, interleave, neox_per_axis=False):
    d = cf + ch + cw
    pa = np.empty(d // 2, np.int32)
    pb = np.empty(d // 2, np.int32)
    lib().qknr_oracle_pairs_3d(cf, ch, cw, int(interleave), int(neox_per_axis), _p(pa), _p(pb))
    return pa, pb


def rotate(y, pa, pb, cos_t, sin_t):
    y = np.ascontiguousarray(y, dtype=np.float64)
    pa = np.ascontiguousarray(pa, np.int32)
    pb = np.ascontiguousarray(pb, np.int32)
    c = np.ascontiguousarray(cos_t, np.float64)
    s = np.ascontiguousarray(sin_t, np.float64)
    out = np.empty_like(y)
    lib().qknr_oracle_rotate(_p(y), y.size, pa.size, _p(pa), _p(pb), _p(c), _p(s), _p(out))
    return out


def position_3d(t, pos_offset, ppf, pph, ppw):
    f, h, w = C.c_int64(), C.c_int64(), C.c_int64()
    lib().qknr_oracle_position_3d(t, pos_offset, ppf, pph, ppw, C.byref(f), C.byref(h),
                                  C.byref(w))
    return f.value, h.value, w.value


def angles_3d(f, h, w, cf, ch, cw, base):
    theta = np.empty((cf + ch + cw) // 2, np.float64)
    lib().qknr_oracle_angles_3d(f, h, w, cf, ch, cw, float(base), _p(theta))
    return theta


# ------------------------------------------------------------- table form --
def rope_table(q, k, q_weight, k_weight, table, eps, rotary_dim=None, interleaved=False,
               exact=False, act="bf16"):
    """Table form. q [T,Hq,D], k [T,Hk,D], weights [D] (uint16 bit patterns of
    the activation type `act`, "bf16" or "f16"); table [T, rotary_dim] as
    float32 or uint16 patterns of the activation type. Returns (q_out, k_out) as
    activation-type bits, or as float64 before rounding when exact=True."""
    q, k = _u16(q), _u16(k)
    qw, kw = _u16(q_weight), _u16(k_weight)
    T, Hq, D = q.shape
    Hk = k.shape[1]
    R = D if rotary_dim is None else rotary_dim
    tbl = np.ascontiguousarray(table)
    is_f32 = tbl.dtype == np.float32
    assert is_f32 or tbl.dtype == np.uint16
    assert tbl.shape == (T, R), (tbl.shape, T, R)
    assert act in ("bf16", "f16")
    f16 = int(act == "f16")
    if exact:
        qo = np.empty(q.shape, np.float64)
        ko = np.empty(k.shape, np.float64)
        fn = lib().qknr_oracle_rope_table_exact_act
    else:
        qo = np.empty(q.shape, np.uint16)
        ko = np.empty(k.shape, np.uint16)
        fn = lib().qknr_oracle_rope_table_act
    rc = fn(_p(q), _p(k), _p(qw), _p(kw), _p(tbl), int(is_f32), f16, T, Hq, Hk, D, R, float(eps),
            int(interleaved), _p(qo), _p(ko))
    if rc != 0:
        raise ValueError("oracle rejected the table-form arguments")
    return qo, ko


# ---------------------------------------------------------------- 3D form --
def rope_3d(qkv, q_weight, k_weight, *, ppf, pph, ppw, num_frame_channels, num_height_channels,
            num_width_channels, num_heads_q, num_heads_k, num_heads_v, head_dim, eps=1e-6,
            base=10000.0, interleave=True, is_qk_norm=True, output_fp8=False,
            output_quant_scale=1.0, v_quant_scale=1.0, pos_offset=0, neox_per_axis=False,
            exact=False):
    """3D form. qkv [T, (Hq+Hk+Hv)*D] (or [B,S,...]) uint16 bf16 bits; weights
    [Hq*D], [Hk*D] bits. Returns (q, k, v) shaped [T, Hx, D]: bf16 bits, E4M3
    bytes with output_fp8, or float64 before scale and rounding with exact."""
    qkv = _u16(qkv)
    D = head_dim
    Hq, Hk, Hv = num_heads_q, num_heads_k, num_heads_v
    flat = qkv.reshape(-1, (Hq + Hk + Hv) * D)
    T = flat.shape[0]
    qw = None if q_weight is None else _u16(q_weight)
    kw = None if k_weight is None else _u16(k_weight)
    args = (T, pos_offset, ppf, pph, ppw, num_frame_channels, num_height_channels,
            num_width_channels, Hq, Hk, Hv, D, float(eps), float(base), int(interleave),
            int(neox_per_axis), int(is_qk_norm))
    if exact:
        qo = np.empty((T, Hq, D), np.float64)
        ko = np.empty((T, Hk, D), np.float64)
        vo = np.empty((T, Hv, D), np.float64)
        rc = lib().qknr_oracle_rope_3d_exact(_p(flat), _p(qw), _p(kw), *args, _p(qo), _p(ko),
                                             _p(vo))
    else:
        dt = np.uint8 if output_fp8 else np.uint16
        qo = np.empty((T, Hq, D), dt)
        ko = np.empty((T, Hk, D), dt)
        vo = np.empty((T, Hv, D), dt)
        rc = lib().qknr_oracle_rope_3d(_p(flat), _p(qw), _p(kw), *args, int(output_fp8),
                                       float(output_quant_scale), float(v_quant_scale), _p(qo),
                                       _p(ko), _p(vo))
    if rc != 0:
        raise ValueError("oracle rejected the 3D-form arguments")
    return qo, ko, vo


# ------------------------------------------------------ UCPE camera prep --
def relu(x):
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    lib().qknr_oracle_relu(_p(x), x.size, _p(y))
    return y


def ray_project(m, x):
    """Every block of four consecutive values of x times the 4x4 matrix m."""
    m = np.ascontiguousarray(m, dtype=np.float64).reshape(16)
    x = np.ascontiguousarray(x, dtype=np.float64)
    assert x.size % 4 == 0
    y = np.empty_like(x)
    lib().qknr_oracle_ray_project(_p(m), _p(x), x.size, _p(y))
    return y


def ucpe_cam_prep(q, k, v, proj_q, proj_kv, rope_cos, rope_sin, k_scale, exact=False,
                  act="bf16"):
    """UCPE camera prep. q, k, v [B,N,H,D] uint16 patterns of the activation type
    `act` ("bf16" or "f16"); proj_q, proj_kv [B,N,4,4] float32; rope_cos,
    rope_sin [N, D/2] float32. Returns (q_trans, k_trans, v_trans) [B,H,D,N] as
    activation-type bits (float64 before rounding when exact=True) and
    inflation_sq [B,H,N] float64."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    assert q.shape == k.shape == v.shape and q.ndim == 4, (q.shape, k.shape, v.shape)
    B, N, H, D = q.shape
    pq = np.ascontiguousarray(proj_q, np.float32)
    pkv = np.ascontiguousarray(proj_kv, np.float32)
    assert pq.shape == pkv.shape == (B, N, 4, 4), (pq.shape, pkv.shape)
    cs = np.ascontiguousarray(rope_cos, np.float32)
    sn = np.ascontiguousarray(rope_sin, np.float32)
    assert cs.shape == sn.shape == (N, D // 2), (cs.shape, sn.shape)
    assert act in ("bf16", "f16")
    dt = np.float64 if exact else np.uint16
    qo = np.empty((B, H, D, N), dt)
    ko = np.empty((B, H, D, N), dt)
    vo = np.empty((B, H, D, N), dt)
    infl = np.empty((B, H, N), np.float64)
    fn = lib().qknr_oracle_ucpe_exact if exact else lib().qknr_oracle_ucpe
    rc = fn(_p(q), _p(k), _p(v), _p(pq), _p(pkv), _p(cs), _p(sn), int(act == "f16"), B, N, H, D,
            float(k_scale), _p(qo), _p(ko), _p(vo), _p(infl))
    if rc != 0:
        raise ValueError("oracle rejected the camera-prep arguments")
    return qo, ko, vo, infl


def threads():
    return lib().qknr_oracle_threads()


def set_threads(n):
    lib().qknr_oracle_set_threads(int(n))


__all__ = ["bf16_to_f64", "bf16_from_f64", "f16_from_f64", "f16_to_f64", "e4m3_from_f64",
           "e4m3_to_f64", "rmsnorm",
           "pairs_table", "pairs_3d", "rotate", "position_3d", "angles_3d", "rope_table",
           "rope_3d", "relu", "ray_project", "ucpe_cam_prep", "threads", "set_threads", "lib"]
