"""Host-side checks of libqknr.so that need no GPU: the library loads, exports
every entry point declared in include/qknr.h, agrees with the Python struct
layout, and turns bad arguments into status codes before touching CUDA."""
import ctypes as C
import os
import re

import pytest

import qk_rmsnorm_rope_qknr_b200 as Q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qknr.h")


@pytest.fixture(scope="module")
def L():
    Q.build()
    return Q.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qknr_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    assert {"qknr_rope_table", "qknr_rope_3d", "qknr_status_string"} <= set(names)
    assert set(names) == set(Q.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_abi_version_and_strings(L):
    assert L.qknr_abi_version() == Q.ABI_VERSION == 4
    for s in range(8):
        assert L.qknr_status_string(s)
    assert L.qknr_status_string(0) == b"ok"


# Fake device addresses: every call below fails validation before any CUDA
# call, so they are never dereferenced.
A = 0x7f0000000000


def _p3(**over):
    kw = dict(ppf=2, pph=4, ppw=4, num_frame_channels=16, num_height_channels=24,
              num_width_channels=24, num_heads_q=4, num_heads_k=4, num_heads_v=4, head_dim=64,
              num_tokens=32)
    kw.update(over)
    qkv = over.pop("qkv_ptr", A)
    p = Q.make_3d_params(None, None, None, None, None, None, **{k: v for k, v in kw.items()
                                                                  if k != "qkv_ptr"})
    T = kw["num_tokens"]
    p.qkv = qkv
    p.q_weight = A + (1 << 30)
    p.k_weight = A + (1 << 30) + 4096
    p.q_out = A + (2 << 30)
    p.k_out = A + (3 << 30)
    p.v_out = A + (4 << 30)
    _ = T
    return p


def _call3d(L, p):
    rc = L.qknr_rope_3d(C.byref(p), None)
    return rc, L.qknr_last_error_detail().decode()


@pytest.mark.parametrize("over,code,needle", [
    (dict(head_dim=96, num_frame_channels=32, num_height_channels=32, num_width_channels=32),
     Q.QKNR_ERR_SHAPE, "head_dim"),
    (dict(num_frame_channels=18), Q.QKNR_ERR_SHAPE, "!= head_dim"),
    (dict(num_frame_channels=15, num_height_channels=25), Q.QKNR_ERR_SHAPE, "even"),
    (dict(num_width_channels=22), Q.QKNR_ERR_SHAPE, "head_dim"),
    (dict(num_tokens=33), Q.QKNR_ERR_SHAPE, "divisible"),
    (dict(ppf=0), Q.QKNR_ERR_SHAPE, "ppf"),
    (dict(factor=2.0), Q.QKNR_ERR_UNSUPPORTED, "YARN"),
    (dict(attention_factor=0.5), Q.QKNR_ERR_SHAPE, "attention_factor"),
    (dict(base=0.0), Q.QKNR_ERR_SHAPE, "base"),
    (dict(num_heads_q=0, num_heads_k=0, num_heads_v=0), Q.QKNR_ERR_SHAPE, "head"),
    (dict(num_heads_q=-1), Q.QKNR_ERR_SHAPE, "head"),
    (dict(num_heads_q=4096), Q.QKNR_ERR_UNSUPPORTED, "heads"),
    (dict(num_tokens=-1, pos_offset=1), Q.QKNR_ERR_SHAPE, "num_tokens"),
    (dict(pos_offset=-3), Q.QKNR_ERR_SHAPE, "pos_offset"),
    (dict(eps=-1.0), Q.QKNR_ERR_SHAPE, "eps"),
    (dict(qkv_ptr=0), Q.QKNR_ERR_NULL, "qkv"),
    (dict(qkv_ptr=A + 8), Q.QKNR_ERR_ALIGN, "16-byte"),
    # NeoX pairs per axis group are built for groups that are multiples of 16
    (dict(interleave=False, neox_per_axis=True), Q.QKNR_ERR_UNSUPPORTED, "multiples of 16"),
])
def test_3d_validation(L, over, code, needle):
    p = _p3(**over)
    rc, detail = _call3d(L, p)
    assert rc == code, (rc, detail)
    assert needle in detail


def test_3d_struct_size_guard(L):
    p = _p3()
    p.struct_size = C.sizeof(Q.Rope3DParams) - 8
    rc, detail = _call3d(L, p)
    assert rc == Q.QKNR_ERR_SHAPE and "struct_size" in detail
    # the real size passes the guard (and then fails on head_dim, proving the layout)
    p = _p3(head_dim=32, num_frame_channels=8, num_height_channels=8, num_width_channels=16)
    rc, detail = _call3d(L, p)
    assert rc == Q.QKNR_ERR_SHAPE and "head_dim 32" in detail


def test_3d_null_outputs_and_weights(L):
    p = _p3()
    p.v_out = None
    assert _call3d(L, p)[0] == Q.QKNR_ERR_NULL
    p = _p3()
    p.q_weight = None
    assert _call3d(L, p)[0] == Q.QKNR_ERR_NULL
    p = _p3(is_qk_norm=False, num_heads_v=0)
    p.q_weight = p.k_weight = None
    p.v_out = None
    p.q_out = A + (2 << 30) + 8
    assert _call3d(L, p)[0] == Q.QKNR_ERR_ALIGN     # passes the NULL checks, fails alignment


def test_3d_aliasing(L):
    p = _p3()
    p.q_out = A + 4096      # inside qkv (32 rows of 1536 bytes)
    assert _call3d(L, p)[0] == Q.QKNR_ERR_ALIAS
    p = _p3()
    p.k_out = p.q_out + 1024
    assert _call3d(L, p)[0] == Q.QKNR_ERR_ALIAS
    p = _p3()
    p.v_out = p.q_weight
    assert _call3d(L, p)[0] == Q.QKNR_ERR_ALIAS


def test_3d_zero_tokens_is_noop(L):
    p = _p3(num_tokens=0)
    p.qkv = p.q_out = p.k_out = p.v_out = None
    assert _call3d(L, p)[0] == Q.QKNR_OK


def _table(L, **over):
    kw = dict(q=A, k=A + (1 << 30), q_out=A + (2 << 30), k_out=A + (3 << 30),
              q_weight=A + (4 << 30), k_weight=A + (4 << 30) + 4096, rope_table=A + (5 << 30),
              table_dtype=Q.QKNR_DT_F32, act=Q.QKNR_DT_BF16, T=16, Hq=4, Hk=2, D=128, R=96, qs=0, ks=0, qos=0,
              kos=0, eps=1e-6, il=0)
    kw.update(over)
    rc = L.qknr_rope_table(kw["q"], kw["k"], kw["q_out"], kw["k_out"], kw["q_weight"],
                           kw["k_weight"], kw["rope_table"], kw["table_dtype"], kw["act"], kw["T"],
                           kw["Hq"],
                           kw["Hk"], kw["D"], kw["R"], kw["qs"], kw["ks"], kw["qos"], kw["kos"],
                           kw["eps"], kw["il"], None)
    return rc, L.qknr_last_error_detail().decode()


@pytest.mark.parametrize("over,code", [
    (dict(D=0), Q.QKNR_ERR_SHAPE), (dict(D=258, R=96), Q.QKNR_ERR_SHAPE),
    (dict(R=97), Q.QKNR_ERR_SHAPE), (dict(R=130), Q.QKNR_ERR_SHAPE),
    (dict(table_dtype=Q.QKNR_DT_E4M3), Q.QKNR_ERR_SHAPE), (dict(T=-1), Q.QKNR_ERR_SHAPE),
    (dict(act=Q.QKNR_DT_F32), Q.QKNR_ERR_SHAPE), (dict(act=Q.QKNR_DT_E4M3), Q.QKNR_ERR_SHAPE),
    (dict(table_dtype=Q.QKNR_DT_F16), Q.QKNR_ERR_SHAPE),             # 16-bit table of another type
    (dict(act=Q.QKNR_DT_F16, table_dtype=Q.QKNR_DT_BF16), Q.QKNR_ERR_SHAPE),
    (dict(Hq=-2), Q.QKNR_ERR_SHAPE), (dict(eps=-1.0), Q.QKNR_ERR_SHAPE),
    (dict(qs=100), Q.QKNR_ERR_SHAPE), (dict(q=0), Q.QKNR_ERR_NULL),
    (dict(k_weight=0), Q.QKNR_ERR_NULL), (dict(rope_table=0), Q.QKNR_ERR_NULL),
    (dict(q_out=A + 64), Q.QKNR_ERR_ALIAS), (dict(k_out=A + (2 << 30) + 256), Q.QKNR_ERR_ALIAS),
    (dict(q_out=A + (5 << 30)), Q.QKNR_ERR_ALIAS),
    (dict(q_out=A, qos=1024), Q.QKNR_ERR_ALIAS),          # in place needs the same stride
    (dict(q=A + 1), Q.QKNR_ERR_ALIGN), (dict(rope_table=A + (5 << 30) + 2), Q.QKNR_ERR_ALIGN),
])
def test_table_validation(L, over, code):
    rc, detail = _table(L, **over)
    assert rc == code, (rc, detail)
    assert detail


def test_table_noops(L):
    assert _table(L, T=0, q=0, k=0, q_out=0, k_out=0)[0] == Q.QKNR_OK
    assert _table(L, Hq=0, Hk=0, q=0, k=0)[0] == Q.QKNR_OK


def test_python_wrapper_raises_valueerror(L):
    import torch

    x = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    w = torch.zeros(64, dtype=torch.bfloat16)
    tbl = torch.zeros(4, 64, dtype=torch.float32)
    with pytest.raises(ValueError):
        Q.fused_qk_norm_rope(x, x, w, w, tbl[:, :63], 1e-6)
    with pytest.raises(ValueError):
        Q.fused_qk_norm_rope(x.float(), x, w, w, tbl, 1e-6)
    with pytest.raises(ValueError):                       # q float16, k bf16
        Q.fused_qk_norm_rope(x.half(), x, w.half(), w.half(), tbl, 1e-6)
    with pytest.raises(ValueError):                       # float16 activations, bf16 weights
        Q.fused_qk_norm_rope(x.half(), x.half(), w, w, tbl, 1e-6)
    with pytest.raises(ValueError):                       # float16 activations, bf16 table
        Q.fused_qk_norm_rope(x.half(), x.half(), w.half(), w.half(), tbl.bfloat16(), 1e-6)



def test_prepared_3d_call_checks_tensors_before_the_library(L):
    """Rope3DCall checks what changes per call (dtype, density, element counts)
    in Python and raises ValueError before any pointer reaches the library."""
    import torch

    p = dict(ppf=1, pph=2, ppw=3, num_frame_channels=16, num_height_channels=24,
             num_width_channels=24, num_heads_q=2, num_heads_k=1, num_heads_v=1, head_dim=64,
             interleave=False, output_fp8=True, pos_offset=0)
    call = Q.Rope3DCall(**p)
    T, row = 6, 4 * 64
    qkv = torch.zeros(T, row, dtype=torch.bfloat16)
    qw = torch.zeros(2 * 64, dtype=torch.bfloat16)
    kw = torch.zeros(64, dtype=torch.bfloat16)
    f8 = torch.float8_e4m3fn
    outs = [torch.zeros(T, h, 64, dtype=f8) for h in (2, 1, 1)]
    bad_cases = [
        (qkv.float(), qw, kw, *outs),                                        # qkv dtype
        (qkv[:, :-8].contiguous(), qw, kw, *outs),                           # not whole rows
        (qkv.t().contiguous().t(), qw, kw, *outs),                           # not dense
        (qkv, qw, kw, torch.zeros(T, 2, 64, dtype=torch.bfloat16), *outs[1:]),  # bf16 out, FP8 call
        (qkv, qw, kw, outs[0][:-1], *outs[1:]),                              # too few tokens
        (qkv, qw, kw, outs[0], outs[1], None),                               # missing output
        (qkv, qw.float(), kw, *outs),                                        # weight dtype
        (qkv, qw, kw[:-1], *outs),                                           # weight size
        (qkv, None, kw, *outs),                                              # missing weight
    ]
    for args in bad_cases:
        with pytest.raises(ValueError):
            call(*args, stream=0)
    with pytest.raises(ValueError):                       # a bad static parameter
        Q.Rope3DCall(**dict(p, num_heads_q=-1))(qkv, qw, kw, *outs, stream=0)


def test_prepared_table_call_checks_tensors_before_the_library(L):
    """RopeTableCall raises ValueError on a wrong shape, dtype, head layout,
    table or weight before any pointer reaches the library."""
    import torch

    call = Q.RopeTableCall(heads_q=3, heads_k=2, head_dim=64, eps=1e-6, rotary_dim=48)
    T = 5
    q = torch.zeros(T, 3, 64, dtype=torch.bfloat16)
    k = torch.zeros(T, 2, 64, dtype=torch.bfloat16)
    w = torch.zeros(64, dtype=torch.bfloat16)
    tbl = torch.zeros(T, 48)
    bad_cases = [
        (q.half(), k, q, k, w, w, tbl),                          # activation dtype
        (q, k[:-1], q, k, w, w, tbl),                            # token counts differ
        (q, k, q[:, :2], k, w, w, tbl),                          # head count
        (q.transpose(1, 2).contiguous().transpose(1, 2), k, q, k, w, w, tbl),  # heads not dense
        (q, k, q, k, w, w, tbl[:, :46]),                         # table width
        (q, k, q, k, w, w, tbl.bfloat16()),                      # table dtype
        (q, k, q, k, w[:-1], w, tbl),                            # weight size
        (q, k, q, k, w, w.float(), tbl),                         # weight dtype
    ]
    for args in bad_cases:
        with pytest.raises(ValueError):
            call(*args, stream=0)
    with pytest.raises(ValueError):                       # table dtype not f32 / activation
        Q.RopeTableCall(heads_q=3, heads_k=2, head_dim=64, eps=1e-6, table_dtype=torch.float16)

def test_wait_fault_hook_argument_checks(L):
    assert L.qknr_test_set_wait_fault(8, 1000) == Q.QKNR_ERR_SHAPE
    assert L.qknr_test_set_wait_fault(16, 0) == Q.QKNR_ERR_SHAPE
    assert L.qknr_test_set_wait_fault(0, 0) == Q.QKNR_OK


def test_tensor_parallel_entry_point_checks(L):
    p = _p3()
    assert L.qknr_rope_3d_partial_ssq(C.byref(p), None, None) == Q.QKNR_ERR_NULL
    assert L.qknr_rope_3d_partial_ssq(C.byref(p), A + (6 << 30) + 4, None) == Q.QKNR_ERR_ALIGN
    assert L.qknr_rope_3d_partial_ssq(C.byref(p), A + 64, None) == Q.QKNR_ERR_ALIAS  # inside qkv
    assert L.qknr_rope_3d_with_ssq(C.byref(p), None, 4, 4, None) == Q.QKNR_ERR_NULL
    assert L.qknr_rope_3d_with_ssq(C.byref(p), A + (6 << 30), 3, 4, None) == Q.QKNR_ERR_SHAPE
    p2 = _p3(is_qk_norm=False)
    assert L.qknr_rope_3d_with_ssq(C.byref(p2), A + (6 << 30), 4, 4, None) == Q.QKNR_ERR_SHAPE
    assert b"is_qk_norm" in L.qknr_last_error_detail()
    p3 = _p3()
    p3.q_out = A + (6 << 30)  # overlaps the supplied sums
    assert L.qknr_rope_3d_with_ssq(C.byref(p3), A + (6 << 30), 4, 4, None) == Q.QKNR_ERR_ALIAS


def test_tp_head_slices():
    from qk_rmsnorm_rope_qknr_b200 import tp

    for total in (1, 5, 24, 32):
        for world in (1, 2, 3, 4, 8):
            sl = [tp.head_slice(total, world, r) for r in range(world)]
            assert sl[0][0] == 0 and sl[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(sl, sl[1:]))


# ---------------------------------------------------------- UCPE camera prep --
def _ucpe(L, **over):
    kw = dict(q=A, k=A + (1 << 30), v=A + (2 << 30), pq=A + (3 << 30), pkv=A + (4 << 30),
              cos=A + (5 << 30), sin=A + (6 << 30), qo=A + (7 << 30), ko=A + (8 << 30),
              vo=A + (9 << 30), infl=A + (10 << 30), act=Q.QKNR_DT_BF16, B=1, N=64, H=2, D=112,
              k_scale=0.1)
    kw.update(over)
    rc = L.qknr_ucpe_cam_prep(kw["q"], kw["k"], kw["v"], kw["pq"], kw["pkv"], kw["cos"],
                              kw["sin"], kw["qo"], kw["ko"], kw["vo"], kw["infl"], kw["act"],
                              kw["B"], kw["N"], kw["H"], kw["D"], kw["k_scale"], None)
    return rc, L.qknr_last_error_detail().decode()


@pytest.mark.parametrize("over,code,needle", [
    (dict(D=100), Q.QKNR_ERR_SHAPE, "multiple of 8"),
    (dict(D=0), Q.QKNR_ERR_SHAPE, "multiple of 8"),
    (dict(D=264), Q.QKNR_ERR_SHAPE, "multiple of 8"),
    (dict(N=-1), Q.QKNR_ERR_SHAPE, ">= 0"),
    (dict(act=Q.QKNR_DT_F32), Q.QKNR_ERR_SHAPE, "dtype"),
    (dict(act=Q.QKNR_DT_E4M3), Q.QKNR_ERR_SHAPE, "dtype"),
    (dict(k_scale=float("inf")), Q.QKNR_ERR_SHAPE, "k_scale"),
    (dict(k_scale=float("nan")), Q.QKNR_ERR_SHAPE, "k_scale"),
    (dict(B=1 << 20, N=1 << 20, H=64, D=256), Q.QKNR_ERR_SHAPE, "too large"),
    (dict(q=None), Q.QKNR_ERR_NULL, "q_normed"),
    (dict(pkv=None), Q.QKNR_ERR_NULL, "proj"),
    (dict(sin=None), Q.QKNR_ERR_NULL, "rope"),
    (dict(vo=None), Q.QKNR_ERR_NULL, "v_trans"),
    (dict(k=A + (1 << 30) + 8), Q.QKNR_ERR_ALIGN, "16-byte"),
    (dict(pq=A + (3 << 30) + 4), Q.QKNR_ERR_ALIGN, "16-byte"),
    (dict(infl=A + (10 << 30) + 4), Q.QKNR_ERR_ALIGN, "16-byte"),
    (dict(qo=A), Q.QKNR_ERR_ALIAS, "overlaps an input"),
    (dict(ko=A + (7 << 30) + 16), Q.QKNR_ERR_ALIAS, "outputs overlap"),
    (dict(infl=A + (6 << 30) + 64), Q.QKNR_ERR_ALIAS, "overlaps an input"),
])
def test_ucpe_host_validation(L, over, code, needle):
    rc, detail = _ucpe(L, **over)
    assert rc == code and needle in detail, (rc, detail)


@pytest.mark.parametrize("over", [dict(B=0), dict(N=0), dict(H=0)])
def test_ucpe_empty_is_a_no_op(L, over):
    # nothing is launched, so the fake addresses are never used
    assert _ucpe(L, **over) == (Q.QKNR_OK, "")


def test_ucpe_binding_checks_shapes(L):
    import torch
    x = torch.zeros(1, 8, 2, 16, dtype=torch.bfloat16)
    good = dict(proj_q=torch.zeros(1, 8, 4, 4), proj_kv=torch.zeros(1, 8, 4, 4),
                rope_cos=torch.zeros(8, 8), rope_sin=torch.zeros(8, 8), k_scale=1.0)
    with pytest.raises(Q.QknrValueError, match="rope_cos"):
        Q.cam_prep_func(x, x, x, **dict(good, rope_cos=torch.zeros(8, 16)))
    with pytest.raises(Q.QknrValueError, match="proj_kv"):
        Q.cam_prep_func(x, x, x, **dict(good, proj_kv=torch.zeros(1, 8, 4, 4,
                                                                  dtype=torch.float64)))
    with pytest.raises(Q.QknrValueError, match="k_normed"):
        Q.cam_prep_func(x, x.float(), x, **good)
    with pytest.raises(Q.QknrValueError, match="bfloat16/float16"):
        Q.cam_prep_func(x.float(), x.float(), x.float(), **good)
