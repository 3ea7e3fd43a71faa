"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerance (tests/_util.py): bf16 outputs within 2 ulp of the oracle's rounded
result, with the ulp taken at max(|ref|, 2^-8 * RMS of the head row); E4M3
outputs within one code step. Pure copies (V in bf16, and Q/K at patch
(0,0,0) without the norm) must be bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle as O
import qk_rmsnorm_rope_qknr_b200 as Q
import workloads as W
from tests._util import act_mismatch, bf16_mismatch, e4m3_mismatch, t2u16, t2u8

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _p3(w: W.Form3D, **over):
    p = w.params()
    p.update(over)
    return p


def run_3d(qkv, qw, kw, stream=None, **p):
    return Q.fused_qk_rmsnorm_rope(qkv, qw, kw, stream=stream, **p)


def oracle_3d(qkv_cpu, qw_cpu, kw_cpu, **p):
    bits = t2u16(qkv_cpu)
    qwb = t2u16(qw_cpu) if qw_cpu is not None else None
    kwb = t2u16(kw_cpu) if kw_cpu is not None else None
    exact = O.rope_3d(bits, qwb, kwb, exact=True, **p)
    rounded = O.rope_3d(bits, qwb, kwb, **p)
    return rounded, exact


def assert_3d_close(outs, ref, exact, fp8, what=""):
    names = ("q", "k", "v")
    for n, o, r, x in zip(names, outs, ref, exact):
        T = r.shape[0]
        if fp8:
            bad, st = e4m3_mismatch(t2u8(o).reshape(r.shape), r)
            assert len(bad) == 0, f"{what} {n}: {len(bad)} E4M3 codes off by >1 step {st}"
        else:
            g = t2u16(o).reshape(r.shape)
            if n == "v":
                assert np.array_equal(g, r), f"{what} v is not a bit copy"
                continue
            bad, st = bf16_mismatch(g, r, x)
            assert len(bad) == 0, f"{what} {n}: {len(bad)} of {g.size} beyond 2 ulp {st}, " \
                                  f"first at {bad[:3].tolist()}"
        _ = T


def check_3d_case(qkv, qw, kw, **p):
    outs = run_3d(qkv, qw, kw, **p)
    torch.cuda.synchronize()
    cpu = lambda t: None if t is None else t.cpu()  # noqa: E731
    ref, exact = oracle_3d(cpu(qkv).reshape(-1, qkv.shape[-1]), cpu(qw), cpu(kw), **p)
    assert_3d_close(outs, ref, exact, p.get("output_fp8", False), str(p))
    return outs


# --------------------------------------------------------------- workloads --
@pytest.mark.parametrize("name", ["tiny3d", "video3d", "fp8neox", "fp8neox_nonorm", "gqa3d"])
def test_3d_workload_ragged_shard(name):
    """The workload's geometry on a shard of 3001 tokens that starts mid-grid:
    several CTAs' worth of tokens per CTA, a ragged end, wrapped positions."""
    w = W.WORKLOADS[name]
    T = 32 if name == "tiny3d" else 3001
    off = 0 if name == "tiny3d" else 12345
    inp = W.make_inputs(w, device="cpu", tokens=T)
    g = {k: v.to(DEV) for k, v in inp.items()}
    check_3d_case(g["qkv"], g["q_weight"], g["k_weight"], pos_offset=off, **_p3(w))


@pytest.mark.parametrize("name", ["video3d", "fp8neox", "fp8neox_nonorm", "gqa3d"])
def test_3d_workload_full_size_every_token(name, capsys):
    """Full-size workload in the benchmark's launch configuration, every
    element of q_out, k_out and v_out against the oracle. The oracle runs over
    the whole call in chunks of tokens (a chunk starting at token t0 is the
    same call's tokens with pos_offset t0), so the kernel's long rings (tens of
    tokens per pipeline, thousands of parity flips) are compared in full."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, device=DEV)
    qkv = inp["qkv"]
    p = _p3(w)
    outs = run_3d(qkv, inp["q_weight"], inp["k_weight"], **p)
    torch.cuda.synchronize()
    T = w.tokens
    flat = qkv.reshape(T, -1).cpu()
    got = [o.reshape(T, -1, w.head_dim).cpu() for o in outs]
    cpu = lambda t: None if t is None else t.cpu()  # noqa: E731
    qw_cpu, kw_cpu = cpu(inp["q_weight"]), cpu(inp["k_weight"])
    bits = lambda t: None if t is None else t2u16(t)  # noqa: E731
    del outs, inp, qkv
    stats = {n: dict(n=0, exact=0, max_err=0.0) for n in "qkv"}
    chunk = 4096
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        rows = flat[t0:t1]
        if w.output_fp8:
            ref = O.rope_3d(t2u16(rows), bits(qw_cpu), bits(kw_cpu), pos_offset=t0, **p)
            exact = (None, None, None)
        else:
            ref, exact = oracle_3d(rows, qw_cpu, kw_cpu, pos_offset=t0, **p)
        for n, g, r, x in zip("qkv", got, ref, exact):
            gs = g[t0:t1]
            if w.output_fp8:
                bad, st = e4m3_mismatch(t2u8(gs).reshape(r.shape), r)
                err = st["max_steps"]
            elif n == "v":
                gb = t2u16(gs).reshape(r.shape)
                bad = np.argwhere(gb != r)
                st = dict(exact_frac=float(np.mean(gb == r)), n=int(r.size))
                err = 0.0 if len(bad) == 0 else float("inf")
            else:
                bad, st = bf16_mismatch(t2u16(gs).reshape(r.shape), r, x)
                err = st["max_err_ulps"]
            assert len(bad) == 0, (f"{name} {n}: {len(bad)} of {r.size} beyond tolerance in "
                                   f"tokens [{t0}, {t1}) {st}, first at {bad[:3].tolist()}")
            s = stats[n]
            s["exact"] += st["exact_frac"] * st["n"]
            s["n"] += st["n"]
            s["max_err"] = max(s["max_err"], err)
    unit = "E4M3 steps" if w.output_fp8 else "bf16 ulp"
    with capsys.disabled():
        print(f"\n[every-token parity] {name} ({T} tokens): " + "; ".join(
            f"{n}_out exact_frac {s['exact'] / s['n']:.6f}, max {s['max_err']:.3g} {unit}"
            for n, s in stats.items()))


@pytest.mark.parametrize("name", ["table_hs", "table_il", "table_hs_f16", "table_d72"])
def test_table_workload_full(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, device="cpu")
    g = {k: v.to(DEV) for k, v in inp.items()}
    qo, ko = Q.fused_qk_norm_rope(g["q"], g["k"], g["q_weight"], g["k_weight"], g["rope_table"],
                                  w.eps, rotary_dim=w.rotary_dim, interleaved=w.interleaved)
    torch.cuda.synchronize()
    check_table_against_oracle(inp, qo, ko, w.eps, w.rotary_dim, w.interleaved)


def _table_bits(t):
    return t.numpy() if t.dtype == torch.float32 else t2u16(t)


def check_table_against_oracle(inp, qo, ko, eps, rd, il, what=""):
    args = (t2u16(inp["q"]), t2u16(inp["k"]), t2u16(inp["q_weight"]), t2u16(inp["k_weight"]),
            _table_bits(inp["rope_table"].cpu().contiguous()), eps, rd)
    act = "f16" if inp["q"].dtype == torch.float16 else "bf16"
    ex_q, ex_k = O.rope_table(*args, interleaved=il, exact=True, act=act)
    rq, rk = O.rope_table(*args, interleaved=il, act=act)
    for n, o, r, x in (("q", qo, rq, ex_q), ("k", ko, rk, ex_k)):
        bad, st = act_mismatch(t2u16(o), r, x, act)
        assert len(bad) == 0, f"{what} {n}: {len(bad)} beyond tolerance {st} at {bad[:3].tolist()}"


# ------------------------------------------------------------- 3D variants --
def _rand3d(T, Hq, Hk, Hv, D, std=1.0, seed=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    qkv = (torch.randn(T, (Hq + Hk + Hv) * D, generator=g) * std).to(torch.bfloat16)
    qw = (1 + 0.1 * torch.randn(Hq * D, generator=g)).to(torch.bfloat16)
    kw = (1 + 0.1 * torch.randn(Hk * D, generator=g)).to(torch.bfloat16)
    return qkv.to(DEV), qw.to(DEV), kw.to(DEV)


CASES_3D = [
    # (T, Hq, Hk, Hv, D, grid, channels, interleave, fp8, norm, pos_offset)
    (12, 5, 3, 2, 64, (1, 3, 4), (16, 24, 24), True, False, True, 0),
    (12, 5, 3, 2, 64, (1, 3, 4), (16, 24, 24), False, True, True, 0),
    (40, 2, 2, 2, 256, (2, 4, 5), (64, 96, 96), True, True, False, 0),
    (40, 2, 6, 1, 256, (2, 4, 5), (0, 128, 128), False, False, True, 0),
    (7, 1, 1, 1, 128, (1, 1, 1), (32, 48, 48), True, False, True, 0),       # P = 1
    (1, 4, 4, 4, 128, (3, 5, 7), (16, 56, 56), False, False, True, 77),     # a single token
    (99, 80, 8, 8, 128, (3, 3, 11), (32, 48, 48), True, False, True, 5),    # 2 slots per thread
    (33, 200, 160, 8, 128, (1, 3, 11), (32, 48, 48), False, True, True, 9),  # 4 slots
    (64, 4, 4, 40, 64, (4, 4, 4), (16, 24, 24), True, False, True, 0),      # V-heavy row
    (10000, 2, 2, 2, 64, (1, 1, 10000), (0, 0, 64), True, False, True, 0),  # no smem table
    (257, 0, 4, 2, 128, (1, 1, 257), (32, 48, 48), True, False, True, 0),   # no Q heads
    (64, 3, 3, 0, 128, (4, 4, 4), (32, 48, 48), False, True, True, 0),      # no V heads
    (3000, 32, 8, 8, 128, (3, 40, 25), (32, 48, 48), True, False, True, 0),  # grouped-query
    (2048, 16, 4, 4, 128, (2, 32, 32), (32, 48, 48), False, True, True, 0),  # GQA, NeoX, E4M3
]


@pytest.mark.parametrize("case", CASES_3D, ids=[str(i) for i in range(len(CASES_3D))])
def test_3d_variants(case):
    T, Hq, Hk, Hv, D, grid, ch, il, fp8, norm, off = case
    qkv, qw, kw = _rand3d(T, Hq, Hk, Hv, D, std=2.0, seed=T + D)
    p = dict(ppf=grid[0], pph=grid[1], ppw=grid[2], num_frame_channels=ch[0],
             num_height_channels=ch[1], num_width_channels=ch[2], num_heads_q=Hq, num_heads_k=Hk,
             num_heads_v=Hv, head_dim=D, eps=1e-5, base=10000.0, interleave=il, is_qk_norm=norm,
             output_fp8=fp8, output_quant_scale=0.75, v_quant_scale=1.5, pos_offset=off)
    check_3d_case(qkv, qw if norm else None, kw if norm else None, **p)


CASES_PER_AXIS = [
    # (T, Hq, Hk, Hv, D, grid, channels, fp8, norm, pos_offset)
    (3001, 24, 24, 24, 128, (31, 24, 40), (32, 48, 48), True, True, 12345),   # FP8 NeoX geometry
    (3001, 24, 24, 24, 128, (31, 24, 40), (32, 48, 48), True, False, 12345),  # without the norm
    (3001, 24, 24, 24, 128, (31, 24, 40), (32, 48, 48), False, True, 5),      # bf16 out
    (500, 5, 3, 2, 64, (2, 5, 50), (16, 16, 32), False, True, 7),             # grouped-query
    (300, 2, 2, 1, 256, (3, 4, 25), (64, 96, 96), False, True, 0),            # head_dim 256
    (300, 2, 2, 1, 256, (3, 4, 25), (64, 96, 96), True, True, 0),
    (400, 4, 4, 4, 128, (1, 20, 20), (0, 64, 64), False, True, 0),            # empty frame group
]


@pytest.mark.parametrize("case", CASES_PER_AXIS, ids=[str(i) for i in range(len(CASES_PER_AXIS))])
def test_3d_neox_per_axis(case):
    """NeoX halves inside each axis group (neox_per_axis), the other reading
    of the page's "NeoX-style", against the oracle's per-axis pair map."""
    T, Hq, Hk, Hv, D, grid, ch, fp8, norm, off = case
    qkv, qw, kw = _rand3d(T, Hq, Hk, Hv, D, std=2.0, seed=T + D + 1)
    p = dict(ppf=grid[0], pph=grid[1], ppw=grid[2], num_frame_channels=ch[0],
             num_height_channels=ch[1], num_width_channels=ch[2], num_heads_q=Hq, num_heads_k=Hk,
             num_heads_v=Hv, head_dim=D, eps=1e-5, base=10000.0, interleave=False,
             is_qk_norm=norm, output_fp8=fp8, output_quant_scale=0.75, v_quant_scale=1.5,
             pos_offset=off, neox_per_axis=True)
    outs = check_3d_case(qkv, qw if norm else None, kw if norm else None, **p)
    whole = run_3d(qkv, qw if norm else None, kw if norm else None, **dict(p, neox_per_axis=False))
    assert not torch.equal(outs[0].view(torch.uint8), whole[0].view(torch.uint8))


def test_3d_neox_per_axis_ignored_when_interleaved():
    """With adjacent pairs the two readings coincide: the flag changes nothing."""
    qkv, qw, kw = _rand3d(200, 4, 4, 4, 128, seed=8)
    p = dict(ppf=2, pph=10, ppw=10, num_frame_channels=32, num_height_channels=48,
             num_width_channels=48, num_heads_q=4, num_heads_k=4, num_heads_v=4, head_dim=128,
             interleave=True)
    a = run_3d(qkv, qw, kw, **p)
    b = run_3d(qkv, qw, kw, neox_per_axis=True, **p)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_3d_rope_only_origin_is_bit_copy():
    qkv, _, _ = _rand3d(16, 4, 4, 4, 64, std=3.0)
    p = dict(ppf=1, pph=4, ppw=4, num_frame_channels=16, num_height_channels=24,
             num_width_channels=24, num_heads_q=4, num_heads_k=4, num_heads_v=4, head_dim=64,
             is_qk_norm=False)
    q, k, v = run_3d(qkv, None, None, **p)
    assert torch.equal(q[0].reshape(-1), qkv[0, :256]) and torch.equal(k[0].reshape(-1),
                                                                         qkv[0, 256:512])
    assert torch.equal(v.reshape(16, -1), qkv[:, 512:])


def test_3d_base_below_one_and_large_positions():
    """base < 1 makes frequencies above one turn; a 60000-wide grid makes large
    angles: the fixed-point angle keeps both within tolerance."""
    qkv, qw, kw = _rand3d(600, 2, 2, 1, 64, seed=3)
    p = dict(ppf=1, pph=1, ppw=60000, num_frame_channels=16, num_height_channels=16,
             num_width_channels=32, num_heads_q=2, num_heads_k=2, num_heads_v=1, head_dim=64,
             base=0.37, pos_offset=59500)
    check_3d_case(qkv, qw, kw, **p)


def test_3d_output_guards_and_poison():
    """Every output element is written and nothing past the end: outputs are
    pre-filled with 0xFF (a NaN pattern the op cannot produce from finite
    inputs) and followed by guard bytes."""
    T, H, D = 48, 3, 128
    qkv, qw, kw = _rand3d(T, H, H, H, D)
    for fp8 in (False, True):
        eb = 1 if fp8 else 2
        n = T * H * D * eb
        bufs = [torch.full((n + 4096,), 0xFF, dtype=torch.uint8, device=DEV) for _ in range(3)]
        odt = torch.float8_e4m3fn if fp8 else torch.bfloat16
        outs = [b[:n].view(odt) for b in bufs]
        p = dict(ppf=1, pph=6, ppw=8, num_frame_channels=32, num_height_channels=48,
                 num_width_channels=48, num_heads_q=H, num_heads_k=H, num_heads_v=H, head_dim=D,
                 output_fp8=fp8, output_quant_scale=0.5, v_quant_scale=0.5)
        Q.qknr_rope_3d(qkv, qw, kw, *outs, **p)
        torch.cuda.synchronize()
        for b in bufs:
            assert torch.all(b[n:] == 0xFF), "guard bytes overwritten"
            body = b[:n]
            if fp8:
                assert not torch.any(body == 0xFF)
            else:
                assert not torch.any(body.view(torch.int16) == -1)


def test_3d_pinned_host_buffers():
    """The C ABI accepts page-locked host memory: the kernel reads and writes it
    across the bus. Same results as device buffers."""
    qkv, qw, kw = _rand3d(64, 4, 4, 4, 64, seed=11)
    p = dict(ppf=4, pph=4, ppw=4, num_frame_channels=16, num_height_channels=24,
             num_width_channels=24, num_heads_q=4, num_heads_k=4, num_heads_v=4, head_dim=64)
    dev_out = run_3d(qkv, qw, kw, **p)
    h_qkv = qkv.cpu().pin_memory()
    h_out = [torch.empty(64, 4, 64, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    Q.qknr_rope_3d(h_qkv, qw, kw, *h_out, stream=torch.cuda.current_stream(), **p)
    torch.cuda.synchronize()
    for a, b in zip(dev_out, h_out):
        assert torch.equal(a.cpu(), b)


@pytest.mark.parametrize("D,R,il", [(128, 96, False), (72, 40, True)], ids=["fast", "smem"])
def test_table_pinned_host_buffers(D, R, il):
    """The table form on page-locked host q, k, table and outputs (the kernels'
    bulk copies and table loads cross the bus): the same bits as on device
    buffers, for the fast kernel and the shared-memory kernel."""
    inp = _rand_table_inputs(256, 6, 2, D, R, True, seed=D)
    g = {n: t.to(DEV) for n, t in inp.items()}
    dq, dk = Q.fused_qk_norm_rope(g["q"], g["k"], g["q_weight"], g["k_weight"], g["rope_table"],
                                  1e-6, rotary_dim=R, interleaved=il)
    h = {n: inp[n].pin_memory() for n in ("q", "k", "rope_table")}
    hq, hk = torch.empty_like(h["q"]).pin_memory(), torch.empty_like(h["k"]).pin_memory()
    Q.qknr_rope_table(h["q"], h["k"], hq, hk, g["q_weight"], g["k_weight"], h["rope_table"],
                      eps=1e-6, rotary_dim=R, interleaved=il,
                      stream=torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert torch.equal(dq.cpu(), hq) and torch.equal(dk.cpu(), hk)


def test_3d_pageable_host_memory_is_rejected():
    qkv, qw, kw = _rand3d(16, 4, 4, 4, 64)
    p = dict(ppf=1, pph=4, ppw=4, num_frame_channels=16, num_height_channels=24,
             num_width_channels=24, num_heads_q=4, num_heads_k=4, num_heads_v=4, head_dim=64)
    with pytest.raises(ValueError, match="device cannot access|pageable"):
        Q.fused_qk_rmsnorm_rope(qkv.cpu(), qw, kw, q_out=torch.empty(16, 4, 64, dtype=torch.bfloat16,
                                                                      device=DEV),
                                k_out=torch.empty(16, 4, 64, dtype=torch.bfloat16, device=DEV),
                                v_out=torch.empty(16, 4, 64, dtype=torch.bfloat16, device=DEV),
                                **p)


def test_3d_deterministic_and_streams():
    w = W.WORKLOADS["tiny3d"]
    inp = {k: v.to(DEV) for k, v in W.make_inputs(w).items()}
    a = run_3d(inp["qkv"], inp["q_weight"], inp["k_weight"], **w.params())
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = run_3d(inp["qkv"], inp["q_weight"], inp["k_weight"], stream=s, **w.params())
    s.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)



@pytest.mark.parametrize("case", [CASES_3D[1], CASES_3D[6], CASES_3D[13]], ids=["neox_e4m3", "slots2", "gqa"])
def test_3d_prepared_call_matches_wrapper(case):
    """Rope3DCall (parameters fixed once) gives the wrapper's bytes, for a whole
    call and for shards of other token counts through the same instance."""
    T, Hq, Hk, Hv, D, grid, ch, il, fp8, norm, off = case
    qkv, qw, kw = _rand3d(T, Hq, Hk, Hv, D, std=2.0, seed=T + D + 1)
    p = dict(ppf=grid[0], pph=grid[1], ppw=grid[2], num_frame_channels=ch[0],
             num_height_channels=ch[1], num_width_channels=ch[2], num_heads_q=Hq, num_heads_k=Hk,
             num_heads_v=Hv, head_dim=D, eps=1e-5, base=10000.0, interleave=il, is_qk_norm=norm,
             output_fp8=fp8, output_quant_scale=0.75, v_quant_scale=1.5, pos_offset=off)
    call = Q.Rope3DCall(**p)
    odt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    s = torch.cuda.Stream()
    for t in (T, max(1, T // 3), 1):
        ref = run_3d(qkv[:t], qw, kw, **p)
        got = [torch.empty((t, h, D), dtype=odt, device=DEV) for h in (Hq, Hk, Hv)]
        for g in got:
            g.view(torch.uint8).fill_(7)
        call(qkv[:t], qw, kw, *got, stream=s)
        s.synchronize()
        for x, y in zip(ref, got):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), t
    with pytest.raises(Q.QknrValueError):
        call(qkv[:, :-1].contiguous(), qw, kw, *got, stream=s)

def test_3d_batch_shape():
    w = W.WORKLOADS["tiny3d"]
    qkv, qw, kw = _rand3d(64, 4, 4, 4, 64)
    q, k, v = run_3d(qkv.reshape(2, 32, -1), qw, kw, **w.params())
    assert q.shape == (2, 32, 4, 64) and v.shape == (2, 32, 4, 64)
    q2, _, _ = run_3d(qkv, qw, kw, **w.params())
    assert torch.equal(q.reshape(64, 4, 64), q2)


# ----------------------------------------------------------- table variants --
def _rand_table_inputs(T, Hq, Hk, D, R, f32, seed=0, std=1.0, act=torch.bfloat16):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = (torch.randn(T, Hq, D, generator=g) * std).to(act)
    k = (torch.randn(T, Hk, D, generator=g) * std).to(act)
    qw = (1 + 0.1 * torch.randn(D, generator=g)).to(act)
    kw = (1 + 0.1 * torch.randn(D, generator=g)).to(act)
    tbl = W.rope_table_input(T, R, 10000.0, f32, act=act)
    return dict(q=q, k=k, q_weight=qw, k_weight=kw, rope_table=tbl)


CASES_TABLE = [
    # (T, Hq, Hk, D, R, f32, interleaved)
    (37, 3, 5, 128, 96, True, False),
    (37, 3, 5, 128, 64, False, True),
    (20, 2, 1, 256, 256, True, False),
    (20, 2, 1, 256, 248, False, True),
    (50, 4, 4, 16, 16, True, True),
    (50, 4, 4, 48, 32, True, False),     # 3 lanes per head, padded group of 4
    (30, 2, 3, 72, 40, True, True),      # head_dim % 16 != 0: general kernel
    (30, 2, 3, 128, 40, False, False),   # half split with rd % 16 != 0: general kernel
    (30, 2, 3, 2, 2, True, True),        # smallest head
    (30, 3, 0, 64, 64, True, False),     # no K heads
    (40, 3, 0, 72, 40, True, True),      # shared-memory (vector) kernel, no K heads
    (40, 0, 2, 72, 40, True, False),     # shared-memory (vector, half split) kernel, no Q heads
    (40, 2, 3, 128, 36, True, False),    # shared-memory pairwise kernel (rd % 8 != 0)
    (70, 5, 3, 8, 8, True, True),        # vector kernel, head_dim 8: 32 heads per warp step
    (70, 5, 3, 24, 16, False, False),    # vector kernel, half split, 3 chunks per head
    (70, 5, 3, 200, 104, True, True),    # vector kernel, head_dim 200: 25 chunks over 32 lanes
]


@pytest.mark.parametrize("case", CASES_TABLE, ids=[str(i) for i in range(len(CASES_TABLE))])
def test_table_variants(case):
    T, Hq, Hk, D, R, f32, il = case
    inp = _rand_table_inputs(T, Hq, Hk, D, R, f32, seed=D + R, std=2.0)
    g = {k: v.to(DEV) for k, v in inp.items()}
    qo, ko = Q.fused_qk_norm_rope(g["q"], g["k"], g["q_weight"], g["k_weight"], g["rope_table"],
                                  1e-5, rotary_dim=R, interleaved=il)
    torch.cuda.synchronize()
    check_table_against_oracle(inp, qo.cpu(), ko.cpu(), 1e-5, R, il, str(case))


@pytest.mark.parametrize("case", [CASES_TABLE[0], CASES_TABLE[1], CASES_TABLE[6], CASES_TABLE[11]],
                         ids=["fast_hs", "fast_il", "general", "smem_no_q"])
def test_table_prepared_call_matches_wrapper(case):
    """RopeTableCall gives the wrapper's bytes, on dense tensors and on Q/K
    views of one fused [T, Hq + Hk, D] tensor (token stride above the row)."""
    T, Hq, Hk, D, R, f32, il = case
    inp = _rand_table_inputs(T, Hq, Hk, D, R, f32, seed=D + R + 2, std=2.0)
    g = {k: v.to(DEV) for k, v in inp.items()}
    call = Q.RopeTableCall(heads_q=Hq, heads_k=Hk, head_dim=D, eps=1e-5, rotary_dim=R,
                           interleaved=il, table_dtype=g["rope_table"].dtype)
    fused = torch.cat([g["q"], g["k"]], dim=1)
    fused_out = torch.empty_like(fused)
    for q, k, qo, ko in ((g["q"], g["k"], torch.empty_like(g["q"]), torch.empty_like(g["k"])),
                         (fused[:, :Hq], fused[:, Hq:], fused_out[:, :Hq], fused_out[:, Hq:])):
        rq, rk = Q.fused_qk_norm_rope(q, k, g["q_weight"], g["k_weight"], g["rope_table"], 1e-5,
                                      rotary_dim=R, interleaved=il)
        call(q, k, qo, ko, g["q_weight"], g["k_weight"], g["rope_table"])
        torch.cuda.synchronize()
        assert torch.equal(rq.view(torch.int16), qo.contiguous().view(torch.int16))
        assert torch.equal(rk.view(torch.int16), ko.contiguous().view(torch.int16))

@pytest.mark.parametrize("case", CASES_TABLE, ids=[str(i) for i in range(len(CASES_TABLE))])
def test_table_variants_f16(case):
    """The same shapes with IEEE binary16 activations and weights (the table
    float32 or binary16 as the case says)."""
    T, Hq, Hk, D, R, f32, il = case
    inp = _rand_table_inputs(T, Hq, Hk, D, R, f32, seed=D + R + 1, std=2.0, act=torch.float16)
    g = {k: v.to(DEV) for k, v in inp.items()}
    qo, ko = Q.fused_qk_norm_rope(g["q"], g["k"], g["q_weight"], g["k_weight"], g["rope_table"],
                                  1e-5, rotary_dim=R, interleaved=il)
    torch.cuda.synchronize()
    assert qo.dtype == torch.float16 and ko.dtype == torch.float16
    check_table_against_oracle(inp, qo.cpu(), ko.cpu(), 1e-5, R, il, f"f16 {case}")


def test_table_f16_small_and_large_magnitudes():
    """binary16 has a narrow range: rows of 1e-3 and of 3e3 (squares past
    binary16's range, but the sums are fp32) and a weight that sends outputs to
    the subnormals must still match the oracle."""
    T, H, D, R = 48, 3, 128, 128
    for std, wscale in ((1e-3, 1.0), (3e3, 1.0), (1.0, 1e-4)):
        inp = _rand_table_inputs(T, H, H, D, R, False, seed=17, std=std, act=torch.float16)
        inp["q_weight"] = (inp["q_weight"].float() * wscale).half()
        g = {k: v.to(DEV) for k, v in inp.items()}
        qo, ko = Q.fused_qk_norm_rope(g["q"], g["k"], g["q_weight"], g["k_weight"],
                                      g["rope_table"], 1e-6, interleaved=False)
        torch.cuda.synchronize()
        check_table_against_oracle(inp, qo.cpu(), ko.cpu(), 1e-6, R, False,
                                   f"std {std} wscale {wscale}")


@pytest.mark.parametrize("act", [torch.bfloat16, torch.float16], ids=["bf16", "f16"])
def test_table_strided_inplace_and_misaligned(act):
    """q and k as views into a packed QKV buffer (token stride 3*H*D), updated
    in place; then the same with every pointer shifted by one element (general
    kernel); all must match the oracle on dense copies."""
    T, H, D, R = 64, 4, 128, 96
    inp = _rand_table_inputs(T, H, H, D, R, True, seed=5, act=act)
    for shift in (0, 1):
        buf = torch.zeros(T * 3 * H * D + 64, dtype=act, device=DEV)
        packed = buf[shift:shift + T * 3 * H * D].view(T, 3 * H, D)
        packed[:, :H] = inp["q"].to(DEV)
        packed[:, H:2 * H] = inp["k"].to(DEV)
        q, k = packed[:, :H], packed[:, H:2 * H]
        g = {n: inp[n].to(DEV) for n in ("q_weight", "k_weight", "rope_table")}
        Q.fused_qk_norm_rope(q, k, g["q_weight"], g["k_weight"], g["rope_table"], 1e-6,
                             rotary_dim=R, interleaved=False, q_out=q, k_out=k)
        torch.cuda.synchronize()
        check_table_against_oracle(inp, q.cpu(), k.cpu(), 1e-6, R, False, f"shift {shift}")
        assert torch.all(packed[:, 2 * H:] == 0)


@pytest.mark.parametrize("act", [torch.bfloat16, torch.float16], ids=["bf16", "f16"])
@pytest.mark.parametrize("il,R", [(True, 36), (False, 40), (False, 72), (False, 36)])
def test_table_smem_path_strided_inplace(act, il, R):
    """head_dim 72 (not a multiple of 16) with 16-byte aligned rows takes the
    shared-memory kernel: q and k as views into a packed buffer (token stride
    3*H*D), updated in place, over enough tokens that each warp's ring turns
    over several times."""
    T, H, D = 12000, 5, 72  # about 5 items per warp: the rings turn over
    inp = _rand_table_inputs(T, H, H, D, R, True, seed=R, act=act)
    buf = torch.zeros(T * 3 * H * D, dtype=act, device=DEV)
    packed = buf.view(T, 3 * H, D)
    packed[:, :H] = inp["q"].to(DEV)
    packed[:, H:2 * H] = inp["k"].to(DEV)
    q, k = packed[:, :H], packed[:, H:2 * H]
    g = {n: inp[n].to(DEV) for n in ("q_weight", "k_weight", "rope_table")}
    Q.fused_qk_norm_rope(q, k, g["q_weight"], g["k_weight"], g["rope_table"], 1e-6,
                         rotary_dim=R, interleaved=il, q_out=q, k_out=k)
    torch.cuda.synchronize()
    check_table_against_oracle(inp, q.cpu(), k.cpu(), 1e-6, R, il, f"smem {act} {il} {R}")
    assert torch.all(packed[:, 2 * H:] == 0)


def test_table_outputs_written_exactly():
    T, Hq, Hk, D, R = 33, 3, 2, 128, 128
    inp = _rand_table_inputs(T, Hq, Hk, D, R, False, seed=9)
    g = {k: v.to(DEV) for k, v in inp.items()}
    qb = torch.full((T * Hq * D + 512,), -1, dtype=torch.int16, device=DEV)
    kb = torch.full((T * Hk * D + 512,), -1, dtype=torch.int16, device=DEV)
    qo = qb[:T * Hq * D].view(torch.bfloat16).view(T, Hq, D)
    ko = kb[:T * Hk * D].view(torch.bfloat16).view(T, Hk, D)
    Q.fused_qk_norm_rope(g["q"], g["k"], g["q_weight"], g["k_weight"], g["rope_table"], 1e-6,
                         rotary_dim=R, interleaved=True, q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    assert torch.all(qb[T * Hq * D:] == -1) and torch.all(kb[T * Hk * D:] == -1)
    assert not torch.any(qb[:T * Hq * D] == -1) and not torch.any(kb[:T * Hk * D] == -1)


def test_empty_inputs_both_forms():
    """No tokens: both entry points succeed, return empty outputs and launch
    nothing."""
    w = W.WORKLOADS["tiny3d"]
    qkv = torch.empty(0, w.row, dtype=torch.bfloat16, device=DEV)
    qw = torch.ones(w.hq * w.head_dim, dtype=torch.bfloat16, device=DEV)
    kw = torch.ones(w.hk * w.head_dim, dtype=torch.bfloat16, device=DEV)
    q, k, v = run_3d(qkv, qw, kw, **w.params())
    assert q.shape == (0, w.hq, w.head_dim) and k.shape[0] == 0 and v.shape[0] == 0
    for act in (torch.bfloat16, torch.float16):
        x = torch.empty(0, 4, 128, dtype=act, device=DEV)
        wt = torch.ones(128, dtype=act, device=DEV)
        tbl = torch.empty(0, 96, dtype=torch.float32, device=DEV)
        qo, ko = Q.fused_qk_norm_rope(x, x[:, :2], wt, wt, tbl, 1e-6, rotary_dim=96)
        assert qo.shape == (0, 4, 128) and ko.shape == (0, 2, 128)
    torch.cuda.synchronize()


def test_zero_rows_give_zero_outputs():
    """A token whose Q (or one head) is all zeros: r = 1/sqrt(eps) is finite and
    every output of that row is exactly zero, as in the oracle."""
    qkv, qw, kw = _rand3d(24, 3, 3, 2, 128, seed=11)
    qkv[5, :3 * 128] = 0          # token 5: every Q head
    qkv[9, 3 * 128:6 * 128] = 0   # token 9: every K head
    p = dict(ppf=2, pph=3, ppw=4, num_frame_channels=32, num_height_channels=48,
             num_width_channels=48, num_heads_q=3, num_heads_k=3, num_heads_v=2, head_dim=128,
             eps=1e-6)
    q, k, _ = check_3d_case(qkv, qw, kw, **p)
    assert torch.all(q[5].float() == 0) and torch.all(k[9].float() == 0)
    for act in (torch.bfloat16, torch.float16):
        inp = _rand_table_inputs(16, 3, 2, 128, 96, True, seed=12, act=act)
        inp["q"][4, 1] = 0
        inp["k"][7] = 0
        g = {n: t.to(DEV) for n, t in inp.items()}
        qo, ko = Q.fused_qk_norm_rope(g["q"], g["k"], g["q_weight"], g["k_weight"],
                                      g["rope_table"], 1e-6, rotary_dim=96)
        torch.cuda.synchronize()
        check_table_against_oracle(inp, qo.cpu(), ko.cpu(), 1e-6, 96, False, f"zero rows {act}")
        assert torch.all(qo[4, 1].float() == 0) and torch.all(ko[7].float() == 0)


def test_3d_sequence_shards_match_whole_call():
    """Sequence sharding (what each rank of a multi-GPU run does): the token
    shards of sharding.token_shard, each called with its pos_offset, give the
    whole call's outputs bit for bit."""
    from qk_rmsnorm_rope_qknr_b200 import sharding

    w = W.WORKLOADS["video3d"]
    T = 3 * 1000 + 7
    inp = W.make_inputs(w, device="cpu", tokens=T)
    qkv = inp["qkv"].to(DEV)
    qw, kw = inp["q_weight"].to(DEV), inp["k_weight"].to(DEV)
    whole = run_3d(qkv, qw, kw, pos_offset=11, **_p3(w))
    P = w.ppf * w.pph * w.ppw
    for world in (2, 3, 8):
        parts = [[], [], []]
        for rank in range(world):
            s, c = sharding.token_shard(T, world, rank)
            out = run_3d(qkv[s:s + c], qw, kw, pos_offset=sharding.shard_pos_offset(s, 11, P),
                         **_p3(w))
            for lst, o in zip(parts, out):
                lst.append(o)
        for lst, o in zip(parts, whole):
            assert torch.equal(torch.cat(lst), o)


def test_concurrent_host_threads_match_serial():
    """Several host threads calling the entry points at once, each on its own
    stream and with its own shapes (the launch caches and lane plans are shared
    state), give the bits of the same calls made one after another."""
    import threading

    jobs = []
    for i in range(4):
        qkv, qw, kw = _rand3d(48, 2 + i, 2, 1, 64, seed=20 + i)
        p3 = dict(ppf=2, pph=4, ppw=6, num_frame_channels=16, num_height_channels=24,
                  num_width_channels=24, num_heads_q=2 + i, num_heads_k=2, num_heads_v=1,
                  head_dim=64)
        D, R = (128, 96) if i % 2 == 0 else (72, 40)
        t = {n: v.to(DEV) for n, v in _rand_table_inputs(64, 3, 1 + i, D, R, True,
                                                          seed=30 + i).items()}
        wu = W.FormUcpe("u", batch=1, seq=(96, 150, 64, 130)[i], heads=2 + i,
                        head_dim=(112, 64, 128, 48)[i], spatial=16, seed=40 + i)
        u = {n: v.to(DEV) for n, v in W.make_inputs(wu).items()}
        jobs.append((qkv, qw, kw, p3, t, R, bool(i % 2), u, wu.k_scale))

    def run(job, stream):
        qkv, qw, kw, p3, t, R, il, u, ks = job
        outs = []
        for _ in range(10):
            a = run_3d(qkv, qw, kw, stream=stream, **p3)
            b = Q.fused_qk_norm_rope(t["q"], t["k"], t["q_weight"], t["k_weight"], t["rope_table"],
                                     1e-6, rotary_dim=R, interleaved=il, stream=stream)
            c = Q.cam_prep_func(u["q_normed"], u["k_normed"], u["v_raw"], proj_q=u["proj_q"],
                                proj_kv=u["proj_kv"], rope_cos=u["rope_cos"],
                                rope_sin=u["rope_sin"], k_scale=ks, stream=stream)
            outs.append([x.clone() for x in (*a, *b, *c)])
        return outs

    serial = [run(j, torch.cuda.current_stream()) for j in jobs]
    torch.cuda.synchronize()
    results = [None] * len(jobs)
    streams = [torch.cuda.Stream() for _ in jobs]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())

    def worker(i):
        with torch.cuda.stream(streams[i]):
            results[i] = run(jobs[i], streams[i])

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(jobs))]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    torch.cuda.synchronize()
    for i in range(len(jobs)):
        for rep_s, rep_c in zip(serial[i], results[i]):
            for x, y in zip(rep_s, rep_c):
                assert torch.equal(x, y)
