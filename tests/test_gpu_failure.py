"""Failure detection on the GPU without faulting it.

The pipelined 3D and table kernels bound every wait on their own bulk copies,
and the camera prep's warp-specialised kernel every wait on its copy warp and
on its compute warps. The test
hook makes each ring buffer expect 16 bytes more than its copy delivers (a
count that nothing completes), with a 20 ms limit: the waits run out, the
launch abandons its tokens, raises bit 0 of the device status word, drains its
copies and ends. The context must stay usable: a normal call right after
gives correct results.
"""
import pytest
import torch

import qk_rmsnorm_rope_qknr_b200 as Q
import workloads as W

pytestmark = pytest.mark.gpu


def _tiny():
    w = W.WORKLOADS["tiny3d"]
    inp = {k: v.cuda() for k, v in W.make_inputs(w).items()}
    return w, inp


def test_device_status_clean_after_normal_runs():
    w, inp = _tiny()
    Q.qknr_device_status(clear=True)
    for _ in range(3):
        Q.fused_qk_rmsnorm_rope(inp["qkv"], inp["q_weight"], inp["k_weight"], **w.params())
    assert Q.qknr_device_status() == 0


def test_wait_timeout_raises_status_and_context_survives():
    w, inp = _tiny()
    good = Q.fused_qk_rmsnorm_rope(inp["qkv"], inp["q_weight"], inp["k_weight"], **w.params())
    torch.cuda.synchronize()
    Q.qknr_device_status(clear=True)
    L = Q.lib()
    assert L.qknr_test_set_wait_fault(16, 20_000_000) == 0
    try:
        outs = [torch.zeros_like(o) for o in good]
        Q.qknr_rope_3d(inp["qkv"], inp["q_weight"], inp["k_weight"], *outs, **w.params())
        torch.cuda.synchronize()
    finally:
        assert L.qknr_test_set_wait_fault(0, 0) == 0
    assert Q.qknr_device_status(clear=True) & 1
    assert Q.qknr_device_status() == 0
    again = Q.fused_qk_rmsnorm_rope(inp["qkv"], inp["q_weight"], inp["k_weight"], **w.params())
    torch.cuda.synchronize()
    for a, b in zip(good, again):
        assert torch.equal(a, b)
    assert Q.qknr_device_status() == 0


def _table_inputs(shape):
    if shape == "table_hs":  # the fast (register) kernel
        w = W.WORKLOADS["table_hs"]
        inp = {k: v.cuda() for k, v in W.make_inputs(w, tokens=64).items()}
        return inp, w.rotary_dim, w.interleaved
    # head_dim 72, rotary_dim 40: the shared-memory kernel
    g = torch.Generator(device="cpu").manual_seed(3)
    inp = dict(q=torch.randn(64, 6, 72, generator=g), k=torch.randn(64, 2, 72, generator=g),
               q_weight=torch.ones(72), k_weight=torch.ones(72))
    inp = {k: v.to(torch.bfloat16).cuda() for k, v in inp.items()}
    inp["rope_table"] = W.rope_table_input(64, 40, 10000.0, True, "cuda")
    return inp, 40, True


@pytest.mark.parametrize("shape", ["table_hs", "d72_r40"])
def test_table_wait_timeout_raises_status_and_context_survives(shape):
    inp, R, il = _table_inputs(shape)

    def call(qo, ko):
        Q.qknr_rope_table(inp["q"], inp["k"], qo, ko, inp["q_weight"], inp["k_weight"],
                          inp["rope_table"], eps=1e-6, rotary_dim=R, interleaved=il)

    good = [torch.empty_like(inp["q"]), torch.empty_like(inp["k"])]
    call(*good)
    torch.cuda.synchronize()
    Q.qknr_device_status(clear=True)
    L = Q.lib()
    assert L.qknr_test_set_wait_fault(16, 20_000_000) == 0
    try:
        call(torch.zeros_like(inp["q"]), torch.zeros_like(inp["k"]))
        torch.cuda.synchronize()
    finally:
        assert L.qknr_test_set_wait_fault(0, 0) == 0
    assert Q.qknr_device_status(clear=True) & 1
    again = [torch.empty_like(inp["q"]), torch.empty_like(inp["k"])]
    call(*again)
    torch.cuda.synchronize()
    for a, b in zip(good, again):
        assert torch.equal(a, b)
    assert Q.qknr_device_status() == 0


@pytest.mark.parametrize("N", [128, 136], ids=["direct_stores", "staged_stores"])
def test_ucpe_wait_timeout_raises_status_and_context_survives(N):
    """The camera prep's warp-specialised kernel: its compute warps wait on the copy
    warp's ring stages and the copy warp on them, every wait bounded. With the
    hook, the stages never fill: the waits run out, the launch abandons its
    steps, raises bit 0, waits (bounded) for the copies it issued and ends.
    N = 136 (8 mod 16) takes the staged-store form, whose warps leave together."""
    B, H, D = 1, 3, 112
    w = W.FormUcpe("case", batch=B, seq=N, heads=H, head_dim=D, spatial=N // 4, seed=6)
    inp = W.make_inputs(w, device="cuda")
    args = [inp[k] for k in ("q_normed", "k_normed", "v_raw", "proj_q", "proj_kv", "rope_cos",
                             "rope_sin")]

    def call():
        outs = [torch.empty(B, H, D, N, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
        infl = torch.empty(B, H, N, device="cuda")
        Q.qknr_ucpe_cam_prep(*args, *outs, infl, k_scale=w.k_scale)
        return outs + [infl]

    good = call()
    torch.cuda.synchronize()
    Q.qknr_device_status(clear=True)
    L = Q.lib()
    assert L.qknr_test_set_wait_fault(16, 20_000_000) == 0
    try:
        call()
        torch.cuda.synchronize()
    finally:
        assert L.qknr_test_set_wait_fault(0, 0) == 0
    assert Q.qknr_device_status(clear=True) & 1
    again = call()
    torch.cuda.synchronize()
    for a, b in zip(good, again):
        assert torch.equal(a, b)
    assert Q.qknr_device_status() == 0
