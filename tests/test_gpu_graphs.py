"""Every entry point can be captured in a CUDA graph and replayed: the library
neither allocates nor synchronises, and its host-side checks are not stream
work. Replays must match eager calls bit for bit, also after the inputs change
in place."""
import pytest
import torch

import qk_rmsnorm_rope_qknr_b200 as Q
import workloads as W

pytestmark = pytest.mark.gpu


def test_3d_graph_replay():
    w = W.WORKLOADS["fp8neox"]
    inp = {k: v.cuda() for k, v in W.make_inputs(w, tokens=2 * 2976).items()}
    p = dict(w.params(), pos_offset=0)
    outs = [torch.empty(2 * 2976, h, w.head_dim, dtype=torch.float8_e4m3fn, device="cuda")
            for h in (w.hq, w.hk, w.hv)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        Q.qknr_rope_3d(inp["qkv"], inp["q_weight"], inp["k_weight"], *outs, stream=s, **p)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        Q.qknr_rope_3d(inp["qkv"], inp["q_weight"], inp["k_weight"], *outs, stream=s, **p)
    for trial in range(2):
        inp["qkv"].mul_(-1.5 if trial else 1.0)
        eager = [torch.empty_like(o) for o in outs]
        Q.qknr_rope_3d(inp["qkv"], inp["q_weight"], inp["k_weight"], *eager, **p)
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(eager, outs):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def test_table_graph_replay():
    w = W.WORKLOADS["table_hs"]
    inp = {k: v.cuda() for k, v in W.make_inputs(w, tokens=512).items()}
    qo, ko = torch.empty_like(inp["q"]), torch.empty_like(inp["k"])
    s = torch.cuda.Stream()

    def call(q_out, k_out, stream=None):
        Q.qknr_rope_table(inp["q"], inp["k"], q_out, k_out, inp["q_weight"], inp["k_weight"],
                          inp["rope_table"], eps=w.eps, rotary_dim=w.rotary_dim,
                          interleaved=w.interleaved, stream=stream)

    with torch.cuda.stream(s):
        call(qo, ko, s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call(qo, ko, s)
    inp["q"].mul_(2.0)
    eq, ek = torch.empty_like(qo), torch.empty_like(ko)
    call(eq, ek)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(eq, qo) and torch.equal(ek, ko)


@pytest.mark.parametrize("N", [192, 151])  # pipelined kernel, general kernel
def test_ucpe_graph_replay(N):
    w = W.FormUcpe("g", batch=1, seq=N, heads=4, head_dim=112, spatial=N // 4)
    inp = {k: v.cuda() for k, v in W.make_inputs(w).items()}
    names = ("q_normed", "k_normed", "v_raw", "proj_q", "proj_kv", "rope_cos", "rope_sin")
    outs = [torch.empty(1, 4, 112, N, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    infl = torch.empty(1, 4, N, device="cuda")
    s = torch.cuda.Stream()

    def call(o, f, stream=None):
        Q.qknr_ucpe_cam_prep(*(inp[n] for n in names), *o, f, k_scale=w.k_scale, stream=stream)

    with torch.cuda.stream(s):
        call(outs, infl, s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call(outs, infl, s)
    inp["k_normed"].mul_(-0.5)
    inp["proj_kv"].mul_(2.0)
    eager = [torch.empty_like(o) for o in outs]
    einfl = torch.empty_like(infl)
    call(eager, einfl)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager + [einfl], outs + [infl]):
        assert torch.equal(a, b)
