"""Tensor-parallel 3D form on one GPU: the heads of a call split over R
simulated ranks (their slices run one after another on the same device; the
all-reduce is a sum of their partial-sum arrays), and through tp.py with a
real NCCL process group of one rank. Outputs must match the fp64 oracle of
the unsplit call within the usual tolerance."""
import os
import socket

import numpy as np
import pytest
import torch

import qk_rmsnorm_rope_qknr_b200 as Q
from qk_rmsnorm_rope_qknr_b200 import tp
import workloads as W
from tests.test_gpu_parity import assert_3d_close, oracle_3d

pytestmark = pytest.mark.gpu


def _slice_cols(qkv, heads, D, sl):
    """Columns of heads [sl) of one tensor kind at head offset `heads`."""
    return qkv[:, (heads + sl[0]) * D:(heads + sl[1]) * D]


def _run_simulated(w, T, R, pos_offset=None, per_axis=False):
    inp = W.make_inputs(w, device="cpu", tokens=T)
    qkv, qw, kw = inp["qkv"], inp["q_weight"], inp["k_weight"]
    D = w.head_dim
    p = dict(w.params())
    if pos_offset is not None:
        p["pos_offset"] = pos_offset
    if per_axis:
        p["neox_per_axis"] = True
    slices = [(tp.head_slice(w.hq, R, r), tp.head_slice(w.hk, R, r), tp.head_slice(w.hv, R, r))
              for r in range(R)]
    locals_ = []
    for sq, sk, sv in slices:
        cols = torch.cat([_slice_cols(qkv, 0, D, sq), _slice_cols(qkv, w.hq, D, sk),
                          _slice_cols(qkv, w.hq + w.hk, D, sv)], dim=1).contiguous().cuda()
        lp = dict(p, num_heads_q=sq[1] - sq[0], num_heads_k=sk[1] - sk[0],
                  num_heads_v=sv[1] - sv[0])
        locals_.append((cols, qw[sq[0] * D:sq[1] * D].contiguous().cuda(),
                        kw[sk[0] * D:sk[1] * D].contiguous().cuda(), lp))
    total = torch.zeros(T, 2, dtype=torch.float32, device="cuda")
    for cols, _, _, lp in locals_:
        part = torch.empty(T, 2, dtype=torch.float32, device="cuda")
        Q.qknr_rope_3d_partial_ssq(cols, part, **lp)
        total += part
    odt = torch.float8_e4m3fn if w.output_fp8 else torch.bfloat16
    pieces = [[], [], []]
    for cols, lqw, lkw, lp in locals_:
        outs = [torch.empty(T, h, D, dtype=odt, device="cuda")
                for h in (lp["num_heads_q"], lp["num_heads_k"], lp["num_heads_v"])]
        Q.qknr_rope_3d_with_ssq(cols, lqw, lkw, *outs, total, heads_q_total=w.hq,
                                heads_k_total=w.hk, **lp)
        for lst, o in zip(pieces, outs):
            lst.append(o)
    torch.cuda.synchronize()
    got = [torch.cat(lst, dim=1) for lst in pieces]
    ref, exact = oracle_3d(qkv, qw, kw, **p)
    assert_3d_close(got, ref, exact, w.output_fp8, f"{w.name} TP={R}")
    return total, qkv


@pytest.mark.parametrize("name", ["video3d", "fp8neox", "gqa3d"])
@pytest.mark.parametrize("R", [1, 2, 3, 4])
def test_tp_simulated_matches_oracle(name, R):
    w = W.WORKLOADS[name]
    total, qkv = _run_simulated(w, 1201, R, pos_offset=333)
    # the summed partials are the whole row's sums
    x = qkv.float()
    want_q = x[:, :w.hq * w.head_dim].pow(2).sum(1)
    want_k = x[:, w.hq * w.head_dim:(w.hq + w.hk) * w.head_dim].pow(2).sum(1)
    np.testing.assert_allclose(total[:, 0].cpu().numpy(), want_q.numpy(), rtol=1e-5)
    np.testing.assert_allclose(total[:, 1].cpu().numpy(), want_k.numpy(), rtol=1e-5)


@pytest.mark.parametrize("R", [1, 3])
def test_tp_simulated_neox_per_axis(R):
    """The per-axis NeoX layout through the two tensor-parallel passes."""
    _run_simulated(W.WORKLOADS["fp8neox"], 1201, R, pos_offset=333, per_axis=True)


def test_tp_one_rank_nccl_group():
    import torch.distributed as dist

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda:0"))
    try:
        w = W.WORKLOADS["video3d"]
        inp = {k: v.cuda() for k, v in W.make_inputs(w, tokens=960).items()}
        p = dict(w.params(), pos_offset=0)
        q, k, v = tp.fused_qk_rmsnorm_rope_tp(inp["qkv"], inp["q_weight"], inp["k_weight"],
                                              heads_q_total=w.hq, heads_k_total=w.hk, **p)
        torch.cuda.synchronize()
        ref, exact = oracle_3d(inp["qkv"].cpu(), inp["q_weight"].cpu(), inp["k_weight"].cpu(), **p)
        assert_3d_close([q, k, v], ref, exact, False, "tp world 1")
        # on a side stream: the exchange is ordered between the two kernels there
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        q2, k2, v2 = tp.fused_qk_rmsnorm_rope_tp(inp["qkv"], inp["q_weight"], inp["k_weight"],
                                                 heads_q_total=w.hq, heads_k_total=w.hk,
                                                 stream=side, **p)
        side.synchronize()
        assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    finally:
        dist.destroy_process_group()
