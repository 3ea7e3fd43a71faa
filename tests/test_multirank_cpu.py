"""The multi-rank path on CPU: world size 2 over gloo.

Each rank takes its contiguous token shard of one 3D sequence (and of one
table-form batch, and of one camera-prep call), runs the oracle on it with the
shard's pos_offset (or table rows, or rows of every per-token input), and
all_gathers the pieces; the result must equal the unsharded call bit for
bit. This checks the sharding arithmetic with real collectives; on
GPUs the same shards go to qknr_rope_3d / qknr_rope_table on each rank.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from qk_rmsnorm_rope_qknr_b200 import sharding

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs3d(T, row, seed=3):
    g = torch.Generator().manual_seed(seed)
    qkv = torch.randn(T, row, generator=g).to(torch.bfloat16)
    qw = (1 + 0.1 * torch.randn(2 * 32, generator=g)).to(torch.bfloat16)
    kw = (1 + 0.1 * torch.randn(2 * 32, generator=g)).to(torch.bfloat16)
    return qkv, qw, kw


P3 = dict(ppf=3, pph=2, ppw=5, num_frame_channels=8, num_height_channels=12,
          num_width_channels=12, num_heads_q=2, num_heads_k=2, num_heads_v=1, head_dim=32,
          eps=1e-5, interleave=False)


def _worker(rank, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        import oracle as O
        from tests._util import t2u16

        # --- 3D sequence of 2.4 grids, offset into the sequence by 7 tokens
        T, P = 72, 3 * 2 * 5
        qkv, qw, kw = _inputs3d(T, 5 * 32)
        start, count = sharding.token_shard(T, WORLD, rank)
        off = sharding.shard_pos_offset(start, 7, P)
        mine = O.rope_3d(t2u16(qkv[start:start + count]), t2u16(qw), t2u16(kw), pos_offset=off,
                         **P3)
        for part, ref in zip(mine, O.rope_3d(t2u16(qkv), t2u16(qw), t2u16(kw), pos_offset=7,
                                             **P3)):
            pieces = [None] * WORLD
            dist.all_gather_object(pieces, part)
            assert np.array_equal(np.concatenate(pieces), ref)
        # --- table form: 33 tokens, the shard takes its own table rows
        g = torch.Generator().manual_seed(5)
        q = torch.randn(33, 3, 16, generator=g).to(torch.bfloat16)
        k = torch.randn(33, 1, 16, generator=g).to(torch.bfloat16)
        w = (1 + 0.1 * torch.randn(16, generator=g)).to(torch.bfloat16)
        th = torch.arange(33, dtype=torch.float64)[:, None] * 0.3 ** torch.arange(6.0)[None, :]
        tbl = torch.cat([th.cos(), th.sin()], 1).float().numpy()
        s, c = sharding.token_shard(33, WORLD, rank)
        mine = O.rope_table(t2u16(q[s:s + c]), t2u16(k[s:s + c]), t2u16(w), t2u16(w),
                            tbl[s:s + c].copy(), 1e-6, 12, interleaved=True)
        ref = O.rope_table(t2u16(q), t2u16(k), t2u16(w), t2u16(w), tbl, 1e-6, 12,
                           interleaved=True)
        for part, r in zip(mine, ref):
            pieces = [None] * WORLD
            dist.all_gather_object(pieces, part)
            assert np.array_equal(np.concatenate(pieces), r)
        # --- camera prep: 37 tokens of 2 batch elements; the shard takes its
        # rows of q/k/v and of the matrices and tables, and its outputs are the
        # whole call's columns ([B, H, D, N]: the token axis is the last)
        import workloads as W

        wu = W.FormUcpe("mr", batch=2, seq=37, heads=3, head_dim=16, spatial=9, seed=6)
        u = W.make_inputs(wu, device="cpu")
        s, c = sharding.token_shard(37, WORLD, rank)
        sl = slice(s, s + c)

        def cam(inp, rows):
            return O.ucpe_cam_prep(t2u16(inp["q_normed"][:, rows]), t2u16(inp["k_normed"][:, rows]),
                                   t2u16(inp["v_raw"][:, rows]), inp["proj_q"][:, rows].numpy(),
                                   inp["proj_kv"][:, rows].numpy(), inp["rope_cos"][rows].numpy(),
                                   inp["rope_sin"][rows].numpy(), wu.k_scale)

        mine, ref = cam(u, sl), cam(u, slice(0, 37))
        for part, r in zip(mine, ref):
            pieces = [None] * WORLD
            dist.all_gather_object(pieces, part)
            assert np.array_equal(np.concatenate(pieces, axis=-1), r)
        dist.barrier()
        open(os.path.join(out_dir, f"ok{rank}"), "w").write("ok")
    finally:
        dist.destroy_process_group()


def _tp_worker(rank, port, out_dir):
    """Head-sharded (tensor-parallel) exchange: each rank sums x^2 over its own
    heads, tp.all_reduce_ssq adds the ranks' sums, and the rank's heads,
    normalised with the global sums and rotated with the oracle's own steps,
    equal the oracle's unsplit call."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        import oracle as O
        from qk_rmsnorm_rope_qknr_b200 import tp
        from tests._util import t2u16

        D, Hq, Hk, Hv, T, eps = 32, 3, 2, 1, 30, 1e-5
        g = torch.Generator().manual_seed(11)
        qkv = torch.randn(T, (Hq + Hk + Hv) * D, generator=g).to(torch.bfloat16)
        qw = (1 + 0.1 * torch.randn(Hq * D, generator=g)).to(torch.bfloat16)
        kw = (1 + 0.1 * torch.randn(Hk * D, generator=g)).to(torch.bfloat16)
        p = dict(P3, num_heads_q=Hq, num_heads_k=Hk, num_heads_v=Hv, eps=eps)
        full_q, full_k, _ = O.rope_3d(t2u16(qkv), t2u16(qw), t2u16(kw), exact=True, **p)
        sq, sk = tp.head_slice(Hq, WORLD, rank), tp.head_slice(Hk, WORLD, rank)
        x = qkv.double()
        xq = x[:, sq[0] * D:sq[1] * D]
        xk = x[:, (Hq + sk[0]) * D:(Hq + sk[1]) * D]
        ssq = torch.stack([xq.pow(2).sum(1), xk.pow(2).sum(1)], 1).float()
        tp.all_reduce_ssq(ssq)
        want = torch.stack([x[:, :Hq * D].pow(2).sum(1), x[:, Hq * D:(Hq + Hk) * D].pow(2).sum(1)],
                           1)
        assert torch.allclose(ssq.double(), want, rtol=1e-6)
        pa, pb = O.pairs_3d(8, 12, 12, False)
        for X, xs, sl, w, tot, col, full in ((0, xq, sq, qw, Hq, 0, full_q),
                                             (1, xk, sk, kw, Hk, 1, full_k)):
            r = 1.0 / np.sqrt(ssq[:, col].double().numpy() / (tot * D) + eps)
            wv = O.bf16_to_f64(t2u16(w))[sl[0] * D:sl[1] * D]
            for t in range(T):
                th = O.angles_3d(*O.position_3d(t, 0, 3, 2, 5), 8, 12, 12, 10000.0)
                y = xs[t].numpy() * r[t] * wv
                for hh in range(sl[1] - sl[0]):
                    out = O.rotate(y[hh * D:(hh + 1) * D], pa, pb, np.cos(th), np.sin(th))
                    assert np.allclose(out, full[t, sl[0] + hh], rtol=0, atol=1e-5), (X, t, hh)
        dist.barrier()
        open(os.path.join(out_dir, f"tp{rank}"), "w").write("ok")
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_exchange_over_gloo(tmp_path):
    port = _free_port()
    mp.start_processes(_tp_worker, args=(port, str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    for r in range(WORLD):
        assert (tmp_path / f"tp{r}").read_text() == "ok"


def test_token_shard_arithmetic():
    for T in (0, 1, 5, 72, 15360, 59521):
        for world in (1, 2, 3, 8):
            spans = [sharding.token_shard(T, world, r) for r in range(world)]
            assert spans[0][0] == 0
            assert sum(c for _, c in spans) == T
            for (s0, c0), (s1, _) in zip(spans, spans[1:]):
                assert s0 + c0 == s1
            assert max(c for _, c in spans) - min(c for _, c in spans) <= 1
    assert sharding.shard_pos_offset(40, 7, 30) == 17
    with pytest.raises(ValueError):
        sharding.token_shard(4, 2, 2)


def test_two_ranks_over_gloo(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(port, str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    for r in range(WORLD):
        assert (tmp_path / f"ok{r}").read_text() == "ok"
