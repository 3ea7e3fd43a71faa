"""Inputs beyond 4 GiB: tokens whose rows start past byte 2^32 of the input
(and past element 2^31) must come out right; sampled tokens are checked one by
one against the oracle. About 9 GB of device memory per case."""
import numpy as np
import pytest
import torch

import qk_rmsnorm_rope_qknr_b200 as Q
import workloads as W
from tests._util import bf16_mismatch, t2u16
from tests.test_gpu_parity import assert_3d_close, check_table_against_oracle, oracle_3d

pytestmark = pytest.mark.gpu


def test_3d_rows_past_4_gib():
    w = W.WORKLOADS["video3d"]
    T = 184320  # 12 grids of 15360 tokens: 4.53 GB of input
    g = torch.Generator(device="cuda").manual_seed(21)
    qkv = torch.randn(T, w.row, generator=g, device="cuda").to(torch.bfloat16)
    qw = (1 + 0.1 * torch.randn(w.hq * w.head_dim, generator=g, device="cuda")).to(torch.bfloat16)
    kw = (1 + 0.1 * torch.randn(w.hk * w.head_dim, generator=g, device="cuda")).to(torch.bfloat16)
    assert qkv.numel() * 2 > 2 ** 32
    outs = Q.fused_qk_rmsnorm_rope(qkv, qw, kw, **w.params())
    torch.cuda.synchronize()
    first_far = (2 ** 32) // (w.row * 2) + 1
    picks = [0, first_far - 1, first_far, first_far + 1, T // 2, T - 2, T - 1]
    picks += np.random.default_rng(3).integers(first_far, T, 8).tolist()
    qw_c, kw_c = qw.cpu(), kw.cpu()
    for t in picks:
        ref, exact = oracle_3d(qkv[t:t + 1].cpu(), qw_c, kw_c, pos_offset=t, **w.params())
        got = [o[t:t + 1] for o in outs]
        assert_3d_close(got, ref, exact, False, f"token {t}")
    del qkv, outs
    torch.cuda.empty_cache()


def test_table_past_2g_elements():
    w = W.WORKLOADS["table_il"]
    T = 2048 * 48  # q: 98304 x 24 x 128 bf16 = 302 M elements; strided view below
    g = torch.Generator(device="cuda").manual_seed(5)
    # q as a strided view into a packed buffer so the last token starts past element 2^31
    packed = torch.randn(T, 3 * 24 * 128 * 3, generator=g, device="cuda").to(torch.bfloat16)
    q = packed[:, :24 * 128].view(T, 24, 128)
    k = packed[:, 24 * 128:48 * 128].view(T, 24, 128)
    assert (T - 1) * packed.stride(0) > 2 ** 31
    wq = (1 + 0.1 * torch.randn(128, generator=g, device="cuda")).to(torch.bfloat16)
    wk = (1 + 0.1 * torch.randn(128, generator=g, device="cuda")).to(torch.bfloat16)
    tbl = W.rope_table_input(T, 128, 10000.0, False, "cuda")
    qo, ko = Q.fused_qk_norm_rope(q, k, wq, wk, tbl, 1e-6, rotary_dim=128, interleaved=True)
    torch.cuda.synchronize()
    for t in [0, T // 2, T - 3, T - 1] + np.random.default_rng(4).integers(0, T, 6).tolist():
        inp = dict(q=q[t:t + 1].cpu().contiguous(), k=k[t:t + 1].cpu().contiguous(),
                   q_weight=wq.cpu(), k_weight=wk.cpu(), rope_table=tbl[t:t + 1].cpu())
        check_table_against_oracle(inp, qo[t:t + 1].cpu(), ko[t:t + 1].cpu(), 1e-6, 128, True,
                                   f"token {t}")
    _ = bf16_mismatch, t2u16
