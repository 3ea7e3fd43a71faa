"""Tensor-parallel 3D form: heads split across the ranks of a process group.

Each rank holds packed rows of its own heads, [tokens, (hq+hk+hv)*head_dim],
and the [hq*head_dim] / [hk*head_dim] slices of the norm weights. The
across-heads RMSNorm must still run over all ranks' channels (the SANA-WM UCPE
page, cam_prep_func: a head shard is normalised over the whole channel width,
not its own slice), so one call is
    partial sums of x^2 (this rank's heads)  ->  all-reduce (sum)  ->
    transform with the global sums,
the first and last step in libqknr.so's kernels, the exchange a
torch.distributed all-reduce (NCCL over NVLink on GPUs) of T*8 bytes.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

import qk_rmsnorm_rope_qknr_b200 as Q


def all_reduce_ssq(ssq: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the per-token partial sums of every rank in `group` (in place).
    Without an initialised process group the call is a single rank's."""
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(ssq, op=dist.ReduceOp.SUM, group=group)
    return ssq


def fused_qk_rmsnorm_rope_tp(qkv: torch.Tensor, q_weight: torch.Tensor, k_weight: torch.Tensor,
                             *, heads_q_total: int, heads_k_total: int, group=None,
                             q_out: Optional[torch.Tensor] = None,
                             k_out: Optional[torch.Tensor] = None,
                             v_out: Optional[torch.Tensor] = None, stream=None, **params):
    """This rank's (q, k, v) of the 3D transform of a head-sharded call.

    params are fused_qk_rmsnorm_rope's keyword arguments for THIS rank's slice
    (num_heads_q/k/v = local heads); heads_q_total / heads_k_total count the
    heads of all ranks together. is_qk_norm must be on (without the norm there
    is nothing to exchange: call fused_qk_rmsnorm_rope per rank).
    """
    if not params.get("is_qk_norm", True):
        raise ValueError("the tensor-parallel form exists for the norm; call "
                         "fused_qk_rmsnorm_rope directly with is_qk_norm=False")
    D = params["head_dim"]
    lead = tuple(qkv.shape[:-1])
    T = qkv.numel() // qkv.shape[-1]
    odt = torch.float8_e4m3fn if params.get("output_fp8") else torch.bfloat16
    outs = []
    for o, h in ((q_out, params["num_heads_q"]), (k_out, params["num_heads_k"]),
                 (v_out, params["num_heads_v"])):
        outs.append(o if o is not None else torch.empty(lead + (h, D), dtype=odt,
                                                        device=qkv.device))
    ssq = torch.empty(T, 2, dtype=torch.float32, device=qkv.device)
    Q.qknr_rope_3d_partial_ssq(qkv, ssq, stream=stream, **params)
    # The collective is queued behind the partial sums and ahead of the
    # transform: on the caller's stream when one is given.
    if stream is not None and not isinstance(stream, torch.cuda.Stream):
        stream = torch.cuda.ExternalStream(int(stream), device=qkv.device)
    if stream is not None:
        with torch.cuda.stream(stream):
            all_reduce_ssq(ssq, group)
    else:
        all_reduce_ssq(ssq, group)
    Q.qknr_rope_3d_with_ssq(qkv, q_weight, k_weight, *outs, ssq, heads_q_total=heads_q_total,
                            heads_k_total=heads_k_total, stream=stream, **params)
    return tuple(outs)


def head_slice(total: int, world: int, rank: int):
    """[start, stop) of the heads rank `rank` of `world` holds (contiguous,
    balanced)."""
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)
