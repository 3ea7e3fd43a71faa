"""Seeded synthetic inputs for the fused Q/K RMSNorm + RoPE workloads and the
UCPE camera prep.

This module only draws inputs (and counts their bytes); it holds none of the
transform's arithmetic, and both the CUDA path and the oracle consume the very
tensors it returns. Draw order per workload: qkv (or q then k), q_weight,
k_weight, then the outlier mask; every draw uses one torch.Generator seeded
with the workload's seed, on the device the caller names (so inputs drawn on
"cpu" and on "cuda" differ; a test always feeds one tensor to both sides).

Workloads (shapes from the two API pages' parameter lists, sizes from the
video-DiT and MiniMax-H3 geometries the pages name):
  tiny3d      3D form, 32 tokens, 4+4+4 heads of 64, grid 2x4x4, 16/24/24
  table_hs    table form, half-split, q [4096,32,128], k [4096,8,128], rd 96, fp32 table
  table_il    table form, adjacent pairs, q,k [2048,24,128] (x3, 1% outliers x20),
              rd 128, bf16 table
  table_hs_f16  table_hs with IEEE binary16 activations, weights and table
  table_d72   table form, adjacent pairs, head_dim 72 (off the register fast path:
              the shared-memory kernel), q [4096,32,72], k [4096,8,72], rd 72
  video3d     3D form, [1,15360,(32+32+32)*128], grid 16x30x32, 16/56/56, bf16 out
  fp8neox     3D form, [2,29760,(24+24+24)*128] ~N(0, 2^2), grid 31x24x40,
              32/48/48, NeoX pairs, E4M3 out (scales 0.5 / 0.25)
  fp8neox_nonorm  fp8neox with is_qk_norm=False
  gqa3d       video3d's geometry with grouped-query heads 32+8+8 (parity and TP case)
  ucpe        UCPE camera prep: camera Q, K, V [1, 18480, 20, 112] ~N(0,1) (the SANA-WM
              page's 18480-token ray grid, taken as 21 latent frames of 22x40 tokens;
              20 heads of 112, a 2240-wide model, are not on the page), per-token rigid
              motions G as proj_q = G^T and proj_kv = G^-1, cos/sin of
              n * 10000^(-2j/112), k_scale = 112^-0.5 * 880^-0.5
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Form3D:
    name: str
    batch: int
    seq: int
    ppf: int
    pph: int
    ppw: int
    cf: int
    ch: int
    cw: int
    hq: int
    hk: int
    hv: int
    head_dim: int
    eps: float = 1e-6
    base: float = 10000.0
    interleave: bool = True
    is_qk_norm: bool = True
    output_fp8: bool = False
    q_scale: float = 1.0
    v_scale: float = 1.0
    std: float = 1.0
    seed: int = 0
    input_2d: bool = False
    form: str = "3d"

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    @property
    def row(self) -> int:
        return (self.hq + self.hk + self.hv) * self.head_dim

    def params(self) -> dict:
        """Keyword arguments of the 3D entry point (the page's names)."""
        return dict(ppf=self.ppf, pph=self.pph, ppw=self.ppw, num_frame_channels=self.cf,
                    num_height_channels=self.ch, num_width_channels=self.cw,
                    num_heads_q=self.hq, num_heads_k=self.hk, num_heads_v=self.hv,
                    head_dim=self.head_dim, eps=self.eps, base=self.base,
                    interleave=self.interleave, is_qk_norm=self.is_qk_norm,
                    output_fp8=self.output_fp8, output_quant_scale=self.q_scale,
                    v_quant_scale=self.v_scale)


@dataclasses.dataclass(frozen=True)
class FormTable:
    name: str
    tokens: int
    hq: int
    hk: int
    head_dim: int
    rotary_dim: int
    table_f32: bool
    interleaved: bool
    eps: float = 1e-6
    std: float = 1.0
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    rope_base: float = 10000.0
    seed: int = 0
    act: str = "bf16"  # activation (and 16-bit table) type: "bf16" or "f16"
    form: str = "table"

    @property
    def act_dtype(self) -> torch.dtype:
        return torch.float16 if self.act == "f16" else torch.bfloat16


@dataclasses.dataclass(frozen=True)
class FormUcpe:
    name: str
    batch: int
    seq: int       # tokens N of the ray grid (latent frames x spatial tokens)
    heads: int
    head_dim: int
    spatial: int   # tokens per latent frame (the spatial_tokens of k_scale)
    rope_base: float = 10000.0
    std: float = 1.0
    translation_std: float = 0.5
    seed: int = 0
    act: str = "bf16"
    form: str = "ucpe"

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    @property
    def k_scale(self) -> float:
        return self.head_dim ** -0.5 * self.spatial ** -0.5

    @property
    def act_dtype(self) -> torch.dtype:
        return torch.float16 if self.act == "f16" else torch.bfloat16


WORKLOADS = {
    "tiny3d": Form3D("tiny3d", batch=1, seq=32, ppf=2, pph=4, ppw=4, cf=16, ch=24, cw=24, hq=4,
                     hk=4, hv=4, head_dim=64, input_2d=True),
    "table_hs": FormTable("table_hs", tokens=4096, hq=32, hk=8, head_dim=128, rotary_dim=96,
                          table_f32=True, interleaved=False),
    "table_il": FormTable("table_il", tokens=2048, hq=24, hk=24, head_dim=128, rotary_dim=128,
                          table_f32=False, interleaved=True, std=3.0, outlier_frac=0.01,
                          outlier_mult=20.0),
    "table_hs_f16": FormTable("table_hs_f16", tokens=4096, hq=32, hk=8, head_dim=128,
                              rotary_dim=96, table_f32=False, interleaved=False, act="f16"),
    "table_d72": FormTable("table_d72", tokens=4096, hq=32, hk=8, head_dim=72, rotary_dim=72,
                           table_f32=True, interleaved=True),
    "video3d": Form3D("video3d", batch=1, seq=15360, ppf=16, pph=30, ppw=32, cf=16, ch=56,
                      cw=56, hq=32, hk=32, hv=32, head_dim=128),
    "fp8neox": Form3D("fp8neox", batch=2, seq=29760, ppf=31, pph=24, ppw=40, cf=32, ch=48,
                      cw=48, hq=24, hk=24, hv=24, head_dim=128, interleave=False,
                      output_fp8=True, q_scale=0.5, v_scale=0.25, std=2.0),
    "gqa3d": Form3D("gqa3d", batch=1, seq=15360, ppf=16, pph=30, ppw=32, cf=16, ch=56, cw=56,
                    hq=32, hk=8, hv=8, head_dim=128),
    "fp8neox_nonorm": Form3D("fp8neox_nonorm", batch=2, seq=29760, ppf=31, pph=24, ppw=40,
                             cf=32, ch=48, cw=48, hq=24, hk=24, hv=24, head_dim=128,
                             interleave=False, is_qk_norm=False, output_fp8=True, q_scale=0.5,
                             v_scale=0.25, std=2.0),
    "ucpe": FormUcpe("ucpe", batch=1, seq=18480, heads=20, head_dim=112, spatial=880),
}


def _normal(g: torch.Generator, shape, std: float, device,
            dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    return (x * std).to(dtype) if std != 1.0 else x.to(dtype)


def _weight(g: torch.Generator, n: int, device, dtype: torch.dtype = torch.bfloat16
            ) -> torch.Tensor:
    w = torch.randn(n, generator=g, dtype=torch.float32, device=device)
    return (1.0 + 0.1 * w).to(dtype)


def rope_table_input(tokens: int, rotary_dim: int, base: float, f32: bool,
                     device="cpu", act: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """A caller-built [tokens, rotary_dim] table [cos(theta) | sin(theta)] with
    theta[t, i] = t * base^(-2i/rotary_dim), built in float64 and stored as
    float32 or as the activation dtype `act` (the input the table form
    consumes)."""
    half = rotary_dim // 2
    pos = torch.arange(tokens, dtype=torch.float64).unsqueeze(1)
    inv = base ** (-2.0 * torch.arange(half, dtype=torch.float64) / rotary_dim)
    theta = pos * inv.unsqueeze(0)
    tbl = torch.cat([torch.cos(theta), torch.sin(theta)], dim=1)
    return tbl.to(torch.float32 if f32 else act).to(device)


def camera_matrices(g: torch.Generator, batch: int, tokens: int, translation_std: float,
                    device="cpu"):
    """Per-token rigid motions G = [[R, t], [0, 1]]: R the rotation of a random
    unit quaternion (a normalised Gaussian 4-vector, so R is uniform over the
    rotations), t ~ N(0, translation_std^2). Returns (G^T, G^-1) as float32
    [batch, tokens, 4, 4]: the Q and K/V matrices of a camera pair whose
    relative motion the attention sees (inputs only: the camera prep multiplies
    by whatever it is given)."""
    qv = torch.randn((batch, tokens, 4), generator=g, dtype=torch.float64, device=device)
    qv = qv / qv.norm(dim=-1, keepdim=True)
    w, x, y, z = qv.unbind(-1)
    rot = torch.stack([
        torch.stack([1 - 2 * (y * y + z * z), 2 * (x * y - z * w), 2 * (x * z + y * w)], -1),
        torch.stack([2 * (x * y + z * w), 1 - 2 * (x * x + z * z), 2 * (y * z - x * w)], -1),
        torch.stack([2 * (x * z - y * w), 2 * (y * z + x * w), 1 - 2 * (x * x + y * y)], -1),
    ], -2)
    t = torch.randn((batch, tokens, 3), generator=g, dtype=torch.float64, device=device)
    t = t * translation_std
    G = torch.zeros((batch, tokens, 4, 4), dtype=torch.float64, device=device)
    G[..., :3, :3] = rot
    G[..., :3, 3] = t
    G[..., 3, 3] = 1.0
    inv = torch.zeros_like(G)
    inv[..., :3, :3] = rot.transpose(-1, -2)
    inv[..., :3, 3] = -(rot.transpose(-1, -2) @ t.unsqueeze(-1)).squeeze(-1)
    inv[..., 3, 3] = 1.0
    return G.transpose(-1, -2).contiguous().float(), inv.float()


def ucpe_rope_tables(tokens: int, head_dim: int, base: float, device="cpu"):
    """cos and sin [tokens, head_dim/2] of theta[n, j] = n * base^(-2j/head_dim),
    built in float64 and stored as float32 (the tables the camera prep reads)."""
    pos = torch.arange(tokens, dtype=torch.float64).unsqueeze(1)
    inv = base ** (-2.0 * torch.arange(head_dim // 2, dtype=torch.float64) / head_dim)
    theta = pos * inv.unsqueeze(0)
    return torch.cos(theta).float().to(device), torch.sin(theta).float().to(device)


def make_inputs(w, device="cpu", tokens: Optional[int] = None, seed: Optional[int] = None):
    """Inputs of workload `w` (a Form3D / FormTable or its name) on `device`.

    tokens overrides the token count (3D: a 2D [tokens, row] input; it must stay
    a multiple of ppf*pph*ppw for the 3D form's own rule) for smaller cases.
    Returns a dict of tensors.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    if w.form == "ucpe":
        N = w.seq if tokens is None else tokens
        shape = (w.batch, N, w.heads, w.head_dim)
        q, k, v = (_normal(g, shape, w.std, device, w.act_dtype) for _ in range(3))
        pq, pkv = camera_matrices(g, w.batch, N, w.translation_std, device)
        cos_t, sin_t = ucpe_rope_tables(N, w.head_dim, w.rope_base, device)
        return dict(q_normed=q, k_normed=k, v_raw=v, proj_q=pq, proj_kv=pkv, rope_cos=cos_t,
                    rope_sin=sin_t)
    if w.form == "3d":
        if tokens is None:
            shape = (w.seq, w.row) if w.input_2d else (w.batch, w.seq, w.row)
        else:
            shape = (tokens, w.row)
        qkv = _normal(g, shape, w.std, device)
        qw = _weight(g, w.hq * w.head_dim, device)
        kw = _weight(g, w.hk * w.head_dim, device)
        return dict(qkv=qkv, q_weight=qw, k_weight=kw)
    T = w.tokens if tokens is None else tokens
    act = w.act_dtype
    q = _normal(g, (T, w.hq, w.head_dim), w.std, device, act)
    k = _normal(g, (T, w.hk, w.head_dim), w.std, device, act)
    qw = _weight(g, w.head_dim, device, act)
    kw = _weight(g, w.head_dim, device, act)
    if w.outlier_frac > 0:
        mq = torch.rand(q.shape, generator=g, device=device) < w.outlier_frac
        mk = torch.rand(k.shape, generator=g, device=device) < w.outlier_frac
        q = torch.where(mq, (q.float() * w.outlier_mult).to(act), q)
        k = torch.where(mk, (k.float() * w.outlier_mult).to(act), k)
    table = rope_table_input(T, w.rotary_dim, w.rope_base, w.table_f32, device, act)
    return dict(q=q, k=k, q_weight=qw, k_weight=kw, rope_table=table)


def algorithmic_bytes(w, tokens: Optional[int] = None) -> int:
    """Bytes one launch must move at minimum: every input read once, every
    output written once, the weights (and table) read once."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if w.form == "ucpe":
        # tokens: the sequence length N (per batch element)
        N = w.seq if tokens is None else tokens
        per_tok_head = 3 * 2 * w.head_dim * 2 + 4   # q, k, v in and out; inflation_sq
        return (w.batch * N * (w.heads * per_tok_head + 2 * 64)   # + proj_q, proj_kv
                + N * w.head_dim * 4)                              # cos, sin [N, D/2] fp32
    if w.form == "3d":
        T = w.tokens if tokens is None else tokens
        out_b = 1 if w.output_fp8 else 2
        per_tok = w.row * 2 + w.row * out_b
        weights = 2 * (w.hq + w.hk) * w.head_dim if w.is_qk_norm else 0
        return T * per_tok + weights
    T = w.tokens if tokens is None else tokens
    per_tok = 2 * 2 * (w.hq + w.hk) * w.head_dim + w.rotary_dim * (4 if w.table_f32 else 2)
    return T * per_tok + 2 * 2 * w.head_dim


def bytes_per_token(w) -> float:
    if isinstance(w, str):
        w = WORKLOADS[w]
    return algorithmic_bytes(w) / w.tokens


