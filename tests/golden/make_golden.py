"""Writes the oracle regression fixtures oracle_*.json in this folder.

Every stored number comes from oracle/ (its rounding of the drawn inputs and
its outputs); the inputs are drawn with numpy from fixed seeds. The fixtures
freeze the oracle's results on small cases of every mode, so that a change to
the oracle's arithmetic shows up as a failing test (tests/test_golden.py) and
has to be made on purpose, and so that the CUDA path can be checked against
stored values as well as against the live oracle.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402

CITE_3D = ('"flashinfer.norm.fused_qk_rmsnorm_rope" (FlashInfer API docs): summary, '
           'Parameters, Returns')
CITE_TABLE = ('"vllm_omni.diffusion.layers.fused_qk_norm_rope" (vLLM-Omni API docs): '
              'contract bullets, fused_qk_norm_rope')


def hexs(a: np.ndarray) -> str:
    a = np.ascontiguousarray(a)
    return a.astype(a.dtype.newbyteorder(">")).tobytes().hex()


def arr(a: np.ndarray) -> dict:
    return {"dtype": str(a.dtype), "shape": list(a.shape), "hex": hexs(a)}


def case_3d(name, seed, T, hq, hk, hv, D, grid, ch, interleave, fp8, norm, pos_offset):
    g = np.random.default_rng(seed)
    qkv = O.bf16_from_f64(g.standard_normal((T, (hq + hk + hv) * D)) * 2.0)
    qw = O.bf16_from_f64(1 + 0.1 * g.standard_normal(hq * D))
    kw = O.bf16_from_f64(1 + 0.1 * g.standard_normal(hk * D))
    p = dict(ppf=grid[0], pph=grid[1], ppw=grid[2], num_frame_channels=ch[0],
             num_height_channels=ch[1], num_width_channels=ch[2], num_heads_q=hq,
             num_heads_k=hk, num_heads_v=hv, head_dim=D, eps=1e-5, base=10000.0,
             interleave=interleave, is_qk_norm=norm, output_fp8=fp8, output_quant_scale=0.5,
             v_quant_scale=0.25, pos_offset=pos_offset)
    q, k, v = O.rope_3d(qkv, qw if norm else None, kw if norm else None,
                        **dict(p, pos_offset=pos_offset or 0))
    inputs = {"qkv": arr(qkv)}
    if norm:
        inputs.update(q_weight=arr(qw), k_weight=arr(kw))
    return name, {"form": "3d", "cite": CITE_3D, "params": p, "inputs": inputs,
                  "expected": {"q": arr(q), "k": arr(k), "v": arr(v)}}


def case_table(name, seed, T, hq, hk, D, R, interleaved, table_f32, act):
    g = np.random.default_rng(seed)
    to = O.f16_from_f64 if act == "f16" else O.bf16_from_f64
    q = to(g.standard_normal((T, hq, D)) * 2.0)
    k = to(g.standard_normal((T, hk, D)) * 2.0)
    qw = to(1 + 0.1 * g.standard_normal(D))
    kw = to(1 + 0.1 * g.standard_normal(D))
    theta = np.arange(T)[:, None] * 10000.0 ** (-2.0 * np.arange(R // 2) / R)[None, :]
    tbl = np.concatenate([np.cos(theta), np.sin(theta)], axis=1)
    tbl = tbl.astype(np.float32) if table_f32 else to(tbl)
    qo, ko = O.rope_table(q, k, qw, kw, tbl, 1e-6, R, interleaved=interleaved, act=act)
    p = dict(eps=1e-6, rotary_dim=R, interleaved=interleaved, act=act)
    return name, {"form": "table", "cite": CITE_TABLE, "params": p,
                  "inputs": {"q": arr(q), "k": arr(k), "q_weight": arr(qw),
                             "k_weight": arr(kw), "rope_table": arr(tbl)},
                  "expected": {"q": arr(qo), "k": arr(ko)}}

CITE_UCPE = ('"vllm_omni.diffusion.models.sana_wm.ucpe" (vLLM-Omni API docs): cam_prep_func, '
             'Parameters, Returns')


def _camera_matrices(g, B, N):
    """Per-token rigid motions G = [[R, t], [0, 1]] (R a random rotation, t ~
    N(0, 0.5^2)); proj_q = G^T and proj_kv = G^-1, as float32."""
    pq = np.empty((B, N, 4, 4), np.float32)
    pkv = np.empty((B, N, 4, 4), np.float32)
    for b in range(B):
        for n in range(N):
            m, r = np.linalg.qr(g.standard_normal((3, 3)))
            G = np.eye(4)
            G[:3, :3] = m * np.sign(np.diag(r))
            G[:3, 3] = 0.5 * g.standard_normal(3)
            pq[b, n] = G.T
            pkv[b, n] = np.linalg.inv(G)
    return pq, pkv


def case_ucpe(name, seed, B, N, H, D, act):
    g = np.random.default_rng(seed)
    to = O.f16_from_f64 if act == "f16" else O.bf16_from_f64
    q, k, v = (to(g.standard_normal((B, N, H, D))) for _ in range(3))
    pq, pkv = _camera_matrices(g, B, N)
    theta = np.arange(N)[:, None] * 10000.0 ** (-2.0 * np.arange(D // 2) / D)[None, :]
    cos_t, sin_t = np.cos(theta).astype(np.float32), np.sin(theta).astype(np.float32)
    k_scale = D ** -0.5 * 4 ** -0.5
    qo, ko, vo, infl = O.ucpe_cam_prep(q, k, v, pq, pkv, cos_t, sin_t, k_scale, act=act)
    p = dict(k_scale=k_scale, act=act)
    return name, {"form": "ucpe", "cite": CITE_UCPE, "params": p,
                  "inputs": {"q": arr(q), "k": arr(k), "v": arr(v), "proj_q": arr(pq),
                             "proj_kv": arr(pkv), "rope_cos": arr(cos_t),
                             "rope_sin": arr(sin_t)},
                  "expected": {"q": arr(qo), "k": arr(ko), "v": arr(vo),
                               "inflation_sq": arr(infl)}}


def cases():
    return [
    case_3d("oracle_3d_interleave_bf16", 1, 8, 2, 1, 1, 64, (2, 2, 2), (16, 24, 24), True,
            False, True, None),
    case_3d("oracle_3d_neox_e4m3", 2, 8, 2, 2, 1, 64, (2, 2, 2), (16, 24, 24), False, True,
            True, None),
    case_3d("oracle_3d_rope_only_shard", 3, 5, 1, 1, 1, 64, (2, 2, 2), (16, 24, 24), True,
            False, False, 3),
    case_table("oracle_table_halfsplit_f32", 4, 6, 2, 1, 64, 48, False, True, "bf16"),
    case_table("oracle_table_interleaved_bf16", 5, 6, 1, 2, 64, 64, True, False, "bf16"),
    case_table("oracle_table_halfsplit_f16", 6, 6, 2, 1, 64, 32, False, False, "f16"),
    case_ucpe("oracle_ucpe_bf16", 7, 2, 12, 2, 16, "bf16"),
    case_ucpe("oracle_ucpe_f16", 8, 1, 9, 3, 24, "f16"),
    ]


def main():
    for name, body in cases():
        with open(os.path.join(HERE, name + ".json"), "w") as f:
            json.dump(body, f, indent=1)
            f.write("\n")
        print("wrote", name)


if __name__ == "__main__":
    main()
