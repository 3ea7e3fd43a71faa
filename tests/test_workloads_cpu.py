"""The camera-prep workload's synthetic inputs are what the design says they
are: rigid motions G with proj_q = G^T and proj_kv = G^-1, cos/sin tables of
n * 10000^(-2j/D), the k_scale formula, and the algorithmic byte count the
roofline divides by."""
import math

import torch

import workloads as W


def test_camera_matrices_are_rigid_motion_pairs():
    g = torch.Generator().manual_seed(3)
    pq, pkv = W.camera_matrices(g, 2, 40, 0.5)
    assert pq.shape == pkv.shape == (2, 40, 4, 4) and pq.dtype == torch.float32
    G = pq.double().transpose(-1, -2)
    R, t = G[..., :3, :3], G[..., :3, 3]
    eye3 = torch.eye(3, dtype=torch.float64)
    assert (R @ R.transpose(-1, -2) - eye3).abs().max() < 1e-6       # a rotation
    assert (torch.linalg.det(R) - 1).abs().max() < 1e-6               # no reflection
    assert torch.equal(G[..., 3, :3], torch.zeros_like(G[..., 3, :3]))
    assert torch.all(G[..., 3, 3] == 1)
    assert (G @ pkv.double() - torch.eye(4, dtype=torch.float64)).abs().max() < 1e-6
    assert 0.2 < t.std().item() < 0.9                                 # N(0, 0.5^2) translations


def test_ucpe_tables_and_scale():
    cos_t, sin_t = W.ucpe_rope_tables(50, 16, 10000.0)
    assert cos_t.shape == sin_t.shape == (50, 8) and cos_t.dtype == torch.float32
    for n, j in ((0, 0), (7, 3), (49, 7)):
        th = n * 10000.0 ** (-2.0 * j / 16)
        assert abs(cos_t[n, j].item() - math.cos(th)) < 1e-7
        assert abs(sin_t[n, j].item() - math.sin(th)) < 1e-7
    w = W.WORKLOADS["ucpe"]
    assert w.seq == 18480 == 21 * 22 * 40 and w.spatial == 22 * 40
    assert abs(w.k_scale - 112 ** -0.5 * 880 ** -0.5) < 1e-15


def test_ucpe_algorithmic_bytes_counts_every_tensor_once():
    w = W.FormUcpe("t", batch=2, seq=24, heads=3, head_dim=16, spatial=6)
    inp = W.make_inputs(w)
    read = sum(v.numel() * v.element_size() for v in inp.values())
    written = 3 * 2 * 24 * 3 * 16 * 2 + 2 * 3 * 24 * 4      # q/k/v_trans + inflation_sq
    assert W.algorithmic_bytes(w) == read + written
    assert W.algorithmic_bytes(W.WORKLOADS["ucpe"]) == 508_865_280
