"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each pin cites what fixes it: a closed form, a textbook or library routine,
an invariant of the mathematics, or a tiny case worked out by hand in the
comments. Pages cited by title:
  [T] "vllm_omni.diffusion.layers.fused_qk_norm_rope" -- contract bullets
  [F] "flashinfer.norm.fused_qk_rmsnorm_rope" -- summary, Parameters, Returns
  [U] "vllm_omni.diffusion.models.sana_wm.ucpe" -- cam_prep_func
The pin_* functions are also run by test_oracle_mutations.py against copies of
the oracle with planted mistakes, each of which must fail at least one pin.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(1234)


def _bf16_bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)


def _rand_bf16(shape, std=1.0, rng=RNG):
    return _bf16_bits(rng.standard_normal(shape) * std)


# ----------------------------------------------------------------------------
# Number formats: one RNE rounding, checked against torch's own conversions.
# ----------------------------------------------------------------------------
def pin_bf16_rounding_vs_torch():
    """Every bf16 upper half x a set of lower halves (exact, ties, near ties):
    the oracle's double->bf16 must equal torch's float32->bf16 (one RNE)."""
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0x0000, 0x0001, 0x3FFF, 0x7FFF, 0x8000, 0x8001, 0xBFFF, 0xFFFF]
                    + list(RNG.integers(0, 1 << 16, 8)), dtype=np.uint32)
    bits = (hi[:, None] | lows[None, :]).ravel()
    f = bits.view(np.float32)
    keep = ~np.isnan(f)
    f = f[keep]
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.bf16_from_f64(f.astype(np.float64))
    assert np.array_equal(got, want)


def pin_bf16_single_rounding_of_doubles():
    """Doubles that sit on or just off a bf16 tie: one rounding from double
    (not double->float->bf16). 1 + 2^-8 is the tie between 1 and 1 + 2^-7."""
    one, up = 0x3F80, 0x3F81
    cases = [(1.0 + 2.0 ** -8, one),               # tie -> even (1.0)
             (1.0 + 2.0 ** -8 + 2.0 ** -40, up),   # just above the tie
             (1.0 + 2.0 ** -8 - 2.0 ** -40, one),  # just below the tie
             (1.0 + 3 * 2.0 ** -8, 0x3F82),        # tie between 1+2^-7 and 1+2^-6 -> even
             (-(1.0 + 2.0 ** -8 + 2.0 ** -40), 0x8000 | up),
             (2.0 ** 128, 0x7F80), (-(2.0 ** 200), 0xFF80),          # overflow -> inf
             ((2.0 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),               # max + half ulp -> inf
             ((2.0 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),               # largest finite
             (2.0 ** -133, 0x0001), (2.0 ** -134, 0x0000),           # subnormal, tie -> 0
             (3 * 2.0 ** -135, 0x0001), (0.0, 0x0000), (-0.0, 0x8000)]
    for x, want in cases:
        assert int(O.bf16_from_f64(np.array([x]))[0]) == want, (x, want)


def pin_e4m3_rounding_vs_torch():
    """All bf16-representable floats with |x| <= 464 (plus e4m3 midpoints and
    values 1/64 of a step off them): the oracle equals torch's float32 ->
    float8_e4m3fn, which rounds to nearest even. Above 464 torch gives NaN while
    the saturating conversion gives +-448 (checked by hand below)."""
    allb = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    vals = [allb[np.isfinite(allb) & (np.abs(allb) <= 464)]]
    codes = np.arange(0x7F, dtype=np.uint8)
    mags = O.e4m3_to_f64(codes)
    mids = (mags[:-1] + mags[1:]) / 2
    steps = np.diff(mags)
    for m in (mids, mids + steps / 64, mids - steps / 64):
        vals += [m.astype(np.float32), -m.astype(np.float32)]
    f = np.concatenate(vals)
    want = torch.from_numpy(f.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_from_f64(f.astype(np.float64))
    assert np.array_equal(got, want)


def pin_e4m3_hand_cases():
    """E4M3FN by hand: 1.5 = 1.100b x 2^0 -> exponent field 7, fraction 4 -> 0x3C;
    448 = 1.110b x 2^8 -> 0x7E; beyond it saturate; 2^-9 is the smallest
    subnormal (0x01); 2^-10 is its tie with zero -> 0; 2^-6 is the smallest
    normal (0x08); infinities saturate; NaN -> 0x7F."""
    cases = [(1.5, 0x3C), (-1.5, 0xBC), (448.0, 0x7E), (464.0, 0x7E), (500.0, 0x7E),
             (-1e9, 0xFE), (math.inf, 0x7E), (-math.inf, 0xFE), (2.0 ** -9, 0x01),
             (2.0 ** -10, 0x00), (3 * 2.0 ** -11, 0x01), (2.0 ** -6, 0x08),
             (0.0, 0x00), (1.0 + 2.0 ** -4, 0x38), (1.0 + 2.0 ** -4 + 2.0 ** -30, 0x39)]
    for x, want in cases:
        assert int(O.e4m3_from_f64(np.array([x]))[0]) == want, (x, want)
    assert int(O.e4m3_from_f64(np.array([math.nan]))[0]) == 0x7F


def pin_f16_rounding_vs_torch():
    """IEEE binary16 (table-form activations may be fp16): every finite binary16
    value, every midpoint between neighbours, and points 1/64 of a step off
    them, rounded by the oracle from double, equal torch's float32 -> float16
    (one RNE rounding)."""
    allh = np.arange(1 << 16, dtype=np.uint16).view(np.float16).astype(np.float64)
    fin = np.sort(np.unique(allh[np.isfinite(allh)]))
    mids = (fin[:-1] + fin[1:]) / 2
    steps = np.diff(fin)
    f = np.concatenate([fin, mids, mids + steps / 64, mids - steps / 64, [65520.0, -65520.0,
                                                                         70000.0, 1e-9]])
    f32 = f.astype(np.float32)
    want = torch.from_numpy(f32.copy()).to(torch.float16).view(torch.int16).numpy() \
        .view(np.uint16)
    got = O.f16_from_f64(f32.astype(np.float64))
    assert np.array_equal(got, want)


def pin_f16_hand_cases():
    """binary16 by hand: 65504 is the largest finite (0x7BFF); 65520 is its tie
    with 2^16 and rounds to even, i.e. to infinity (0x7C00); 2^-24 is the
    smallest subnormal (0x0001) and 2^-25 its tie with zero (-> 0); 1 + 2^-11 is
    the tie between 1 and 1 + 2^-10 (-> 1.0, 0x3C00), one 2^-40 above it goes up."""
    cases = [(65504.0, 0x7BFF), (65520.0, 0x7C00), (-65520.0, 0xFC00), (2.0 ** -24, 0x0001),
             (2.0 ** -25, 0x0000), (3 * 2.0 ** -26, 0x0001), (1 + 2.0 ** -11, 0x3C00),
             (1 + 2.0 ** -11 + 2.0 ** -40, 0x3C01), (2.0 ** -14, 0x0400), (-2.0, 0xC000)]
    for x, want in cases:
        assert int(O.f16_from_f64(np.array([x]))[0]) == want, (x, want)
    for bits in (0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0xC000):
        v = O.f16_to_f64(np.array([bits], np.uint16))[0]
        assert O.lib().qknr_oracle_f16_to_double(bits) == v


def pin_table_f16_brute_force():
    """Table form with binary16 activations, weights and table: per-head RMS
    norm, weight, rotation, by numpy matrix products on the exact fp16 values."""
    T, Hq, Hk, D, R = 4, 2, 1, 16, 12
    h = lambda a: np.asarray(a, np.float16).view(np.uint16)  # noqa: E731
    q = h(RNG.standard_normal((T, Hq, D)) * 30)
    k = h(RNG.standard_normal((T, Hk, D)))
    qw, kw = h(1 + 0.2 * RNG.standard_normal(D)), h(1 + 0.2 * RNG.standard_normal(D))
    theta = RNG.uniform(-4, 4, (T, R // 2))
    tbl = h(np.concatenate([np.cos(theta), np.sin(theta)], 1))
    for il in (True, False):
        qo, ko = O.rope_table(q, k, qw, kw, tbl, 1e-5, R, interleaved=il, exact=True, act="f16")
        pa, pb = O.pairs_table(R, il)
        tv = O.f16_to_f64(tbl)
        for t in range(T):
            M = np.eye(D)
            for j in range(R // 2):
                a, b = pa[j], pb[j]
                c, s_ = tv[t, j], tv[t, R // 2 + j]
                M[a, a], M[a, b], M[b, a], M[b, b] = c, -s_, s_, c
            for X, src, wt in ((qo, q, qw), (ko, k, kw)):
                xs = O.f16_to_f64(src[t])
                for hh in range(xs.shape[0]):
                    y = xs[hh] / np.sqrt(np.mean(xs[hh] ** 2) + 1e-5) * O.f16_to_f64(wt)
                    assert np.allclose(X[t, hh], M @ y, rtol=1e-12, atol=1e-12)
        qb, _ = O.rope_table(q, k, qw, kw, tbl, 1e-5, R, interleaved=il, act="f16")
        assert np.array_equal(qb, O.f16_from_f64(qo))


# ----------------------------------------------------------------------------
# Steps: position, angle, norm, rotation, pair maps.
# ----------------------------------------------------------------------------
def pin_position_row_major():
    """[F] Parameters: seq_len = ppf*pph*ppw, tokens divisible by it. Row-major
    (frame, height, width) order, by hand for a 2x3x4 grid."""
    cases = {0: (0, 0, 0), 1: (0, 0, 1), 3: (0, 0, 3), 4: (0, 1, 0), 11: (0, 2, 3),
             12: (1, 0, 0), 17: (1, 1, 1), 23: (1, 2, 3), 24: (0, 0, 0), 30: (0, 1, 2)}
    for t, want in cases.items():
        assert O.position_3d(t, 0, 2, 3, 4) == want, t
    assert O.position_3d(1, 23, 2, 3, 4) == (0, 0, 0)   # offset wraps the grid
    assert O.position_3d(0, 17, 2, 3, 4) == (1, 1, 1)


def pin_angles_closed_form():
    """Channels 2/4/6 (frame/height/width slots 1/2/3), base 64, patch (5,7,11):
    frame slot: 5; height slots: 7, 7*64^(-2/4) = 7/8; width slots: 11,
    11*64^(-2/6) = 11/4, 11*64^(-4/6) = 11/16."""
    th = O.angles_3d(5, 7, 11, 2, 4, 6, 64.0)
    want = [5.0, 7.0, 7.0 / 8, 11.0, 11.0 / 4, 11.0 / 16]
    assert np.allclose(th, want, rtol=1e-15, atol=0)
    th = O.angles_3d(3, 0, 2, 4, 0, 4, 10000.0)   # 10000^(-1/2) = 0.01
    assert np.allclose(th, [3.0, 0.03, 2.0, 0.02], rtol=1e-15, atol=0)


def pin_rmsnorm_hand():
    """x = (3,4,0,0): mean square 25/4. eps = 0 -> r = 2/5, y = (1.2, 1.6, 0, 0).
    eps = 2.75 -> mean square + eps = 9, r = 1/3. Weight (2, .5, 1, 1) multiplies
    channel by channel."""
    x = np.array([3.0, 4.0, 0.0, 0.0])
    assert np.allclose(O.rmsnorm(x, None, 0.0), [1.2, 1.6, 0, 0], rtol=1e-15)
    assert np.allclose(O.rmsnorm(x, None, 2.75), [1.0, 4.0 / 3, 0, 0], rtol=1e-15)
    w = np.array([2.0, 0.5, 1.0, 1.0])
    assert np.allclose(O.rmsnorm(x, w, 2.75), [2.0, 2.0 / 3, 0, 0], rtol=1e-15)


def pin_rotation_is_complex_product():
    """A pair (a, b) rotates like the complex number a + ib times e^{i theta}:
    (1,0) -> (cos, sin), (0,1) -> (-sin, cos); and for random pairs the numpy
    complex product agrees."""
    th = 0.7
    out = O.rotate(np.array([1.0, 0.0, 0.0, 1.0]), [0, 2], [1, 3], [math.cos(th)] * 2,
                   [math.sin(th)] * 2)
    assert np.allclose(out, [math.cos(th), math.sin(th), -math.sin(th), math.cos(th)],
                       rtol=0, atol=1e-16)
    y = RNG.standard_normal(16)
    theta = RNG.uniform(-10, 10, 8)
    pa, pb = np.arange(8), np.arange(8) + 8
    out = O.rotate(y, pa, pb, np.cos(theta), np.sin(theta))
    z = (y[pa] + 1j * y[pb]) * np.exp(1j * theta)
    assert np.allclose(out[pa], z.real, atol=1e-14) and np.allclose(out[pb], z.imag, atol=1e-14)


def pin_pair_maps():
    """[T] contract bullets: half-split pairing of channel d with d + rotary_dim/2; interleaved
    adjacent pairs (2i, 2i+1). [F] interleave=False is NeoX style: whole-head
    half split (the reading taken here)."""
    pa, pb = O.pairs_table(8, True)
    assert pa.tolist() == [0, 2, 4, 6] and pb.tolist() == [1, 3, 5, 7]
    pa, pb = O.pairs_table(6, False)
    assert pa.tolist() == [0, 1, 2] and pb.tolist() == [3, 4, 5]
    pa, pb = O.pairs_3d(4, 2, 2, False)
    assert pa.tolist() == [0, 1, 2, 3] and pb.tolist() == [4, 5, 6, 7]
    pa, pb = O.pairs_3d(4, 2, 2, False, neox_per_axis=True)
    assert pa.tolist() == [0, 1, 4, 6] and pb.tolist() == [2, 3, 5, 7]


# ----------------------------------------------------------------------------
# Whole pipeline: hand cases and brute force.
# ----------------------------------------------------------------------------
def pin_table_hand_case():
    """One head, D = 4, x = (3,4,0,0), unit weights, eps = 0: y = (1.2, 1.6, 0, 0).
    Token 1's table row holds cos = (0, 1), sin = (1, 0): slot 0 turns by 90
    degrees, slot 1 by 0.
      interleaved pairs (0,1),(2,3): (1.2,1.6) -> (-1.6, 1.2); (0,0) stays.
      half-split pairs (0,2),(1,3): (1.2,0) -> (0, 1.2); (1.6,0) stays.
    Token 0 (cos 1, sin 0) returns y."""
    x = _bf16_bits([[[3, 4, 0, 0]], [[3, 4, 0, 0]]])
    w = _bf16_bits([1, 1, 1, 1])
    tbl = np.array([[1, 1, 0, 0], [0, 1, 1, 0]], np.float32)
    q, k = O.rope_table(x, x, w, w, tbl, 0.0, 4, interleaved=True, exact=True)
    assert np.allclose(q[0, 0], [1.2, 1.6, 0, 0], atol=1e-15)
    assert np.allclose(q[1, 0], [-1.6, 1.2, 0, 0], atol=1e-15)
    assert np.array_equal(q, k)
    q, _ = O.rope_table(x, x, w, w, tbl, 0.0, 4, interleaved=False, exact=True)
    assert np.allclose(q[1, 0], [0, 1.6, 1.2, 0], atol=1e-15)
    qb, _ = O.rope_table(x, x, w, w, tbl, 0.0, 4, interleaved=False)
    assert qb[1, 0].tolist() == O.bf16_from_f64(np.array([0, 1.6, 1.2, 0])).tolist()


def pin_weight_before_rotation():
    """[T] (contract bullets: the norm comes first, then the rotation): the weight scales the channel
    before it turns. D = 2, x = (1, 1): mean square 1, so y = (w0, w1) = (2, 0.5);
    a 90-degree turn gives (-0.5, 2). (Weighting after the turn would give
    (-1, 1) * (2, 0.5) = (-2, 0.5).)"""
    x = _bf16_bits([[[1, 1]], [[1, 1]]])
    w = _bf16_bits([2, 0.5])
    tbl = np.array([[1, 0], [0, 1]], np.float32)
    q, _ = O.rope_table(x, x, w, w, tbl, 0.0, 2, interleaved=True, exact=True)
    assert np.allclose(q[1, 0], [-0.5, 2.0], atol=1e-15)


def _rot_matrix(D, pa, pb, theta):
    M = np.eye(D)
    for j in range(len(pa)):
        c, s = np.cos(theta[j]), np.sin(theta[j])
        a, b = pa[j], pb[j]
        M[a, a], M[a, b], M[b, a], M[b, b] = c, -s, s, c
    return M


def pin_3d_brute_force():
    """3D form on a 2x2x3 grid, 2+1+1 heads of 8 channels (2/2/4): each head of
    the output equals M(theta) @ (w * x / rms) with the RMS over ALL Q (or K)
    channels of the token ([F]: across-heads RMSNorm), M the block rotation
    built from the pair map and angles, computed by numpy matrix products."""
    cf, ch, cw, D, Hq, Hk, Hv = 2, 2, 4, 8, 2, 1, 1
    T = 12
    qkv = _rand_bf16((T, (Hq + Hk + Hv) * D))
    qw, kw = _bf16_bits(1 + 0.3 * RNG.standard_normal(Hq * D)), _bf16_bits(
        1 + 0.3 * RNG.standard_normal(Hk * D))
    for interleave in (True, False):
        q, k, v = O.rope_3d(qkv, qw, kw, ppf=2, pph=2, ppw=3, num_frame_channels=cf,
                            num_height_channels=ch, num_width_channels=cw, num_heads_q=Hq,
                            num_heads_k=Hk, num_heads_v=Hv, head_dim=D, eps=0.01, base=7.0,
                            interleave=interleave, exact=True)
        x = O.bf16_to_f64(qkv)
        pa, pb = O.pairs_3d(cf, ch, cw, interleave)
        for t in range(T):
            f, h, w_ = t // 6, (t // 3) % 2, t % 3
            theta = O.angles_3d(f, h, w_, cf, ch, cw, 7.0)
            M = _rot_matrix(D, pa, pb, theta)
            for X, off, H, wt in ((q, 0, Hq, qw), (k, Hq * D, Hk, kw)):
                xs = x[t, off:off + H * D]
                rms = np.sqrt(np.mean(xs ** 2) + 0.01)
                y = xs / rms * O.bf16_to_f64(wt)
                for hh in range(H):
                    want = M @ y[hh * D:(hh + 1) * D]
                    assert np.allclose(X[t, hh], want, rtol=1e-12, atol=1e-12)
            assert np.array_equal(v[t].ravel(), x[t, (Hq + Hk) * D:])


def pin_table_brute_force():
    """Table form, per-head RMSNorm ([T]: weights are [head_dim]); rd < D leaves
    channels >= rd normalised but unrotated; matrix products as above."""
    T, Hq, Hk, D, R = 5, 3, 2, 16, 12
    q = _rand_bf16((T, Hq, D))
    k = _rand_bf16((T, Hk, D), std=3.0)
    qw, kw = _bf16_bits(1 + 0.2 * RNG.standard_normal(D)), _bf16_bits(
        1 + 0.2 * RNG.standard_normal(D))
    theta = RNG.uniform(-4, 4, (T, R // 2))
    tbl = np.concatenate([np.cos(theta), np.sin(theta)], 1).astype(np.float32)
    for il in (True, False):
        qo, ko = O.rope_table(q, k, qw, kw, tbl, 1e-5, R, interleaved=il, exact=True)
        pa, pb = O.pairs_table(R, il)
        for t in range(T):
            th = np.arctan2(tbl[t, R // 2:].astype(np.float64), tbl[t, :R // 2].astype(np.float64))
            M = _rot_matrix(D, pa, pb, th)
            # the table's stored cos/sin (fp32) are used as given: rebuild M from them
            for j in range(R // 2):
                a, b = pa[j], pb[j]
                c, s = float(tbl[t, j]), float(tbl[t, R // 2 + j])
                M[a, a], M[a, b], M[b, a], M[b, b] = c, -s, s, c
            for X, src, wt in ((qo, q, qw), (ko, k, kw)):
                xs = O.bf16_to_f64(src[t])
                for hh in range(xs.shape[0]):
                    y = xs[hh] / np.sqrt(np.mean(xs[hh] ** 2) + 1e-5) * O.bf16_to_f64(wt)
                    assert np.allclose(X[t, hh], M @ y, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# Invariants.
# ----------------------------------------------------------------------------
def _tiny3d(interleave=True, norm=True, T=16, H=(2, 2, 2), D=16, grid=(2, 2, 4), ch=(4, 4, 8),
            std=1.0, base=10000.0, weights=True, pos_offset=0, **extra):
    Hq, Hk, Hv = H
    qkv = _rand_bf16((T, (Hq + Hk + Hv) * D), std=std)
    qw = _bf16_bits(1 + 0.1 * RNG.standard_normal(Hq * D)) if weights else _bf16_bits(
        np.ones(Hq * D))
    kw = _bf16_bits(1 + 0.1 * RNG.standard_normal(Hk * D)) if weights else _bf16_bits(
        np.ones(Hk * D))
    p = dict(ppf=grid[0], pph=grid[1], ppw=grid[2], num_frame_channels=ch[0],
             num_height_channels=ch[1], num_width_channels=ch[2], num_heads_q=Hq, num_heads_k=Hk,
             num_heads_v=Hv, head_dim=D, base=base, interleave=interleave, is_qk_norm=norm,
             pos_offset=pos_offset)
    p.update(extra)
    return qkv, qw, kw, p


def pin_position_zero_identity():
    """Token 0 (patch (0,0,0)) turns by zero: its Q equals the normalised,
    weighted input; rows at s = P (next batch) also sit at (0,0,0)."""
    qkv, qw, kw, p = _tiny3d(T=32)
    q, k, v = O.rope_3d(qkv, qw, kw, eps=1e-6, exact=True, **p)
    x = O.bf16_to_f64(qkv)
    for t in (0, 16):
        xs = x[t, :32]
        y = xs / np.sqrt(np.mean(xs ** 2) + 1e-6) * O.bf16_to_f64(qw)
        assert np.allclose(q[t].ravel(), y, rtol=1e-14)
    assert not np.allclose(q[1].ravel(), O.rmsnorm(x[1, :32], O.bf16_to_f64(qw), 1e-6))


def pin_pair_norm_preserved():
    """Rotation is orthogonal: every pair's a'^2 + b'^2 equals the unrotated
    pair's (token 0 gives the unrotated values of the same row)."""
    for il in (True, False):
        qkv, qw, kw, p = _tiny3d(interleave=il, T=16)
        qkv[5] = qkv[0]
        q, k, _ = O.rope_3d(qkv, qw, kw, eps=1e-6, exact=True, **p)
        pa, pb = O.pairs_3d(4, 4, 8, il)
        for X in (q, k):
            n0 = X[0][:, pa] ** 2 + X[0][:, pb] ** 2
            n5 = X[5][:, pa] ** 2 + X[5][:, pb] ** 2
            assert np.allclose(n0, n5, rtol=1e-12)


def pin_unit_weight_rms_across_heads():
    """[F]: Q is normalised over all heads' channels together, [T]: per head.
    With unit weights, eps = 0 and heads of very different scale, the 3D output
    row has RMS 1 over the whole Q (not per head), the table output per head."""
    qkv, qw, kw, p = _tiny3d(weights=False, T=16)
    qkv = O.bf16_to_f64(qkv)
    qkv[:, 16:32] *= 16.0   # Q head 1 much larger than head 0
    qkv = O.bf16_from_f64(qkv)
    q, k, _ = O.rope_3d(qkv, qw, kw, eps=0.0, exact=True, **p)
    for X in (q, k):
        assert np.allclose(np.sqrt(np.mean(X.reshape(16, -1) ** 2, axis=1)), 1.0, rtol=1e-12)
    per_head = np.sqrt(np.mean(q ** 2, axis=2))
    assert np.all(per_head[:, 1] > 1.3)
    qt = qkv[:, :32].reshape(16, 2, 16)
    w1 = _bf16_bits(np.ones(16))
    tbl = np.tile(np.array([1.0] * 8 + [0.0] * 8, np.float32), (16, 1))
    qo, _ = O.rope_table(qt, qt, w1, w1, tbl, 0.0, 16, interleaved=True, exact=True)
    assert np.allclose(np.sqrt(np.mean(qo ** 2, axis=2)), 1.0, rtol=1e-12)


def pin_rope_only_identity_at_origin():
    """[F] is_qk_norm=False applies RoPE only: at patch (0,0,0) the bf16 output
    is bit-identical to the input, and V is a bit copy everywhere."""
    qkv, qw, kw, p = _tiny3d(norm=False, std=5.0)
    q, k, v = O.rope_3d(qkv, None, None, eps=1e-6, **p)
    assert np.array_equal(q[0].ravel(), qkv[0, :32]) and np.array_equal(k[0].ravel(),
                                                                           qkv[0, 32:64])
    assert np.array_equal(v.reshape(16, -1), qkv[:, 64:])
    assert not np.array_equal(q[3].ravel(), qkv[3, :32])


def pin_fp8_outputs():
    """[F] output_fp8: Q/K use output_quant_scale, V uses v_quant_scale (R9:
    the scale multiplies). At the origin with the norm off, q_out equals
    E4M3(x * 0.5) and v_out E4M3(v * 0.25), compared with torch's own
    float32 -> float8_e4m3fn (the products are exact in float32)."""
    qkv, _, _, p = _tiny3d(norm=False, std=2.0)
    q, k, v = O.rope_3d(qkv, None, None, output_fp8=True, output_quant_scale=0.5,
                        v_quant_scale=0.25, **p)
    x = torch.from_numpy(qkv.view(np.int16).copy()).view(torch.bfloat16).float()
    want_q = (x[0, :32] * 0.5).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    want_v = (x[:, 64:] * 0.25).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q[0].ravel(), want_q)
    assert np.array_equal(v.reshape(16, -1), want_v)


def pin_relative_position():
    """RoPE's defining property: <R(p) a, R(p') b> depends only on p - p' along
    each axis. Shifting both patches by one step along any single axis keeps the
    dot product of each head."""
    cf, ch, cw, D = 4, 6, 6, 16
    a, b = RNG.standard_normal(D), RNG.standard_normal(D)
    for il in (True, False):
        pa, pb = O.pairs_3d(cf, ch, cw, il)

        def rot(x, f, h, w):
            th = O.angles_3d(f, h, w, cf, ch, cw, 100.0)
            return O.rotate(x, pa, pb, np.cos(th), np.sin(th))

        d0 = rot(a, 1, 2, 3) @ rot(b, 4, 0, 5)
        for sh in ((1, 0, 0), (0, 1, 0), (0, 0, 1), (2, 3, 1)):
            d1 = rot(a, 1 + sh[0], 2 + sh[1], 3 + sh[2]) @ rot(b, 4 + sh[0], sh[1], 5 + sh[2])
            assert abs(d0 - d1) < 1e-12
        d2 = rot(a, 1, 2, 3) @ rot(b, 5, 0, 5)   # a different offset changes it
        assert abs(d0 - d2) > 1e-3


def pin_cross_contract():
    """With one Q and one K head the across-heads norm is the per-head norm, so
    the 3D form equals the table form fed the 3D angles as a float64-accurate
    table: interleave <-> interleaved, NeoX <-> half-split with rotary_dim = D."""
    cf, ch, cw, D = 4, 4, 8, 16
    for il in (True, False):
        qkv, qw, kw, p = _tiny3d(interleave=il, T=16, H=(1, 1, 1), std=2.0)
        q3, k3, _ = O.rope_3d(qkv, qw, kw, eps=1e-5, exact=True, **p)
        # a table whose cos/sin are exactly representable: quarter turns only
        # would be too special, so compare against float32 tables within 1e-6.
        th = np.stack([O.angles_3d(*O.position_3d(t, 0, 2, 2, 4), cf, ch, cw, 10000.0)
                       for t in range(16)])
        tbl = np.concatenate([np.cos(th), np.sin(th)], 1).astype(np.float32)
        qt, kt = O.rope_table(qkv[:, None, :D].copy(), qkv[:, None, D:2 * D].copy(), qw, kw, tbl,
                              1e-5, D, interleaved=il, exact=True)
        assert np.allclose(q3, qt, rtol=0, atol=1e-6)
        assert np.allclose(k3, kt, rtol=0, atol=1e-6)


def pin_interleave_neox_permutation():
    """Moving channel j -> 2j and j + D/2 -> 2j + 1 (inputs and weights) turns
    the NeoX computation into the interleaved one."""
    D = 16
    perm = np.empty(D, int)
    perm[0::2] = np.arange(D // 2)
    perm[1::2] = np.arange(D // 2) + D // 2   # interleaved channel c holds NeoX channel perm[c]
    qkv, qw, kw, p = _tiny3d(interleave=False, T=16, std=2.0)
    qn, kn, _ = O.rope_3d(qkv, qw, kw, eps=1e-6, exact=True, **p)
    heads = qkv.reshape(16, 6, D)[:, :, perm].reshape(16, -1)
    p["interleave"] = True
    qi, ki, _ = O.rope_3d(heads, qw.reshape(2, D)[:, perm].ravel(),
                          kw.reshape(2, D)[:, perm].ravel(), eps=1e-6, exact=True, **p)
    assert np.allclose(qi, qn[:, :, perm], rtol=1e-13, atol=1e-14)
    assert np.allclose(ki, kn[:, :, perm], rtol=1e-13, atol=1e-14)


def pin_width_axis_textbook_rope():
    """ppf = pph = 1: only the width position varies. The width channels are a
    textbook 1D RoPE: pairs multiplied by exp(i * w * base^(-2i/Cw)) as numpy
    complex numbers; frame and height channels are not turned."""
    D, cw = 16, 8
    qkv, qw, kw, p = _tiny3d(T=8, grid=(1, 1, 8), ch=(4, 4, 8), weights=False, H=(1, 1, 1))
    q, _, _ = O.rope_3d(qkv, qw, kw, eps=0.0, exact=True, **p)
    x = O.bf16_to_f64(qkv)[:, :D]
    y = x / np.sqrt(np.mean(x ** 2, axis=1, keepdims=True))
    freqs = 10000.0 ** (-np.arange(cw // 2) * 2.0 / cw)
    for t in range(8):
        z = (y[t, 8::2] + 1j * y[t, 9::2]) * np.exp(1j * t * freqs)
        assert np.allclose(q[t, 0, 8::2], z.real, atol=1e-13)
        assert np.allclose(q[t, 0, 9::2], z.imag, atol=1e-13)
        assert np.allclose(q[t, 0, :8], y[t, :8], atol=1e-14)


def pin_neox_per_axis_textbook_rope():
    """The other reading of [F] interleave=False ("NeoX-style"), NeoX halves
    inside each axis group, on a grid where only the height and width positions
    vary: each group is a textbook 1D half-split RoPE of its own channels,
    pairs (o + i, o + i + C/2) multiplied by exp(i * pos * base^(-2i/C)) as
    numpy complex numbers; the frame group (position 0) is not turned. The
    whole-head NeoX reading differs on the same input."""
    D = 32
    ch = (8, 8, 16)
    qkv, qw, kw, p = _tiny3d(T=12, grid=(1, 3, 4), ch=ch, weights=False, H=(1, 1, 1), D=D)
    p = dict(p, interleave=False)
    q, _, _ = O.rope_3d(qkv, qw, kw, eps=0.0, exact=True, neox_per_axis=True, **p)
    q_whole, _, _ = O.rope_3d(qkv, qw, kw, eps=0.0, exact=True, **p)
    x = O.bf16_to_f64(qkv)[:, :D]
    y = x / np.sqrt(np.mean(x ** 2, axis=1, keepdims=True))
    for t in range(12):
        pos = {0: 0, 1: t // 4, 2: t % 4}
        o = 0
        for a, C in enumerate(ch):
            h = C // 2
            freqs = 10000.0 ** (-np.arange(h) * 2.0 / C)
            z = (y[t, o:o + h] + 1j * y[t, o + h:o + C]) * np.exp(1j * pos[a] * freqs)
            assert np.allclose(q[t, 0, o:o + h], z.real, atol=1e-13)
            assert np.allclose(q[t, 0, o + h:o + C], z.imag, atol=1e-13)
            o += C
    assert not np.allclose(q, q_whole)


def pin_offset_and_batch_repeat():
    """A token range computed with pos_offset equals the same rows of the whole
    call, and a second batch (tokens P..2P-1) repeats the first's angles."""
    qkv, qw, kw, p = _tiny3d(T=32)
    full = O.rope_3d(qkv, qw, kw, **p)
    p2 = dict(p, pos_offset=5)
    part = O.rope_3d(qkv[5:21].copy(), qw, kw, **p2)
    for a, b in zip(full, part):
        assert np.array_equal(a[5:21], b)
    qkv2 = qkv.copy()
    qkv2[16:] = qkv2[:16]
    q, k, v = O.rope_3d(qkv2, qw, kw, **p)
    assert np.array_equal(q[:16], q[16:]) and np.array_equal(k[:16], k[16:])


# ----------------------------------------------------------------------------
# UCPE camera prep ([U] cam_prep_func), readings U1..U6 of the oracle.
# ----------------------------------------------------------------------------
def _ucpe_inputs(B, N, H, D, rng=RNG):
    q, k, v = (_rand_bf16((B, N, H, D), rng=rng) for _ in range(3))
    return q, k, v


def _bf16_value_bits(x):
    """bf16 bit patterns of values that are exactly representable in bf16."""
    b = _bf16_bits(x)
    assert np.array_equal(O.bf16_to_f64(b), np.asarray(x, np.float64)), "not exact in bf16"
    return b


def pin_ucpe_identity_geometry():
    """Identity matrices and zero angles leave only the element steps and the
    layout: q_trans = ReLU(q), k_trans = k_scale * ReLU(k), v_trans = v, each
    moved from [B,N,H,D] to [B,H,D,N] (U5), all exact in bf16 because k_scale
    is a power of two; inflation_sq = 1 (an identity projection keeps every
    norm). Sizes differ in every axis so that a swapped index shows."""
    B, N, H, D = 2, 5, 3, 8
    q, k, v = _ucpe_inputs(B, N, H, D)
    eye = np.broadcast_to(np.eye(4, dtype=np.float32), (B, N, 4, 4))
    c = np.ones((N, D // 2), np.float32)
    s = np.zeros((N, D // 2), np.float32)
    qo, ko, vo, infl = O.ucpe_cam_prep(q, k, v, eye, eye, c, s, 0.25)
    t = (0, 2, 3, 1)
    xq, xk = O.bf16_to_f64(q), O.bf16_to_f64(k)
    assert np.array_equal(qo, _bf16_value_bits(np.maximum(xq, 0)).transpose(t))
    assert np.array_equal(ko, _bf16_value_bits(0.25 * np.maximum(xk, 0)).transpose(t))
    assert np.array_equal(vo, v.transpose(t))
    assert np.array_equal(infl, np.ones((B, H, N)))


def pin_ucpe_projection_orientation():
    """Permutation matrices move channels inside each block of four (U3):
    with y_i = sum_j M[i][j] x_j, row i of M having its 1 in column p(i) gives
    y_i = x_p(i). proj_q uses the 3-cycle p = (1, 2, 0, 3), proj_kv p = (3, 1,
    0, 2); neither equals its own transpose, and they differ from each other,
    so a transposed matrix or a swapped Q/KV matrix moves the wrong channel.
    Positive inputs and zero angles keep every value exact."""
    B, N, H, D = 1, 3, 2, 12
    rng = np.random.default_rng(7)
    q, k, v = (_bf16_bits(np.abs(rng.standard_normal((B, N, H, D))) + 0.1) for _ in range(3))
    pq_map, pkv_map = (1, 2, 0, 3), (3, 1, 0, 2)
    mq = np.zeros((4, 4), np.float32)
    mkv = np.zeros((4, 4), np.float32)
    for i in range(4):
        mq[i, pq_map[i]] = 1.0
        mkv[i, pkv_map[i]] = 1.0
    c = np.ones((N, D // 2), np.float32)
    s = np.zeros((N, D // 2), np.float32)
    qo, ko, vo, infl = O.ucpe_cam_prep(q, k, v, np.broadcast_to(mq, (B, N, 4, 4)),
                                       np.broadcast_to(mkv, (B, N, 4, 4)), c, s, 1.0)
    perm_q = np.array([4 * (d // 4) + pq_map[d % 4] for d in range(D)])
    perm_kv = np.array([4 * (d // 4) + pkv_map[d % 4] for d in range(D)])
    t = (0, 2, 3, 1)
    assert np.array_equal(qo, q[..., perm_q].transpose(t))
    assert np.array_equal(ko, k[..., perm_kv].transpose(t))
    assert np.array_equal(vo, v[..., perm_kv].transpose(t))
    assert np.allclose(infl, 1.0, rtol=0, atol=1e-15)


def pin_ucpe_hand_case():
    """One head of four channels, two tokens, worked by hand (k_scale 0.25).
    Token 0, angles 90 deg (pair 0: cos 0, sin 1) and 180 deg (pair 1):
      q = (1, -2, 3, 0.5): ReLU (1, 0, 3, 0.5); proj_q rows (1,0,0,0),
        (2,1,0,0), (0,0,1,0), (0,0,-1,2) give (1, 2, 3, -2); rotation:
        pair (1, 2) -> (1*0 - 2*1, 2*0 + 1*1) = (-2, 1); pair (3, -2) ->
        (-3, 2). q_trans = (-2, 1, -3, 2).
      k = (-1, 4, 2, 2): ReLU and scale (0, 1, 0.5, 0.5); proj_kv rows
        (0,1,0,0), (0,0,1,0), (1,0,0,0), (0,0,0,3) give (1, 0.5, 0, 1.5);
        |k'|^2 = 1.5, |y|^2 = 3.5, inflation_sq = 7/3; rotation: (1, 0.5) ->
        (-0.5, 1), (0, 1.5) -> (0, -1.5). k_trans = (-0.5, 1, 0, -1.5).
      v = (1, 2, 3, 4): proj_kv gives (2, 3, 1, 12), not rotated.
    Token 1, identity matrices, pair 0 at cos 0.6, sin 0.8 (as float32),
    pair 1 at 0 deg:
      q = (2, 1, -1, 1): ReLU (2, 1, 0, 1); pair (2, 1) -> (2*0.6 - 0.8,
        1*0.6 + 2*0.8) = (0.4, 2.2); q_trans = (0.4, 2.2, 0, 1).
      k = (1, 1, 1, 1): k' = 0.25 each, inflation_sq = 1; pair 0 ->
        (0.25*0.6 - 0.25*0.8, 0.25*0.6 + 0.25*0.8) = (-0.05, 0.35);
        k_trans = (-0.05, 0.35, 0.25, 0.25).
      v = (-1, 0, 5, 7) unchanged."""
    q = _bf16_bits([[[[1, -2, 3, 0.5]], [[2, 1, -1, 1]]]])
    k = _bf16_bits([[[[-1, 4, 2, 2]], [[1, 1, 1, 1]]]])
    v = _bf16_bits([[[[1, 2, 3, 4]], [[-1, 0, 5, 7]]]])
    eye = np.eye(4, dtype=np.float32)
    pq = np.stack([np.array([[1, 0, 0, 0], [2, 1, 0, 0], [0, 0, 1, 0], [0, 0, -1, 2]],
                            np.float32), eye])[None]
    pkv = np.stack([np.array([[0, 1, 0, 0], [0, 0, 1, 0], [1, 0, 0, 0], [0, 0, 0, 3]],
                             np.float32), eye])[None]
    c = np.array([[0, -1], [0.6, 1]], np.float32)
    s = np.array([[1, 0], [0.8, 0]], np.float32)
    qo, ko, vo, infl = O.ucpe_cam_prep(q, k, v, pq, pkv, c, s, 0.25, exact=True)
    c06, s08 = float(np.float32(0.6)), float(np.float32(0.8))
    want_q = [[-2, 1, -3, 2], [2 * c06 - s08, 1 * c06 + 2 * s08, 0, 1]]
    want_k = [[-0.5, 1, 0, -1.5], [0.25 * (c06 - s08), 0.25 * (c06 + s08), 0.25, 0.25]]
    want_v = [[2, 3, 1, 12], [-1, 0, 5, 7]]
    for got, want in ((qo, want_q), (ko, want_k), (vo, want_v)):
        assert got.shape == (1, 1, 4, 2)
        assert np.allclose(got[0, 0].T, want, rtol=1e-15, atol=1e-15), (got[0, 0].T, want)
    assert np.allclose(infl[0, 0], [7 / 3, 1.0], rtol=1e-15, atol=0)
    # rounded: token 1 of q is (0.4, 2.2, 0, 1) to bf16's precision
    qr = O.ucpe_cam_prep(q, k, v, pq, pkv, c, s, 0.25)[0]
    assert np.array_equal(O.bf16_to_f64(qr[0, 0, :, 1]),
                          O.bf16_to_f64(_bf16_bits([0.4, 2.2, 0.0, 1.0])))


def _random_rotation4(rng):
    m, r = np.linalg.qr(rng.standard_normal((4, 4)))
    return m * np.sign(np.diag(r))


def pin_ucpe_orthogonal_geometry_keeps_norms():
    """Orthogonal ray projections and rotations keep the Euclidean norm of
    every (token, head) vector: |q_trans| = |ReLU(q)|, |k_trans| = k_scale *
    |ReLU(k)|, |v_trans| = |v|, and inflation_sq = 1. The float32 matrices and
    cos/sin are orthogonal only to about 1e-7, hence the tolerance."""
    B, N, H, D = 2, 4, 3, 16
    rng = np.random.default_rng(11)
    q, k, v = _ucpe_inputs(B, N, H, D, rng)
    pq = np.stack([[_random_rotation4(rng) for _ in range(N)] for _ in range(B)]).astype(np.float32)
    pkv = np.stack([[_random_rotation4(rng) for _ in range(N)] for _ in range(B)]).astype(np.float32)
    th = rng.uniform(-np.pi, np.pi, (N, D // 2))
    c, s = np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    qo, ko, vo, infl = O.ucpe_cam_prep(q, k, v, pq, pkv, c, s, 0.3, exact=True)
    t = (0, 2, 3, 1)
    for got, x in ((qo, np.maximum(O.bf16_to_f64(q), 0)),
                   (ko, 0.3 * np.maximum(O.bf16_to_f64(k), 0)),
                   (vo, O.bf16_to_f64(v))):
        want = np.linalg.norm(x.transpose(t), axis=2)
        assert np.allclose(np.linalg.norm(got, axis=2), want, rtol=1e-6, atol=1e-12)
    assert np.allclose(infl, 1.0, rtol=0, atol=1e-6)


def pin_ucpe_scaled_identity_inflation():
    """proj_kv = c_n * I multiplies every key by c_n, so inflation_sq = c_n^2
    for every head (U6), whatever proj_q is; a key whose ReLU is all zero has
    inflation_sq = 1."""
    B, N, H, D = 1, 6, 2, 8
    rng = np.random.default_rng(5)
    q, k, v = _ucpe_inputs(B, N, H, D, rng)
    k = k.copy()
    k[0, 2, 1] = _bf16_bits(-np.abs(rng.standard_normal(D)) - 0.5)  # ReLU(k) = 0 here
    cn = np.arange(1, N + 1, dtype=np.float32) * 0.5
    pkv = (cn[:, None, None] * np.eye(4, dtype=np.float32))[None]
    pq = np.stack([_random_rotation4(rng) * 3 for _ in range(N)]).astype(np.float32)[None]
    th = rng.uniform(-np.pi, np.pi, (N, D // 2))
    c, s = np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    _, _, _, infl = O.ucpe_cam_prep(q, k, v, pq, pkv, c, s, 0.7, exact=True)
    want = np.broadcast_to((cn.astype(np.float64) ** 2)[None, None, :], (B, H, N)).copy()
    want[0, 1, 2] = 1.0
    assert np.allclose(infl, want, rtol=1e-14, atol=0)


def pin_ucpe_complex_brute_force():
    """Random everything, checked against a restatement in other terms: the
    projection as a batched matrix product over blocks (numpy einsum), the
    rotation as multiplication of z_j = y_2j + i y_2j+1 by cos_j + i sin_j
    (numpy complex128), the layout by transposing the result."""
    B, N, H, D = 2, 3, 2, 12
    rng = np.random.default_rng(3)
    q, k, v = _ucpe_inputs(B, N, H, D, rng)
    pq = rng.standard_normal((B, N, 4, 4)).astype(np.float32)
    pkv = rng.standard_normal((B, N, 4, 4)).astype(np.float32)
    th = rng.uniform(-np.pi, np.pi, (N, D // 2))
    c, s = np.cos(th).astype(np.float32), np.sin(th).astype(np.float32)
    ks = 0.37
    qo, ko, vo, infl = O.ucpe_cam_prep(q, k, v, pq, pkv, c, s, ks, exact=True)

    def project(m, x):  # x [B,N,H,D], m [B,N,4,4]
        blocks = x.reshape(B, N, H, D // 4, 4)
        return np.einsum("bnij,bnhcj->bnhci", m.astype(np.float64), blocks).reshape(B, N, H, D)

    def rope(y):
        z = (y[..., 0::2] + 1j * y[..., 1::2]) * (c + 1j * s).astype(np.complex128)[None, :, None]
        out = np.empty_like(y)
        out[..., 0::2], out[..., 1::2] = z.real, z.imag
        return out

    xq, xk, xv = (O.bf16_to_f64(a) for a in (q, k, v))
    kk = ks * np.maximum(xk, 0)
    yk = project(pkv, kk)
    t = (0, 2, 3, 1)
    assert np.allclose(qo, rope(project(pq, np.maximum(xq, 0))).transpose(t), rtol=1e-12,
                       atol=1e-12)
    assert np.allclose(ko, rope(yk).transpose(t), rtol=1e-12, atol=1e-12)
    assert np.allclose(vo, project(pkv, xv).transpose(t), rtol=1e-12, atol=1e-12)
    want = np.where((kk ** 2).sum(-1) > 0, (yk ** 2).sum(-1) / np.maximum((kk ** 2).sum(-1), 1e-300), 1.0)
    assert np.allclose(infl, want.transpose(0, 2, 1), rtol=1e-12, atol=0)


def pin_ucpe_f16_activations():
    """binary16 activations (as R13): the same steps on binary16 inputs, each
    result rounded once to binary16; identity geometry and a power-of-two
    k_scale keep every value exact, so the results are the inputs' ReLU (and
    scale) in binary16, checked against numpy's float16 conversion."""
    B, N, H, D = 1, 3, 2, 8
    rng = np.random.default_rng(9)
    xs = [rng.standard_normal((B, N, H, D)).astype(np.float16) for _ in range(3)]
    q, k, v = (x.view(np.uint16) for x in xs)
    eye = np.broadcast_to(np.eye(4, dtype=np.float32), (B, N, 4, 4))
    c = np.ones((N, D // 2), np.float32)
    s = np.zeros((N, D // 2), np.float32)
    qo, ko, vo, _ = O.ucpe_cam_prep(q, k, v, eye, eye, c, s, 2.0, act="f16")
    t = (0, 2, 3, 1)
    assert np.array_equal(qo, np.maximum(xs[0], 0).astype(np.float16).view(np.uint16).transpose(t))
    assert np.array_equal(ko, (2 * np.maximum(xs[1], 0)).astype(np.float16).view(np.uint16).transpose(t))
    assert np.array_equal(vo, v.transpose(t))


ALL_PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_") and callable(v)]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    O.use_library()   # the built oracle, in case a mutation test swapped it
    pin()


def test_threads_do_not_change_results():
    qkv, qw, kw, p = _tiny3d(T=64)
    O.set_threads(1)
    a = O.rope_3d(qkv, qw, kw, **p)
    O.set_threads(4)
    b = O.rope_3d(qkv, qw, kw, **p)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
