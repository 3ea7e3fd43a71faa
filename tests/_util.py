"""Test helpers: bit-pattern conversions and the parity tolerance.

Tolerance (the fused op's outputs against the oracle's):
  bf16: |gpu - ref| <= 2 ulp_bf16(max(|ref|, 2^-8 * rms)) where rms is the RMS
        of the oracle's exact output over the same (token, head) row. The floor
        exists because a rotation that cancels to near zero leaves an fp32
        kernel an absolute error of ~1e-7 |y|, far above the bf16 ulp of the
        tiny result; 2^-8 rms is the ulp scale of the row's typical element.
  f16:  the same rule in IEEE binary16: 2 ulp_f16(max(|ref|, 2^-11 * rms)),
        2^-11 being binary16's relative precision as 2^-8 is bf16's.
  e4m3: at most one step apart in the ordered code space (the codes of +-x are
        ordered like the values), which also covers the subnormal floor 2^-9.
"""
import numpy as np
import torch


def t2u16(t: torch.Tensor) -> np.ndarray:
    """bf16 or float16 torch tensor (any device) -> uint16 bit patterns (numpy)."""
    assert t.dtype in (torch.bfloat16, torch.float16)
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def t2u8(t: torch.Tensor) -> np.ndarray:
    assert t.dtype in (torch.float8_e4m3fn, torch.uint8)
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def u16_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    x = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(x)) - 7)


def f16u_to_f64(b: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64 (numpy's own binary16 decoding)."""
    return np.asarray(b, np.uint16).view(np.float16).astype(np.float64)


def ulp_f16(x: np.ndarray) -> np.ndarray:
    x = np.maximum(np.abs(x), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(x)) - 10)


_ACT = {"bf16": (u16_to_f64, ulp_bf16, 2.0 ** -8), "f16": (f16u_to_f64, ulp_f16, 2.0 ** -11)}


def act_mismatch(gpu_bits, ref_bits, ref_exact, act="bf16", ulps=2.0):
    """Indices where gpu misses ref by more than the tolerance of the 16-bit
    type `act` ("bf16" or "f16"); plus stats. Arrays are [..., D] (last axis =
    one head row)."""
    decode, ulp, floor = _ACT[act]
    g = decode(gpu_bits)
    r = decode(ref_bits)
    if g.size == 0:
        return np.zeros((0, g.ndim), int), dict(exact_frac=1.0, max_err_ulps=0.0, n=0)
    rms = np.sqrt(np.mean(np.square(ref_exact), axis=-1, keepdims=True))
    scale = np.maximum(np.abs(r), floor * rms)
    tol = ulps * ulp(scale)
    err = np.abs(g - r)
    bad = ~(err <= tol)  # NaN counts as bad
    stats = dict(
        exact_frac=float(np.mean(np.asarray(gpu_bits) == np.asarray(ref_bits))),
        max_err_ulps=float(np.max(err / ulp(scale))) if err.size else 0.0,
        n=int(err.size),
    )
    return np.argwhere(bad), stats


def bf16_mismatch(gpu_bits, ref_bits, ref_exact, ulps=2.0):
    return act_mismatch(gpu_bits, ref_bits, ref_exact, "bf16", ulps)


def e4m3_ordered(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, np.uint8).astype(np.int32)
    mag = b & 0x7F
    return np.where(b & 0x80, -mag, mag)


def e4m3_mismatch(gpu_bytes, ref_bytes, steps=1):
    g = e4m3_ordered(gpu_bytes)
    r = e4m3_ordered(ref_bytes)
    d = np.abs(g - r)
    bad = d > steps
    return np.argwhere(bad), dict(exact_frac=float(np.mean(d == 0)) if d.size else 1.0,
                                  max_steps=int(d.max()) if d.size else 0, n=int(d.size))
