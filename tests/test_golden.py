"""Stored fixtures under tests/golden/.

worked_examples.json: hand-worked examples whose expected outputs are
closed-form expressions (derived by hand, cited in the file); the oracle's
unrounded outputs must match them.

oracle_*.json (written by tests/golden/make_golden.py, which calls only the
oracle): the oracle must still produce the stored bits on the stored inputs,
and the CUDA path, run on the same stored inputs through the C ABI, must match
the stored bits within the parity tolerance (tests/_util.py).
"""
import glob
import json
import math
import os

import numpy as np
import pytest

import oracle as O
from tests._util import act_mismatch, e4m3_mismatch

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FIXTURES = sorted(os.path.basename(p)[:-5] for p in glob.glob(os.path.join(HERE, "oracle_*.json")))
EXPR_NAMES = {"cos": math.cos, "sin": math.sin, "sqrt": math.sqrt, "__builtins__": {}}


def _load(name):
    with open(os.path.join(HERE, name + ".json")) as f:
        return json.load(f)


def _unhex(d) -> np.ndarray:
    dt = np.dtype(d["dtype"])
    a = np.frombuffer(bytes.fromhex(d["hex"]), dtype=dt.newbyteorder(">"))
    return a.astype(dt).reshape(d["shape"])


def _eval(exprs) -> np.ndarray:
    return np.vectorize(lambda e: float(eval(e, EXPR_NAMES)), otypes=[np.float64])(
        np.array(exprs, dtype=object))


def _bits(values, act="bf16") -> np.ndarray:
    v = np.asarray(values, np.float64)
    return O.f16_from_f64(v) if act == "f16" else O.bf16_from_f64(v)


def test_fixture_set_present():
    assert len(FIXTURES) >= 8, FIXTURES


@pytest.mark.parametrize("ex", _load("worked_examples")["examples"],
                         ids=lambda e: e["name"])
def test_worked_example(ex):
    p = ex["params"]
    if ex["form"] == "table":
        tbl = np.asarray(ex["rope_table"], np.float32)
        q, k = O.rope_table(_bits(ex["q"]), _bits(ex["k"]), _bits(ex["q_weight"]),
                            _bits(ex["k_weight"]), tbl, p["eps"], p["rotary_dim"],
                            interleaved=p["interleaved"], exact=True)
        outs = (("q", q), ("k", k))
    else:
        q, k, v = O.rope_3d(_bits(ex["qkv"]), _bits(ex["q_weight"]), _bits(ex["k_weight"]),
                            exact=True, **p)
        outs = (("q", q), ("k", k), ("v", v))
    for n, got in outs:
        want = _eval(ex["expected_" + n])
        assert got.shape == want.shape, (n, got.shape, want.shape)
        assert np.allclose(got, want, rtol=0, atol=1e-14), (ex["name"], n, got, want)


@pytest.mark.parametrize("name", FIXTURES)
def test_oracle_reproduces_stored_bits(name):
    fx = _load(name)
    p, inp = fx["params"], fx["inputs"]
    if fx["form"] == "3d":
        norm = p["is_qk_norm"]
        got = O.rope_3d(_unhex(inp["qkv"]), _unhex(inp["q_weight"]) if norm else None,
                        _unhex(inp["k_weight"]) if norm else None,
                        **dict(p, pos_offset=p["pos_offset"] or 0))
        names = ("q", "k", "v")
    elif fx["form"] == "ucpe":
        got = O.ucpe_cam_prep(*(_unhex(inp[n]) for n in ("q", "k", "v", "proj_q", "proj_kv",
                                                          "rope_cos", "rope_sin")),
                              p["k_scale"], act=p["act"])
        names = ("q", "k", "v", "inflation_sq")
    else:
        tbl = _unhex(inp["rope_table"])
        got = O.rope_table(_unhex(inp["q"]), _unhex(inp["k"]), _unhex(inp["q_weight"]),
                           _unhex(inp["k_weight"]), tbl, p["eps"], p["rotary_dim"],
                           interleaved=p["interleaved"], act=p["act"])
        names = ("q", "k")
    for n, g in zip(names, got):
        want = _unhex(fx["expected"][n])
        assert g.dtype == want.dtype and np.array_equal(g, want), (name, n)


@pytest.mark.gpu
@pytest.mark.parametrize("name", FIXTURES)
def test_cuda_path_matches_stored_bits(name):
    import torch

    import qk_rmsnorm_rope_qknr_b200 as Q

    fx = _load(name)
    p, inp = fx["params"], fx["inputs"]

    def dev(d, torch_dtype):
        return torch.from_numpy(_unhex(d).view(np.int16)).view(torch_dtype).cuda()

    if fx["form"] == "3d":
        norm = p["is_qk_norm"]
        qkv = dev(inp["qkv"], torch.bfloat16)
        qw = dev(inp["q_weight"], torch.bfloat16) if norm else None
        kw = dev(inp["k_weight"], torch.bfloat16) if norm else None
        outs = Q.fused_qk_rmsnorm_rope(qkv, qw, kw, **p)
        names = ("q", "k", "v")
    elif fx["form"] == "ucpe":
        act = torch.float16 if p["act"] == "f16" else torch.bfloat16
        f32 = {n: torch.from_numpy(_unhex(inp[n]).copy()).cuda()
               for n in ("proj_q", "proj_kv", "rope_cos", "rope_sin")}
        outs = Q.cam_prep_func(dev(inp["q"], act), dev(inp["k"], act), dev(inp["v"], act),
                               k_scale=p["k_scale"], **f32)
        torch.cuda.synchronize()
        want = _unhex(fx["expected"]["inflation_sq"])
        np.testing.assert_allclose(outs[3].cpu().double().numpy(), want, rtol=2.0 ** -14, atol=0)
        # the tolerance's rows are the head vectors: compare as [B, H, N, D]
        outs = tuple(o.transpose(2, 3) for o in outs[:3])
        fx = dict(fx, expected={n: dict(fx["expected"][n], hex=None,
                                        arr=_unhex(fx["expected"][n]).transpose(0, 1, 3, 2))
                                for n in ("q", "k", "v")})
        names = ("q", "k", "v")
    else:
        act = torch.float16 if p["act"] == "f16" else torch.bfloat16
        tbl_np = _unhex(inp["rope_table"])
        tbl = (torch.from_numpy(tbl_np).cuda() if tbl_np.dtype == np.float32
               else dev(inp["rope_table"], act))
        outs = Q.fused_qk_norm_rope(dev(inp["q"], act), dev(inp["k"], act),
                                    dev(inp["q_weight"], act), dev(inp["k_weight"], act), tbl,
                                    p["eps"], rotary_dim=p["rotary_dim"],
                                    interleaved=p["interleaved"])
        names = ("q", "k")
    torch.cuda.synchronize()
    for n, o in zip(names, outs):
        e = fx["expected"][n]
        want = e["arr"] if "arr" in e else _unhex(e)
        got = o.cpu().contiguous()
        if want.dtype == np.uint8:
            bad, st = e4m3_mismatch(got.view(torch.uint8).numpy(), want)
        else:
            act = p.get("act", "bf16")
            got_bits = got.view(torch.int16).numpy().view(np.uint16)
            decode = O.f16_to_f64 if act == "f16" else O.bf16_to_f64
            bad, st = act_mismatch(got_bits, want, decode(want), act)
        assert len(bad) == 0, f"{name} {n}: {len(bad)} beyond tolerance {st}"
