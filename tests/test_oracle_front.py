"""Pins of the oracle's latent front end (RMSNorm then RoPE, then bf16) on the CPU.

Independent references: hand-worked cases (tests/golden/front_end_cases.txt) whose
arithmetic is exact under the defined order and changes under the plausible other
orders; the L2-norm statement of the jdon.com article ("缓存压缩真的是越大越好吗": an
RMSNorm'd 512-channel latent has L2 norm about sqrt(512), and RoPE keeps it); a float64
RMSNorm + rotation within a rounding bound; torch's round-to-nearest-even bf16 conversion.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "front_end_cases.txt")


def _load():
    cases, cur = [], None
    with open(GOLDEN, encoding="utf-8") as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "case":
                cur = dict(name=tok[1], x=np.zeros(512, np.float32), w=None, cos=np.ones(32, np.float32),
                           sin=np.zeros(32, np.float32), out=np.zeros(512, np.float32))
            elif tok[0] == "x":
                cur["x"][int(tok[1])] = float.fromhex(tok[2])
            elif tok[0] == "w":
                if cur["w"] is None:
                    cur["w"] = np.ones(512, np.float32)
                cur["w"][int(tok[1])] = float.fromhex(tok[2])
            elif tok[0] == "rope":
                cur["cos"][int(tok[1])] = float.fromhex(tok[2])
                cur["sin"][int(tok[1])] = float.fromhex(tok[3])
            elif tok[0] == "out":
                cur["out"][int(tok[1])] = float.fromhex(tok[2])
            elif tok[0] == "end":
                cases.append(cur)
    return cases


CASES = _load()


def _bits(v):
    v = np.asarray(v, np.float32)
    u = v.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c["name"])
def test_front_end_hand_worked(case):
    x = _bits(case["x"]).reshape(1, 512)
    got = oracle.front_end(x, case["cos"], case["sin"], case["w"], f32=True)[0]
    assert np.array_equal(got.view(np.uint32), case["out"].view(np.uint32)), np.nonzero(got != case["out"])
    y = oracle.front_end(x, case["cos"], case["sin"], case["w"])[0]
    assert np.array_equal(y, _bits(case["out"]))


def _rope_tables(pos, rows):
    k = np.arange(32, dtype=np.float64)
    ang = np.asarray(pos, np.float64).reshape(rows, 1) * 10000.0 ** (-2.0 * k / 64.0)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def test_front_end_l2_norm_is_sqrt512():
    """[Jdon]: weight 1 gives an L2 norm of about sqrt(512) ~ 22.6, and RoPE keeps it."""
    rows = 64
    x = synth.normal(5, (rows, 512)).to(torch.bfloat16)
    cos, sin = _rope_tables(np.arange(rows) * 977, rows)
    y = oracle.front_end(synth.bf16_bits(x), cos, sin, f32=True).astype(np.float64)
    xd = x.double().numpy()
    expect = np.sqrt(512.0 * (xd ** 2).mean(1) / ((xd ** 2).mean(1) + 1e-6))
    assert np.allclose(np.linalg.norm(y, axis=1), expect, rtol=2e-6)
    assert np.all(np.abs(np.linalg.norm(y, axis=1) - math.sqrt(512)) < 1e-3)


def test_front_end_float64_reference():
    """Each output within a few fp32 roundings of the exact RMSNorm and rotation."""
    rows = 32
    x = (synth.normal(6, (rows, 512)) * 3.0).to(torch.bfloat16)
    w = (0.5 + synth.uniform(7, 512).numpy()).astype(np.float32)
    cos, sin = _rope_tables(np.arange(rows) * 4099 + 11, rows)
    got = oracle.front_end(synth.bf16_bits(x), cos, sin, w, f32=True).astype(np.float64)
    xd = x.double().numpy()
    n = xd / np.sqrt((xd ** 2).mean(1, keepdims=True) + 1e-6) * w.astype(np.float64)
    ref = n.copy()
    a, b = n[:, 448::2], n[:, 449::2]
    c, s = cos.astype(np.float64), sin.astype(np.float64)
    ref[:, 448::2] = a * c - b * s
    ref[:, 449::2] = a * s + b * c
    # a 512-term fp32 chain can be off by up to ~512 roundings relative to ss, half of
    # that reaches r; then a few more roundings per output
    scale = np.abs(n).max(1, keepdims=True)
    assert np.all(np.abs(got - ref) <= (256 + 8) * 2.0 ** -24 * (np.abs(ref) + scale))


def test_front_end_bf16_is_nearest_even_of_f32():
    rows = 40
    x = (synth.normal(8, (rows, 512)) * 0.01).to(torch.bfloat16)
    cos, sin = _rope_tables(np.arange(rows), rows)
    f = oracle.front_end(synth.bf16_bits(x), cos, sin, f32=True)
    y = oracle.front_end(synth.bf16_bits(x), cos, sin)
    ref = synth.bf16_bits(torch.from_numpy(f).to(torch.bfloat16))
    assert np.array_equal(y, ref)


def test_front_end_rope_keeps_pair_norms():
    rows = 16
    x = synth.normal(9, (rows, 512)).to(torch.bfloat16)
    cos, sin = _rope_tables(np.arange(rows) * 12345, rows)
    idc, ids = np.ones((rows, 32), np.float32), np.zeros((rows, 32), np.float32)
    bx = synth.bf16_bits(x)
    y = oracle.front_end(bx, cos, sin, f32=True).astype(np.float64)
    n = oracle.front_end(bx, idc, ids, f32=True).astype(np.float64)   # identity rotation
    assert np.array_equal(y[:, :448], n[:, :448])
    pr = np.hypot(y[:, 448::2], y[:, 449::2])
    pn = np.hypot(n[:, 448::2], n[:, 449::2])
    assert np.all(np.abs(pr - pn) <= 4 * 2.0 ** -24 * pn + 1e-30)


def test_front_end_eps_at_small_magnitudes():
    """Constant rows x_c = v: n_c = v / sqrt(v^2 + eps) (the chain of 512 equal squares is
    exact for these powers of two); at v = 2^-10, v^2 is close to eps = 1e-6, so eps counts."""
    vals = [2.0 ** -10, 2.0 ** -8, 2.0 ** -12, 1.0]
    x = torch.tensor([[v] * 512 for v in vals], dtype=torch.float32).to(torch.bfloat16)
    idc, ids = np.ones((len(vals), 32), np.float32), np.zeros((len(vals), 32), np.float32)
    got = oracle.front_end(synth.bf16_bits(x), idc, ids, f32=True).astype(np.float64)
    for i, v in enumerate(vals):
        ref = v / math.sqrt(v * v + float(np.float32(1e-6)))
        assert np.all(np.abs(got[i] - ref) <= 4 * 2.0 ** -24 * ref), (v, got[i, 0], ref)
