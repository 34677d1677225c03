"""Pins of the oracle's sparse attention, replay mask and layer modes (CPU only).

Independent references: a dense softmax attention written here with
scipy.special (library routines) over an explicitly built key list, closed
forms (one key; uniform logits), the hand-worked replay-mask table in
tests/golden, and the layer patterns the pages print.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
D, H = 512, 16


def _case(seed, B=1, Q=1, cap=64, T=16, k=8):
    g = torch.Generator().manual_seed(seed)
    lat_bf = synth.latent(seed, B * cap)
    lat, lat_sc = oracle.quant_nvfp4(synth.bf16_bits(lat_bf))
    lat = lat.reshape(B, cap, 256)
    lat_sc = lat_sc.reshape(B, cap, 32)
    swa = np.stack([synth.swa_kv(seed * 10 + b, T, 0)[0].numpy() for b in range(B)]) if T else np.zeros((B, 0, D), np.uint8)
    swa_sc = np.stack([synth.swa_kv(seed * 10 + b, T, 0)[1].numpy() for b in range(B)]) if T else np.zeros((B, 0), np.float32)
    q = synth.attn_q(seed, B, Q)
    idx = torch.randint(0, cap, (B, Q, k), generator=g).numpy().astype(np.int32)
    return q, lat, lat_sc, swa, swa_sc, idx


def _dense(qvec, keys, scale):
    z = keys @ qvec * scale
    p = softmax(z)
    return p @ keys, logsumexp(z)


def _swa_rows(swa, swa_sc, b):
    return np.array([[oracle.e4m3_value(c) for c in row] for row in swa[b]], np.float64) * swa_sc[b][:, None]


def _mask_bounds():
    rows = []
    with open(os.path.join(GOLD, "replay_mask_cases.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(v) for v in line.split()])
    return rows


def test_dense_equivalence_when_k_covers_everything():
    """Pin (b): Top-K >= visible entries -> sparse attention = dense attention."""
    cap = 48
    q, lat, lat_sc, swa, swa_sc, _ = _case(1, cap=cap, T=0)
    idx = np.arange(cap, dtype=np.int32)[None, None, :]
    out, lse = oracle.sparse_attn(synth.bf16_bits(q), lat, lat_sc, np.array([cap], np.int32), idx,
                                  swa, swa_sc, np.array([0], np.int32), 128, None,
                                  np.array([[cap - 1]], np.int32))
    keys = oracle.dequant_nvfp4(lat[0], lat_sc[0])
    qd = q.double().numpy()
    for h in range(H):
        o, l = _dense(qd[0, 0, h], keys, 1 / math.sqrt(D))
        assert np.allclose(out[0, 0, h], o, rtol=1e-12, atol=1e-14)
        assert abs(lse[0, 0, h] - l) < 1e-10


def test_single_key_returns_value():
    q, lat, lat_sc, swa, swa_sc, _ = _case(2, cap=8, T=0)
    idx = np.array([[[5, -1, -1, 99]]], np.int32)  # -1 and out-of-range are padding
    out, lse = oracle.sparse_attn(synth.bf16_bits(q), lat, lat_sc, np.array([8], np.int32), idx,
                                  swa, swa_sc, np.array([0], np.int32), 128, None, np.array([[7]], np.int32))
    v = oracle.dequant_nvfp4(lat[0, 5:6], lat_sc[0, 5:6])[0]
    for h in range(H):
        assert np.array_equal(out[0, 0, h], v)
        assert abs(lse[0, 0, h] - float(q[0, 0, h].double() @ torch.from_numpy(v)) / math.sqrt(D)) < 1e-9


def test_uniform_logits_give_mean():
    q, lat, lat_sc, swa, swa_sc, idx = _case(3, cap=32, T=8, k=6)
    qz = torch.zeros_like(q)
    out, lse = oracle.sparse_attn(synth.bf16_bits(qz), lat, lat_sc, np.array([32], np.int32), idx,
                                  swa, swa_sc, np.array([0], np.int32), 128, None, np.array([[7]], np.int32))
    keys = np.concatenate([oracle.dequant_nvfp4(lat[0, idx[0, 0]], lat_sc[0, idx[0, 0]]), _swa_rows(swa, swa_sc, 0)])
    assert np.allclose(out[0, 0, 0], keys.mean(0), rtol=1e-12, atol=1e-15)
    assert abs(lse[0, 0, 0] - math.log(len(keys))) < 1e-12


@pytest.mark.parametrize("row", _mask_bounds())
def test_replay_mask_golden(row):
    """Pin (e): the replay mask matches the hand-worked table and a brute-force
    per-key visibility loop."""
    s, i, W, lo, hi = row
    T = 32
    pos0 = max(0, i - T + 1)
    g = torch.Generator().manual_seed(i)
    swa, swa_sc = synth.swa_kv(i, T, pos0)
    swa, swa_sc = swa.numpy()[None], swa_sc.numpy()[None]
    q = synth.attn_q(i, 1, 1)
    lat = np.zeros((1, 1, 256), np.uint8)
    lat_sc = np.zeros((1, 1, 32), np.uint8)
    idx = np.full((1, 1, 1), -1, np.int32)
    out, lse = oracle.sparse_attn(synth.bf16_bits(q), lat, lat_sc, np.array([0], np.int32), idx, swa, swa_sc,
                                  np.array([pos0], np.int32), W, np.array([s], np.int32), np.array([[i]], np.int32))
    visible = [tau for tau in range(pos0, pos0 + T) if tau <= i and tau >= i - W + 1 and tau >= s]
    assert visible == list(range(max(lo, pos0), hi + 1))
    rows = _swa_rows(swa, swa_sc, 0)[[tau - pos0 for tau in visible]]
    qd = q.double().numpy()[0, 0]
    for h in range(H):
        o, l = _dense(qd[h], rows, 1 / math.sqrt(D))
        assert np.allclose(out[0, 0, h], o, rtol=1e-12, atol=1e-14) and abs(lse[0, 0, h] - l) < 1e-10


def test_no_replay_start_is_plain_window():
    T, W = 20, 6
    swa, swa_sc = synth.swa_kv(5, T, 100)
    q = synth.attn_q(5, 1, 1)
    lat = np.zeros((1, 1, 256), np.uint8)
    lat_sc = np.zeros((1, 1, 32), np.uint8)
    idx = np.full((1, 1, 1), -1, np.int32)
    out, _ = oracle.sparse_attn(synth.bf16_bits(q), lat, lat_sc, np.array([0], np.int32), idx,
                                swa.numpy()[None], swa_sc.numpy()[None], np.array([100], np.int32), W, None,
                                np.array([[110]], np.int32))
    rows = _swa_rows(swa.numpy()[None], swa_sc.numpy()[None], 0)[105 - 100:111 - 100]
    o, _ = _dense(q.double().numpy()[0, 0, 3], rows, 1 / math.sqrt(D))
    assert np.allclose(out[0, 0, 3], o, rtol=1e-12, atol=1e-14)


def test_main_and_swa_share_one_softmax():
    q, lat, lat_sc, swa, swa_sc, idx = _case(6, cap=40, T=10, k=7)
    out, lse = oracle.sparse_attn(synth.bf16_bits(q), lat, lat_sc, np.array([40], np.int32), idx,
                                  swa, swa_sc, np.array([0], np.int32), 128, None, np.array([[9]], np.int32))
    keys = np.concatenate([oracle.dequant_nvfp4(lat[0, idx[0, 0]], lat_sc[0, idx[0, 0]]), _swa_rows(swa, swa_sc, 0)])
    qd = q.double().numpy()[0, 0]
    for h in (0, 15):
        o, l = _dense(qd[h], keys, 1 / math.sqrt(D))
        assert np.allclose(out[0, 0, h], o, rtol=1e-12, atol=1e-14) and abs(lse[0, 0, h] - l) < 1e-10


def test_layer_patterns_from_pages():
    consts = {}
    with open(os.path.join(GOLD, "page_constants.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                consts[line.split()[0]] = float(line.split()[1])
    assert len(oracle.DECODER_PATTERN) == consts["decoder_layers"]
    assert oracle.DECODER_PATTERN[:4] == ["full", "reuse", "reuse", "reuse"]
    assert all(oracle.DECODER_PATTERN[4 + 4 * g:8 + 4 * g] == ["reindex", "reuse", "reuse", "reuse"] for g in range(4))
    assert len(oracle.ENCODER_CSA2_PATTERN) == consts["encoder_csa2_layers"]
    fulls = oracle.DECODER_PATTERN.count("full") + oracle.ENCODER_CSA2_PATTERN.count("full")
    assert fulls == consts["full_layers_total"]


def test_reuse_equals_attention_with_borrowed_indices():
    """Pin (d): a Reuse layer's output is attention with the borrowed indices,
    its own query and its own SWA KV, bit for bit."""
    B, cap = 2, 200
    lat_bf = synth.latent(60, B * cap)
    lat, lat_sc = oracle.quant_nvfp4(synth.bf16_bits(lat_bf))
    W = synth.proj_w().numpy()
    ik, iks = oracle.index_k_proj(synth.bf16_bits(lat_bf), W)
    st = dict(lat=lat.reshape(B, cap, 256), lat_sc=lat_sc.reshape(B, cap, 32), ik=ik.reshape(B, cap, 32),
              iks=iks.reshape(B, cap, 4), n_entries=np.array([200, 150], np.int32), m=1, k=32)
    q_pos = np.array([[199], [149]], np.int32)

    def layer(seed):
        iq, iqs = oracle.quant_nvfp4(synth.bf16_bits(synth.index_q(seed, B, 1)).reshape(-1, 64))
        sw = [synth.swa_kv(seed * 7 + b, 16, int(q_pos[b, 0]) - 15) for b in range(B)]
        return dict(q=synth.bf16_bits(synth.attn_q(seed, B, 1)), iq=iq.reshape(B, 1, 128), iqs=iqs.reshape(B, 1, 16),
                    w=synth.index_w(B, 1).numpy(), swa=np.stack([s[0].numpy() for s in sw]),
                    swa_sc=np.stack([s[1].numpy() for s in sw]), swa_pos0=q_pos[:, 0] - 15, window=128,
                    q_pos=q_pos)

    full, reuse = layer(1), layer(2)
    oracle.layer_step("full", st, full)
    borrowed = st["idx"].copy()
    o1, l1 = oracle.layer_step("reuse", st, reuse)
    o2, l2 = oracle.sparse_attn(reuse["q"], st["lat"], st["lat_sc"], st["n_entries"], borrowed, reuse["swa"],
                                reuse["swa_sc"], reuse["swa_pos0"], 128, None, q_pos)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
