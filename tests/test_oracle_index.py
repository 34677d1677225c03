"""Pins of the oracle's indexer: projection, score, visibility, Top-K, pool (CPU only).

Independent references: exact rational arithmetic for the score, numpy float64
dot products of dequantised values (exact for these bit widths), Python's
sort for the Top-K / pool order, brute-force block maxima, and the pins the
pages fix (Top-K covering every visible entry; a pool covering every block).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth


def _rand_fp4(rng, rows, ch, scale_lo=0x20, scale_hi=0x50):
    codes = rng.integers(0, 256, (rows, ch // 2), dtype=np.uint8)
    scales = rng.integers(scale_lo, scale_hi, (rows, ch // 16), dtype=np.uint8)
    return codes, scales


def _exact_score(q, qs, w, k, ks):
    deq_q = oracle.dequant_nvfp4(q.reshape(4, 32), qs.reshape(4, 4))
    deq_k = oracle.dequant_nvfp4(k.reshape(1, 32), ks.reshape(1, 4))[0]
    total, mag = Fraction(0), Fraction(0)
    for h in range(4):
        d = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(deq_q[h], deq_k))
        total += Fraction(float(w[h])) * max(d, Fraction(0))
        mag += abs(Fraction(float(w[h]))) * sum(abs(Fraction(float(a)) * Fraction(float(b)))
                                                for a, b in zip(deq_q[h], deq_k))
    return total, mag


def test_score_close_to_exact_real_value():
    rng = np.random.default_rng(10)
    w = np.full(4, 0.25, np.float32)
    for _ in range(200):
        q, qs = _rand_fp4(rng, 4, 64)
        k, ks = _rand_fp4(rng, 1, 64)
        s = oracle.index_score(q, qs, w, k, ks)
        exact, mag = _exact_score(q, qs, w, k, ks)
        # 3 fp32 adds per head + 4 rounded products + 3 adds across heads
        assert abs(Fraction(float(s)) - exact) <= Fraction(10, 2 ** 24) * mag


def test_score_exact_when_no_rounding():
    """One live block per head and one live head: every fp32 step is exact."""
    rng = np.random.default_rng(11)
    w = np.array([0.25, 0.5, 1.0, 2.0], np.float32)
    for _ in range(100):
        q, qs = _rand_fp4(rng, 4, 64)
        k, ks = _rand_fp4(rng, 1, 64)
        live_h, live_b = rng.integers(0, 4), rng.integers(0, 4)
        qz = np.zeros_like(q)
        qz[live_h, 8 * live_b:8 * live_b + 8] = q[live_h, 8 * live_b:8 * live_b + 8]
        s = oracle.index_score(qz, qs, w, k, ks)
        exact, _ = _exact_score(qz, qs, w, k, ks)
        assert Fraction(float(s)) == exact


def test_score_block_scale_mapping_float64_dot():
    """d_h must equal the float64 dot product of the dequantised vectors whenever the
    fp32 block sums are exact (one live block): pins nibble order, block/scale
    mapping and the factor-of-4 bookkeeping."""
    rng = np.random.default_rng(12)
    w = np.array([1.0, 0.0, 0.0, 0.0], np.float32)
    for _ in range(100):
        q, qs = _rand_fp4(rng, 4, 64)
        k, ks = _rand_fp4(rng, 1, 64)
        b = rng.integers(0, 4)
        qz = np.zeros_like(q)
        qz[0, 8 * b:8 * b + 8] = q[0, 8 * b:8 * b + 8]
        dq = oracle.dequant_nvfp4(qz, qs)[0]
        dk = oracle.dequant_nvfp4(k, ks)[0]
        ref = max(float(np.dot(dq, dk)), 0.0)
        assert oracle.index_score(qz, qs, w, k, ks) == np.float32(ref)


def test_score_relu_and_sign():
    rng = np.random.default_rng(13)
    w = np.full(4, 0.25, np.float32)
    q, qs = _rand_fp4(rng, 4, 64)
    k, ks = _rand_fp4(rng, 1, 64)
    s = oracle.index_score(q, qs, w, k, ks)
    qn = q ^ 0x88  # flip every sign bit: each head's d changes sign
    sn = oracle.index_score(qn, qs, w, k, ks)
    deq_q = oracle.dequant_nvfp4(q, qs)
    dk = oracle.dequant_nvfp4(k, ks)[0]
    d = deq_q @ dk
    assert (s > 0) == bool((d > 0).any()) and (sn > 0) == bool((d < 0).any())


def test_projection_fma_chain_close_to_float64():
    x = synth.latent(21, 64)
    W = synth.proj_w().numpy()
    bits = synth.bf16_bits(x)
    got = oracle.index_k_proj_f32(bits, W)
    ref = x.double().numpy() @ W.astype(np.float64)
    bound = (np.abs(x.double().numpy()) @ np.abs(W.astype(np.float64))) * 512 * 2.0 ** -24
    assert np.all(np.abs(got - ref) <= bound)
    # a single non-zero channel is exact
    xs = torch.zeros((1, 512), dtype=torch.bfloat16)
    xs[0, 37] = 1.5
    g1 = oracle.index_k_proj_f32(synth.bf16_bits(xs), W)
    assert np.array_equal(g1[0], (W[37] * np.float32(1.5)).astype(np.float32))
    codes, scales = oracle.index_k_proj(bits, W)
    c2, s2 = oracle.quant_nvfp4(got)
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2)


@pytest.mark.parametrize("m", [1, 2])
def test_visibility_brute_force(m):
    for p in range(0, 40):
        for n in (0, 1, 5, 17, 100):
            want = sum(1 for e in range(n) if m * e + m - 1 <= p)
            assert oracle.n_visible(p, n, m) == want


def _make_index_case(seed, B, Q, cap, n_entries, dup=False):
    rng = np.random.default_rng(seed)
    q, qs = _rand_fp4(rng, B * Q * 4, 64)
    q = q.reshape(B, Q, 128)
    qs = qs.reshape(B, Q, 16)
    ik, iks = _rand_fp4(rng, B * cap, 64)
    ik = ik.reshape(B, cap, 32)
    iks = iks.reshape(B, cap, 4)
    if dup:  # many identical keys -> exact score ties
        ik[:, 1::3] = ik[:, 0:1]
        iks[:, 1::3] = iks[:, 0:1]
    w = np.full((B, Q, 4), 0.25, np.float32)
    return q, qs, w, ik, iks, np.array(n_entries, np.int32)


def _brute_topk(scores, k):
    order = sorted(range(len(scores)), key=lambda t: (-scores[t], t))[:k]
    return sorted(order) + [-1] * (k - min(k, len(scores)))


@pytest.mark.parametrize("dup", [False, True])
@pytest.mark.parametrize("m", [1, 2])
def test_index_topk_brute_force(dup, m):
    B, Q, cap = 2, 3, 300
    q, qs, w, ik, iks, ne = _make_index_case(20 + m, B, Q, cap, [300, 211], dup)
    q_pos = np.array([[299 * m, 150, 40], [10, 600, 421]], np.int32)
    k = 37
    idx, bm = oracle.index_topk(q, qs, w, ik, iks, ne, m, q_pos, k, blockmax=True)
    for b in range(B):
        for qi in range(Q):
            nv = oracle.n_visible(q_pos[b, qi], ne[b], m)
            sc = [oracle.index_score(q[b, qi], qs[b, qi], w[b, qi], ik[b, t], iks[b, t]) for t in range(nv)]
            assert list(idx[b, qi]) == _brute_topk(sc, k)
            # block maxima over visible positions; -inf past the last visible block
            for j in range(bm.shape[-1]):
                vals = sc[8 * j:8 * j + 8]
                assert bm[b, qi, j] == (max(vals) if vals else -np.inf)


def test_topk_all_visible_when_k_large():
    """Pin (b), index half: K >= visible entries returns every visible entry."""
    q, qs, w, ik, iks, ne = _make_index_case(30, 1, 1, 64, [64])
    idx = oracle.index_topk(q, qs, w, ik, iks, ne, 1, np.array([[40]], np.int32), 512)
    assert list(idx[0, 0, :41]) == list(range(41)) and np.all(idx[0, 0, 41:] == -1)


def test_topk_all_zero_scores_prefers_low_positions():
    q, qs, w, ik, iks, ne = _make_index_case(31, 1, 1, 100, [100])
    q[:] = 0  # every score is +0
    idx = oracle.index_topk(q, qs, w, ik, iks, ne, 1, np.array([[99]], np.int32), 10)
    assert list(idx[0, 0]) == list(range(10))


def test_pool_build_brute_force_and_inclusion():
    B, Q, cap = 1, 2, 900
    q, qs, w, ik, iks, ne = _make_index_case(40, B, Q, cap, [900], dup=True)
    q_pos = np.array([[899, 500]], np.int32)
    k, P = 16, 20
    idx, bm = oracle.index_topk(q, qs, w, ik, iks, ne, 1, q_pos, k, blockmax=True)
    pool = oracle.pool_build(bm, ne, 1, q_pos, P)
    for qi in range(Q):
        nv = oracle.n_visible(q_pos[0, qi], 900, 1)
        nblk = (nv + 7) // 8
        want = _brute_topk([float(v) for v in bm[0, qi, :nblk]], P)
        assert list(pool[0, qi]) == want
        # every block holding a Top-K pick is in the pool (P >= k)
        assert set(int(t) // 8 for t in idx[0, qi] if t >= 0) <= set(int(b) for b in pool[0, qi] if b >= 0)


def test_pool_covering_all_blocks_equals_unrestricted():
    """Pin (c): a pool that holds every block gives the same indices as a full search."""
    B, Q, cap = 2, 2, 1000
    q, qs, w, ik, iks, ne = _make_index_case(41, B, Q, cap, [1000, 777], dup=True)
    q_pos = np.array([[999, 300], [776, 5]], np.int32)
    k = 64
    idx, bm = oracle.index_topk(q, qs, w, ik, iks, ne, 1, q_pos, k, blockmax=True)
    pool = oracle.pool_build(bm, ne, 1, q_pos, 2048)
    rq, rqs = _rand_fp4(np.random.default_rng(42), B * Q * 4, 64)  # the Reindex layer's own query
    rq, rqs = rq.reshape(B, Q, 128), rqs.reshape(B, Q, 16)
    a = oracle.pool_topk(rq, rqs, w, ik, iks, ne, 1, pool, q_pos, k)
    b = oracle.index_topk(rq, rqs, w, ik, iks, ne, 1, q_pos, k)
    assert np.array_equal(a, b)


def test_pool_topk_brute_force():
    B, Q, cap = 1, 1, 4096
    q, qs, w, ik, iks, ne = _make_index_case(43, B, Q, cap, [4096])
    q_pos = np.array([[4095]], np.int32)
    rng = np.random.default_rng(44)
    blocks = np.sort(rng.choice(512, 30, replace=False)).astype(np.int32)
    pool = np.full((1, 1, 40), -1, np.int32)
    pool[0, 0, :30] = blocks
    k = 50
    got = oracle.pool_topk(q, qs, w, ik, iks, ne, 1, pool, q_pos, k)
    cand = [int(8 * b + j) for b in blocks for j in range(8)]
    sc = {t: oracle.index_score(q[0, 0], qs[0, 0], w[0, 0], ik[0, t], iks[0, t]) for t in cand}
    want = sorted(sorted(cand, key=lambda t: (-sc[t], t))[:k])
    assert list(got[0, 0]) == want
