"""GPU parity of every call of the C ABI against the CPU oracle (small and ragged cases).

Bit-exact: quantised bytes, indexer-K bytes, Top-K indices, block maxima, pools.
Tolerance (attention, bf16 out): |gpu - ref| <= 2e-3 + 1e-2 |ref| elementwise.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import (SM_SCALE, Group, attn_close, bits, ik_untile, index_query, kv_ik_rows, np_, set_kv_ik_rows,
                        swa_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    import sparse_attention_fp4_quant_b200 as m
    m.lib()
    return m


# ---------------------------------------------------------------- quantisation
def test_quant_exhaustive_bf16(csa):
    """Every finite bf16 pattern appears in some group, next to every kind of amax."""
    allb = np.arange(0, 1 << 16, dtype=np.uint32)
    finite = allb[((allb >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    rng = np.random.default_rng(0)
    groups = []
    for rot in range(3):
        perm = rng.permutation(finite)
        pad = (-perm.size) % 16
        groups.append(np.concatenate([perm, perm[:pad]]).reshape(-1, 16))
    x = np.concatenate(groups)
    pad_rows = (-x.shape[0]) % 32
    x = np.concatenate([x, x[:pad_rows]]).reshape(-1, 512)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    c, s = csa.csa2_quant_nvfp4(xt)
    oc, os_ = oracle.quant_nvfp4(x)
    assert np.array_equal(np_(s), os_)
    assert np.array_equal(np_(c), oc)


def test_quant_special_groups(csa):
    vals = [0.0, -0.0, 1e-30, -1e-30, 448 * 6.0, 448 * 7.5, 3e38, -3e38, 0.25, 0.75, 1.25, 5.0, -5.0]
    rows = []
    for v in vals:
        g = np.zeros(16, np.float32)
        g[0] = v
        g[1:] = np.float32(v) * np.array([0.5, 0.25, 0.125, 1.0, -1.0, 0.7, 0.1, 0, -0.0, 0.33, 0.9, 0.99, 0.6, 0.4,
                                          0.2], np.float32)
        rows.append(g)
    x = torch.tensor(np.stack(rows)).to(torch.bfloat16).reshape(-1, 16)
    x = torch.cat([x, torch.zeros((3, 16), dtype=torch.bfloat16)]).reshape(-1, 16)
    xc = x.cuda().contiguous()
    c, s = csa.csa2_quant_nvfp4(xc)
    oc, os_ = oracle.quant_nvfp4(bits(x))
    assert np.array_equal(np_(s), os_) and np.array_equal(np_(c), oc)


@pytest.mark.parametrize("ch", [16, 64, 512, 4096])
def test_quant_latents_and_dst_rows(csa, ch):
    x = synth.normal(ch, (300, ch), "cuda").to(torch.bfloat16)
    c, s = csa.csa2_quant_nvfp4(x)
    oc, os_ = oracle.quant_nvfp4(bits(x))
    assert np.array_equal(np_(c), oc) and np.array_equal(np_(s), os_)
    # scatter into a larger buffer at given rows
    dst = torch.randperm(1000, device="cuda")[:300].to(torch.int64)
    big_c = torch.zeros((1000, ch // 2), dtype=torch.uint8, device="cuda")
    big_s = torch.zeros((1000, ch // 16), dtype=torch.uint8, device="cuda")
    csa.csa2_quant_nvfp4(x, big_c, big_s, dst)
    assert np.array_equal(np_(big_c)[np_(dst)], oc) and np.array_equal(np_(big_s)[np_(dst)], os_)


def test_index_k_proj_bit_exact(csa):
    x = synth.latent(5, 1000, 0, "cuda")
    W = synth.proj_w(3).cuda()
    kc, ks = csa.csa2_index_k_proj(x, W)   # 1024 rows: whole tiles of the cache order
    assert kc.shape == (1024, 32)
    oc, os_ = oracle.index_k_proj(bits(x), np_(W))
    gc, gs = ik_untile(np_(kc), np_(ks))
    assert np.array_equal(gc[:1000], oc) and np.array_equal(gs[:1000], os_)
    dst = (torch.arange(1000, device="cuda", dtype=torch.int64) * 3 + 1)
    bc = torch.zeros((3072, 32), dtype=torch.uint8, device="cuda")
    bs = torch.zeros((3072, 4), dtype=torch.uint8, device="cuda")
    csa.csa2_index_k_proj(x, W, bc, bs, dst)
    gc, gs = ik_untile(np_(bc), np_(bs))
    assert np.array_equal(gc[1::3][:1000], oc) and np.array_equal(gs[1::3][:1000], os_)
    with pytest.raises(RuntimeError):   # output rows must be whole tiles
        csa.csa2_index_k_proj(x, W, bc[:3001], bs[:3001], dst)


@pytest.mark.parametrize("rows", [1, 32, 45, 2049])
def test_append_tokens_bit_exact(csa, rows):
    # one launch = csa2_quant_nvfp4 + csa2_index_k_proj of the same rows (2049: the two-launch path)
    x = synth.latent(synth.seed_of("append", rows), rows, 100, "cuda")
    W = synth.proj_w(rows).cuda()
    lb = bits(x)
    olc, ols = oracle.quant_nvfp4(lb)
    okc, oks = oracle.index_k_proj(lb, np_(W))
    out_rows = (3 * rows + 1 + 127) // 128 * 128   # whole tiles of the indexer-K order
    dst = torch.arange(rows, device="cuda", dtype=torch.int64) * 3 + 1
    lc = torch.zeros((out_rows, 256), dtype=torch.uint8, device="cuda")
    ls = torch.zeros((out_rows, 32), dtype=torch.uint8, device="cuda")
    kc = torch.zeros((out_rows, 32), dtype=torch.uint8, device="cuda")
    ks = torch.zeros((out_rows, 4), dtype=torch.uint8, device="cuda")
    csa.csa2_append_tokens(x, W, (lc, ls, kc, ks), dst)
    assert np.array_equal(np_(lc)[1::3][:rows], olc) and np.array_equal(np_(ls)[1::3][:rows], ols)
    gkc, gks = ik_untile(np_(kc), np_(ks))
    assert np.array_equal(gkc[1::3][:rows], okc) and np.array_equal(gks[1::3][:rows], oks)
    untouched = np.ones(out_rows, bool)
    untouched[1::3][:rows] = False
    assert not np_(lc)[untouched].any() and not gkc[untouched].any() and not gks[untouched].any()


# ---------------------------------------------------------------- index / Top-K
def _index_case(seed, B, Q, cap, n_entries, m, q_pos, k, rows=None):
    grp = Group(seed, B, cap, n_entries, m, rows=rows)
    o = grp.oracle_cache()
    gik, giks = kv_ik_rows(grp.kv)
    assert np.array_equal(gik, o["ik"]) and np.array_equal(giks, o["iks"])
    iq, iqs, w, oiq, oiqs, ow = index_query(seed + 1, B, Q)
    assert np.array_equal(np_(iq), oiq) and np.array_equal(np_(iqs), oiqs)
    qp = torch.tensor(q_pos, dtype=torch.int32, device="cuda")
    return grp, o, iq, iqs, w, oiq, oiqs, ow, qp


@pytest.mark.parametrize("m", [1, 2])
@pytest.mark.parametrize("k", [1, 37, 512, 2048])
def test_index_topk_ragged(csa, m, k):
    B, Q, cap = 3, 2, 9088
    n_entries = [9000, 4097, 1]
    q_pos = [[9000 * m - 1, 3000], [4096 * m + 50, 511], [0, 77]]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(11 * m + k, B, Q, cap, n_entries, m, q_pos, k)
    idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, k, blockmax=True)
    ridx, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, m, np.array(q_pos, np.int32), k,
                                  blockmax=True)
    assert np.array_equal(np_(idx), ridx)
    assert np.array_equal(np_(bm), rbm)


@pytest.mark.parametrize("B,Q", [(2, 80), (1, 150)])
def test_index_topk_many_queries(csa, B, Q):
    # more queries than one wave of clusters holds: the many-query kernels serve
    # them (prefill-like causal positions; 150 = 18 groups of 8 and one of 6)
    cap, m, k = 3072, 2, 512
    n_entries = [3000, 2100][:B]
    rng = np.random.default_rng(5 + Q)
    q_pos = rng.integers(0, 6000, size=(B, Q)).astype(np.int32)
    q_pos[0, :4] = [0, 1, 1023, 5999]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(77 + Q, B, Q, cap, n_entries, m, q_pos.tolist(), k)
    idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, k, blockmax=True)
    ridx, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, m, q_pos, k, blockmax=True)
    assert np.array_equal(np_(idx), ridx)
    assert np.array_equal(np_(bm), rbm)


def test_index_topk_many_queries_large_cache(csa):
    # the many-query path above 65,536 entries: 152 queries = 19 groups of 8, so the
    # scoring splits each group's entry range into 7 shares whose histograms add up,
    # and the selector keeps 131,072-entry position bitmaps
    B, Q, cap, m, k = 1, 152, 131072, 1, 512
    rng = np.random.default_rng(57)
    q_pos = np.sort(rng.integers(0, 130000, size=(B, Q))).astype(np.int32)
    q_pos[0, :5] = [0, 7, 127, 65535, 65536]
    q_pos[0, -3:] = [129998, 129999, 129999]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(151, B, Q, cap, [130000], m, q_pos.tolist(), k)
    idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, k, blockmax=True)
    ridx, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, m, q_pos, k, blockmax=True)
    assert np.array_equal(np_(idx), ridx)
    assert np.array_equal(np_(bm).view(np.uint32), rbm.view(np.uint32))


def test_index_topk_shares_with_keys_in_workspace(csa):
    # 8 decode queries over a cache sized above 16 x 32,768 entries: the workspace holds
    # every order key, eight 16-CTA clusters do not fit at once, so the per-share kernel
    # keeps its keys there and selects through a histogram (short ragged caches: shares
    # with no entries, ragged tails; one query with zero weights ties every score)
    B, Q, m = 8, 1, 1
    cap = 524288 + 128
    n_entries = [30000, 1, 129, 5000, 45000, 20000, 7, 44000]
    q_pos = [[n - 1] for n in n_entries]
    q_pos[4] = [40000]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(171, B, Q, cap, n_entries, m, q_pos, 512, rows=45056)
    w[5] = 0.0
    ow = np_(w)
    assert csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, B, Q, cap, 512, 0) >= B * cap * 4   # the keys' space
    for k in (512, 2048):
        idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, k, blockmax=True)
        ridx, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, m, np.array(q_pos, np.int32),
                                      k, blockmax=True)
        assert np.array_equal(np_(idx), ridx), k
        assert np.array_equal(np_(bm).view(np.uint32), rbm.view(np.uint32)), k


def test_index_topk_many_queries_threshold_bin_overflow(csa):
    # all-tie queries on the many-query path: with zero query codes or zero head
    # weights every visible score is +0, so the threshold bin holds every visible
    # entry (up to 8,000 > the selector's 4,096-entry candidate list) and the
    # selector resolves it with its re-scoring passes; the other queries are normal
    B, Q, cap, m = 1, 160, 8192, 1
    rng = np.random.default_rng(31)
    q_pos = rng.integers(3000, 8000, size=(B, Q)).astype(np.int32)
    q_pos[0, :6] = [7999, 4096, 4095, 5000, 100, 0]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(131, B, Q, cap, [8000], m, q_pos.tolist(), 512)
    zero_q = [0, 1, 2, 3, 17, 90, 159]
    zero_w = [4, 5, 40, 41, 150]
    iq[0, zero_q] = 0
    oiq = oiq.copy()
    oiq[0, zero_q] = 0
    w[0, zero_w] = 0.0
    ow = np_(w)
    for k in (512, 2048):
        idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, k, blockmax=True)
        ridx, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, m, q_pos, k, blockmax=True)
        assert np.array_equal(np_(idx), ridx)
        assert np.array_equal(np_(bm).view(np.uint32), rbm.view(np.uint32))
        for qi in zero_q + zero_w:
            nv = min(int(q_pos[0, qi]) + 1, 8000)
            assert list(np_(idx)[0, qi, :min(k, nv)]) == list(range(min(k, nv)))


@pytest.mark.parametrize("n", [128, 129, 255, 1001])
def test_index_topk_small_ragged_caches(csa, n):
    # visible ranges of a tile, just over one, one short of two, and ragged: the
    # cluster kernel's last tile and the per-share kernel's last stage
    B, Q, m = 2, 1, 1
    cap = (n + 127) // 128 * 128
    n_entries = [n, max(1, n - 3)]
    q_pos = [[n - 1], [n - 4]]
    for k in (64, 512):
        grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(90 + n % 7, B, Q, cap, n_entries, m, q_pos, k)
        idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, k, blockmax=True)
        ridx, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, m, np.array(q_pos, np.int32),
                                      k, blockmax=True)
        assert np.array_equal(np_(idx), ridx)
        assert np.array_equal(np_(bm), rbm)


def test_kv_capacity_must_be_whole_tiles(csa):
    with pytest.raises(ValueError):
        csa.KV(1, 1000, 1, "cuda")


def test_index_blockmax_signed_zero_and_negative_weights(csa):
    # negative head weights make scores <= 0, with -0 and +0 in the same block;
    # a block maximum keeps the first of equal values in position order
    B, Q, cap, m, k = 1, 2, 4096, 1, 512
    q_pos = [[3999, 2500]]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(95, B, Q, cap, [4000], m, q_pos, k)
    w = torch.tensor([[[-0.25, 0.5, -0.75, 0.125], [-1.0, -0.5, -0.25, -0.125]]], dtype=torch.float32, device="cuda")
    idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, k, blockmax=True)
    ridx, rbm = oracle.index_topk(oiq, oiqs, np_(w), o["ik"], o["iks"], grp.n_entries, m, np.array(q_pos, np.int32),
                                  k, blockmax=True)
    assert np.array_equal(np_(idx), ridx)
    assert np.array_equal(np_(bm).view(np.uint32), rbm.view(np.uint32))   # bits, so -0 != +0


def test_index_scores_extreme_block_scales(csa):
    # block scales at the ends of E4M3 (subnormal 2^-9 .. 448) on keys and queries, mixed within
    # a row: each accumulator column of the block-scaled MMA holds one block, so the scores (seen
    # directly through the block maxima) stay bit-exact whatever the exponent spread
    B, Q, cap, k = 1, 2, 4096, 512
    rng = np.random.default_rng(17)
    grp = Group(18, B, cap, [cap])
    o = {kk: v.copy() for kk, v in grp.oracle_cache().items()}
    extremes = np.array([0x01, 0x02, 0x08, 0x30, 0x40, 0x77, 0x7E], np.uint8)
    iks = extremes[rng.integers(0, len(extremes), size=(B, cap, 4))].astype(np.uint8)
    o["iks"] = iks
    set_kv_ik_rows(grp.kv, o["ik"], iks)
    iq, iqs, w, oiq, oiqs, ow = index_query(19, B, Q)
    qsc = extremes[rng.integers(0, len(extremes), size=(B, Q, 16))].astype(np.uint8)
    oiqs = qsc
    iqs.copy_(torch.from_numpy(qsc))
    q_pos = np.array([[cap - 1, cap // 2]], np.int32)
    idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, torch.from_numpy(q_pos).cuda(), k, blockmax=True)
    ridx, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, 1, q_pos, k, blockmax=True)
    assert np.array_equal(np_(bm).view(np.uint32), rbm.view(np.uint32))
    assert np.array_equal(np_(idx), ridx)


def test_index_topk_ties_and_zero_scores(csa):
    B, Q, cap = 1, 3, 20096
    grp = Group(21, B, cap, [20000])
    # duplicate one key everywhere in a stripe: many exactly equal scores
    gik, giks = kv_ik_rows(grp.kv)
    gik[0, 1000:9000] = gik[0, 5]
    giks[0, 1000:9000] = giks[0, 5]
    set_kv_ik_rows(grp.kv, gik, giks)
    o = grp.oracle_cache()
    o = dict(o)
    o["ik"] = o["ik"].copy()
    o["iks"] = o["iks"].copy()
    o["ik"][0, 1000:9000] = o["ik"][0, 5]
    o["iks"][0, 1000:9000] = o["iks"][0, 5]
    iq, iqs, w, oiq, oiqs, ow = index_query(22, B, Q)
    iq[0, 2].zero_()   # query 2 scores every entry +0
    oiq = oiq.copy()
    oiq[0, 2] = 0
    q_pos = np.array([[19999, 15000, 19999]], np.int32)
    for k in (512, 2048):
        idx = csa.csa2_index_topk(iq, iqs, w, grp.kv, torch.from_numpy(q_pos).cuda(), k)
        ridx = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, 1, q_pos, k)
        assert np.array_equal(np_(idx), ridx)
        assert list(np_(idx)[0, 2]) == list(range(k))


def test_index_topk_ties_at_threshold_across_ctas(csa):
    # 400 copies of a high-scoring key and 600 of a slightly lower one, spread over
    # the whole range: the threshold is the lower key, its ties are split over the
    # cluster's CTAs and the lowest positions must win.  The threshold bin stays
    # small, so the gathered-candidate select decides it.
    B, Q, cap, k = 1, 1, 65536, 512
    grp = Group(23, B, cap, [cap])
    o = grp.oracle_cache()
    iq, iqs, w, oiq, oiqs, ow = index_query(24, B, Q)
    sc = np.array([oracle.index_score(oiq[0, 0], oiqs[0, 0], ow[0, 0], o["ik"][0, e], o["iks"][0, e])
                   for e in range(0, cap, 61)], np.float64)
    top = np.argsort(-sc)[:2] * 61                  # two of the best entries of a sample
    hi, lo = (int(top[0]), int(top[1])) if sc[top[0] // 61] > sc[top[1] // 61] else (int(top[1]), int(top[0]))
    assert sc[hi // 61] > sc[lo // 61]
    rng = np.random.default_rng(25)
    pos = rng.permutation(cap)
    pos = pos[(pos != hi) & (pos != lo)]
    gik, giks = kv_ik_rows(grp.kv)
    oik, oiks = o["ik"].copy(), o["iks"].copy()
    for dst, src in ((pos[:400], hi), (pos[400:1000], lo)):
        gik[0, dst], giks[0, dst] = gik[0, src], giks[0, src]
        oik[0, dst], oiks[0, dst] = oik[0, src], oiks[0, src]
    set_kv_ik_rows(grp.kv, gik, giks)
    q_pos = np.array([[cap - 1]], np.int32)
    idx = csa.csa2_index_topk(iq, iqs, w, grp.kv, torch.from_numpy(q_pos).cuda(), k)
    ridx = oracle.index_topk(oiq, oiqs, ow, oik, oiks, grp.n_entries, 1, q_pos, k)
    assert np.array_equal(np_(idx), ridx)
    assert np.isin(np.concatenate([pos[:400], [hi]]), ridx).all()   # every copy of the higher key


def test_device_error_flag_stays_clear(csa):
    B, Q, cap, k = 2, 1, 3072, 64
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(31, B, Q, cap, [3000, 2000], 1, [[2999], [1999]], k)
    ws = torch.zeros(csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, B, Q, cap, k), dtype=torch.uint8, device="cuda")
    idx = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, k, ws=ws)
    torch.cuda.synchronize()
    assert csa.device_error_flag(ws, B, Q) == 0
    csa.csa2_device_status(ws, B, Q)   # raises on CSA2_ERR_TIMEOUT
    ridx = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, 1, np.array([[2999], [1999]], np.int32), k)
    assert np.array_equal(np_(idx), ridx)


def test_binding_rejects_mismatched_shapes(csa):
    kv = csa.KV(1, 128, 1, "cuda")
    q = torch.zeros((2, 1, 128), dtype=torch.uint8, device="cuda")
    qs = torch.zeros((2, 1, 16), dtype=torch.uint8, device="cuda")
    w = torch.zeros((2, 1, 4), dtype=torch.float32, device="cuda")
    qp = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):   # two query rows, one cache row
        csa.csa2_index_topk(q, qs, w, kv, qp, 8)
    with pytest.raises(ValueError):   # q of the wrong size
        csa.csa2_index_topk(q[:1, :, :64].contiguous(), qs[:1], w[:1], kv, qp[:1], 8)


# ---------------------------------------------------------------- pool
def test_pool_build_and_pool_topk(csa):
    B, Q, cap = 2, 2, 30080
    n_entries = [30000, 17001]
    q_pos = [[29999, 20000], [17000, 9]]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(31, B, Q, cap, n_entries, 1, q_pos, 512)
    idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, 512, blockmax=True)
    _, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, 1, np.array(q_pos, np.int32), 512,
                               blockmax=True)
    assert np.array_equal(np_(bm), rbm)
    for P in (2048, 300):
        pool = csa.csa2_pool_build(bm, grp.kv, qp, P)
        rpool = oracle.pool_build(rbm, grp.n_entries, 1, np.array(q_pos, np.int32), P)
        assert np.array_equal(np_(pool), rpool)
        riq, riqs, rw, roiq, roiqs, row_ = index_query(32 + P, B, Q)
        for k in (512, 64):
            got = csa.csa2_pool_topk(riq, riqs, rw, grp.kv, pool, qp, k)
            ref = oracle.pool_topk(roiq, roiqs, row_, o["ik"], o["iks"], grp.n_entries, 1, rpool,
                                   np.array(q_pos, np.int32), k)
            assert np.array_equal(np_(got), ref)


def test_pool_topk_through_layer_step(csa):
    """The Reindex layer of csa2_layer_step searches a pool csa2_pool_build wrote (block ids
    ascending) with the cluster select: indices equal the oracle's, also for a query whose
    weights are all zero (every score +0, so the lowest positions win every tie)."""
    B, Q, cap, T = 4, 1, 30080, 128
    n_entries = [30000, 17001, 29000, 25000]
    q_pos = [[29999], [17000], [28999], [24000]]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(33, B, Q, cap, n_entries, 1, q_pos, 512)
    _, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, 512, blockmax=True)
    _, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, 1, np.array(q_pos, np.int32), 512,
                               blockmax=True)
    pos0 = [n - T for n in n_entries]
    swa, swa_sc = swa_for(34, B, T, pos0)
    p0 = torch.tensor(pos0, dtype=torch.int32, device="cuda")
    q = synth.attn_q(35, B, Q, "cuda")
    for P in (2048, 300):
        pool = csa.csa2_pool_build(bm, grp.kv, qp, P)
        rpool = oracle.pool_build(rbm, grp.n_entries, 1, np.array(q_pos, np.int32), P)
        assert np.array_equal(np_(pool), rpool)
        for zero_w in (False, True):
            riq, riqs, rw, roiq, roiqs, row_ = index_query(36 + P, B, Q)
            if zero_w:
                rw.zero_()
                row_ = np.zeros_like(row_)
            idx = torch.full((B, Q, 512), -7, dtype=torch.int32, device="cuda")
            csa.csa2_layer_step("reindex", grp.kv, qp, q, swa, swa_sc, p0, idx, 512, riq, riqs, rw, pool=pool)
            ref = oracle.pool_topk(roiq, roiqs, row_, o["ik"], o["iks"], grp.n_entries, 1, rpool,
                                   np.array(q_pos, np.int32), 512)
            assert np.array_equal(np_(idx), ref), (P, zero_w)


def test_pool_topk_many_queries_layer_step(csa):
    """Pool build and Reindex for many queries (one CTA per query: the radix select over the
    block maxima; the pool search with its order keys in the workspace and a histogram
    pre-selection): pools and indices equal the oracle's for pools of 2,048 and 300 blocks,
    queries that see a few blocks only, and all-zero weights (every score +0: one histogram
    bin holds every entry, so the exact Top-K has to make room as it fills; for the build,
    every block maximum ties and the lowest blocks win)."""
    B, Q, cap, T = 2, 80, 30080, 128
    n_entries = [30000, 22001]
    q_pos = [[n_entries[b] - 1 - 97 * j for j in range(Q)] for b in range(B)]
    q_pos[1][-3:] = [5, 700, 4100]
    grp, o, iq, iqs, w, oiq, oiqs, ow, qp = _index_case(41, B, Q, cap, n_entries, 1, q_pos, 512)
    _, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, 512, blockmax=True)
    _, rbm = oracle.index_topk(oiq, oiqs, ow, o["ik"], o["iks"], grp.n_entries, 1, np.array(q_pos, np.int32), 512,
                               blockmax=True)
    assert np.array_equal(np_(bm), rbm)
    w0 = torch.zeros_like(w)
    _, bm0 = csa.csa2_index_topk(iq, iqs, w0, grp.kv, qp, 512, blockmax=True)
    _, rbm0 = oracle.index_topk(oiq, oiqs, np.zeros_like(ow), o["ik"], o["iks"], grp.n_entries, 1,
                                np.array(q_pos, np.int32), 512, blockmax=True)
    assert np.array_equal(np_(bm0), rbm0)
    for P in (2048, 300):
        pool0 = csa.csa2_pool_build(bm0, grp.kv, qp, P)
        assert np.array_equal(np_(pool0), oracle.pool_build(rbm0, grp.n_entries, 1, np.array(q_pos, np.int32), P)), P
    pos0 = [n - T for n in n_entries]
    swa, swa_sc = swa_for(42, B, T, pos0)
    p0 = torch.tensor(pos0, dtype=torch.int32, device="cuda")
    q = synth.attn_q(43, B, Q, "cuda")
    for P in (2048, 300):
        pool = csa.csa2_pool_build(bm, grp.kv, qp, P)
        rpool = oracle.pool_build(rbm, grp.n_entries, 1, np.array(q_pos, np.int32), P)
        assert np.array_equal(np_(pool), rpool)
        for zero_w in (False, True):
            riq, riqs, rw, roiq, roiqs, row_ = index_query(44 + P, B, Q)
            if zero_w:
                rw.zero_()
                row_ = np.zeros_like(row_)
            idx = torch.full((B, Q, 512), -7, dtype=torch.int32, device="cuda")
            csa.csa2_layer_step("reindex", grp.kv, qp, q, swa, swa_sc, p0, idx, 512, riq, riqs, rw, pool=pool)
            ref = oracle.pool_topk(roiq, roiqs, row_, o["ik"], o["iks"], grp.n_entries, 1, rpool,
                                   np.array(q_pos, np.int32), 512)
            assert np.array_equal(np_(idx), ref), (P, zero_w)


# ---------------------------------------------------------------- attention
def _attn_case(csa, seed, B, Q, cap, n_entries, k, T, window, q_pos, pos0, replay, idx_np):
    grp = Group(seed, B, cap, n_entries)
    o = grp.oracle_cache()
    assert np.array_equal(np_(grp.kv.lat), o["lat"]) and np.array_equal(np_(grp.kv.lat_sc), o["lat_sc"])
    q = synth.attn_q(seed, B, Q, "cuda")
    swa, swa_sc = swa_for(seed, B, T, pos0)
    qp = torch.tensor(q_pos, dtype=torch.int32, device="cuda")
    p0 = torch.tensor(pos0, dtype=torch.int32, device="cuda")
    rs = None if replay is None else torch.tensor(replay, dtype=torch.int32, device="cuda")
    idx = torch.from_numpy(idx_np).cuda()
    out, lse = csa.csa2_sparse_attn(q, grp.kv, idx, swa, swa_sc, p0, qp, window, rs, SM_SCALE, lse=True)
    ref, rlse = oracle.sparse_attn(bits(q), o["lat"], o["lat_sc"], grp.n_entries, idx_np, np_(swa), np_(swa_sc),
                                   np.array(pos0, np.int32), window, None if replay is None else np.array(replay, np.int32),
                                   np.array(q_pos, np.int32), SM_SCALE)
    ok, st = attn_close(out, ref)
    assert ok, st
    fin = np.isfinite(rlse)
    assert np.array_equal(fin, np.isfinite(np_(lse)))
    assert np.allclose(np_(lse)[fin], rlse[fin], rtol=1e-4, atol=1e-4)
    return st


@pytest.mark.parametrize("B,Q", [(1, 1), (3, 2), (32, 1)])
def test_sparse_attn_decode(csa, B, Q):
    cap, k, T = 5120, 512, 128
    rng = np.random.default_rng(B * 10 + Q)
    n_entries = [5000 - 7 * b for b in range(B)]
    idx = np.sort(rng.integers(0, 4990, (B, Q, k)), axis=-1).astype(np.int32)
    idx[:, :, -20:] = -1
    q_pos = [[n_entries[b] - 1 - qi for qi in range(Q)] for b in range(B)]
    pos0 = [n_entries[b] - T for b in range(B)]
    _attn_case(csa, 40 + B, B, Q, cap, n_entries, k, T, 128, q_pos, pos0, None, idx)


@pytest.mark.parametrize("B,Q,k,T,cap", [(8, 2, 512, 128, 1536), (32, 1, 500, 128, 1152), (1, 1, 2048, 128, 3072),
                                         (37, 1, 512, 100, 1152), (2, 1, 37, 128, 1024)],
                         ids=["c8", "c4_ragged", "c16_2048", "c4_short_window", "c16_small_k"])
def test_sparse_attn_decode_cluster_shapes(csa, B, Q, k, T, cap):
    # the decode cluster kernel at cluster sizes 8, 4 and 16: ragged key shares
    # (500 main slots), the most main rows a query takes (2048 over 16 CTAs),
    # fewer stored window rows than the window (dead window slots), and a few
    # main rows per CTA (37 over 16)
    rng = np.random.default_rng(B + k)
    n_entries = [cap - 50 - 3 * b for b in range(B)]
    idx = np.sort(rng.integers(0, cap - 60, (B, Q, k)), axis=-1).astype(np.int32)
    idx[:, :, ::37] = -1
    q_pos = [[n_entries[b] - 1 - 2 * qi for qi in range(Q)] for b in range(B)]
    pos0 = [n_entries[b] - T for b in range(B)]
    _attn_case(csa, 80 + B, B, Q, cap, n_entries, k, T, 128, q_pos, pos0, None, idx)


def test_sparse_attn_two_cta_clusters(csa):
    # 40 queries with 280 main rows each: two CTAs per query hold 148 slots each
    B, Q, k, T, cap = 40, 1, 280, 16, 640
    rng = np.random.default_rng(9)
    n_entries = [600 - b for b in range(B)]
    idx = np.sort(rng.integers(0, 560, (B, Q, k)), axis=-1).astype(np.int32)
    q_pos = [[n_entries[b] - 1] for b in range(B)]
    pos0 = [n_entries[b] - T for b in range(B)]
    _attn_case(csa, 90, B, Q, cap, n_entries, k, T, 16, q_pos, pos0, None, idx)


@pytest.mark.parametrize("window", [1, 2, 4, 77, 128])
@pytest.mark.parametrize("Q", [8, 128])   # 16 queries: one cluster each; 256: split-K kernel
def test_sparse_attn_replay_mask(csa, window, Q):
    B, cap, k, T = 2, 3072, 64, 128
    rng = np.random.default_rng(window + Q)
    s = [3000 - 128, 2500]
    q_pos = [[s[b] + qi for qi in range(Q)] for b in range(B)]
    pos0 = [s[0], s[1] - 3]
    idx = np.sort(rng.integers(0, 2900, (B, Q, k)), axis=-1).astype(np.int32)
    _attn_case(csa, 50 + window, B, Q, cap, [3000, 2900], k, T, window, q_pos, pos0, s, idx)


def test_sparse_attn_edge_cases(csa):
    B, Q, cap = 2, 3, 640
    # k = 0 (SWA only); T = 0 (main only); query with nothing visible -> zeros
    rng = np.random.default_rng(7)
    idx = np.full((B, Q, 0), -1, np.int32)
    _attn_case(csa, 60, B, Q, cap, [600, 600], 0, 16, 128, [[599, 598, 10], [599, 300, 599]], [584, 584], None, idx)
    idx = rng.integers(-5, 700, (B, Q, 100)).astype(np.int32)   # padding and out-of-range ids
    _attn_case(csa, 61, B, Q, cap, [600, 321], 100, 0, 128, [[599, 598, 10], [599, 300, 599]], [0, 0], None, idx)
    idx = np.full((B, Q, 8), -1, np.int32)
    _attn_case(csa, 62, B, Q, cap, [600, 600], 8, 4, 128, [[599, 5000, 599], [10, 300, 599]], [0, 0], None, idx)


# ---------------------------------------------------------------- layer dispatch
def test_layer_dispatch_decoder_pattern(csa):
    """The decoder pattern F R R R (X R R R) x 4 through csa2_layer_step equals the
    oracle's layer composition (bit-exact indices; attention within tolerance)."""
    B, Q, cap, T = 2, 1, 6016, 128
    n_before = [5000, 4321]
    grp = Group(70, B, cap, n_before)
    o = {kk: v.copy() for kk, v in grp.oracle_cache().items()}
    # the new token of this step: appended by the Full layer at position n_before[b]
    new_lat = torch.stack([synth.latent(synth.seed_of("new", 70, b), 1, n_before[b], "cuda")[0] for b in range(B)])
    new_rows = torch.tensor([b * cap + n_before[b] for b in range(B)], dtype=torch.int64, device="cuda")
    nb = bits(new_lat)
    olat, olsc = oracle.quant_nvfp4(nb)
    oik, oiks = oracle.index_k_proj(nb, np_(grp.W))
    n_after = np.array(n_before, np.int32) + 1
    for b in range(B):
        o["lat"][b, n_before[b]] = olat[b]
        o["lat_sc"][b, n_before[b]] = olsc[b]
        o["ik"][b, n_before[b]] = oik[b]
        o["iks"][b, n_before[b]] = oiks[b]
    grp.kv.n_entries.copy_(torch.from_numpy(n_after))
    q_pos_np = (n_after - 1).reshape(B, 1).astype(np.int32)
    qp = torch.from_numpy(q_pos_np).cuda()
    idx = torch.zeros((B, Q, 512), dtype=torch.int32, device="cuda")
    pool = torch.zeros((B, Q, 2048), dtype=torch.int32, device="cuda")
    bm = torch.zeros((B, Q, (cap + 7) // 8), dtype=torch.float32, device="cuda")
    st = dict(lat=o["lat"], lat_sc=o["lat_sc"], ik=o["ik"], iks=o["iks"], n_entries=n_after, m=1, k=512,
              build_pool=True, pool_blocks=2048)
    for li, mode in enumerate(oracle.DECODER_PATTERN):
        q = synth.attn_q(synth.seed_of("layer-q", li), B, Q, "cuda")
        pos0 = n_after - T
        swa, swa_sc = swa_for(synth.seed_of("layer-swa", li), B, T, pos0)
        p0 = torch.from_numpy(pos0.astype(np.int32)).cuda()
        iq = iqs = w = oiq = oiqs = ow = None
        if mode != "reuse":
            iq, iqs, w, oiq, oiqs, ow = index_query(synth.seed_of("layer-iq", li), B, Q)
        first = li == 0
        out = csa.csa2_layer_step(mode, grp.kv, qp, q, swa, swa_sc, p0, idx, 512, iq, iqs, w,
                                  pool=pool, blockmax=bm, new_latent=new_lat if first else None,
                                  new_rows=new_rows if first else None, k_proj=grp.W)
        layer = dict(q=bits(q), iq=oiq, iqs=oiqs, w=ow, swa=np_(swa), swa_sc=np_(swa_sc), swa_pos0=pos0.astype(np.int32),
                     window=128, q_pos=q_pos_np)
        ref, _ = oracle.layer_step(mode, st, layer)
        if first:
            assert np.array_equal(np_(grp.kv.lat), o["lat"]) and np.array_equal(kv_ik_rows(grp.kv)[0], o["ik"])
            assert np.array_equal(np_(pool), st["pool"])
        assert np.array_equal(np_(idx), st["idx"]), (li, mode)
        ok, stats = attn_close(out, ref)
        assert ok, (li, mode, stats)


# ---------------------------------------------------------------- fused front end
def _rope_tables(pos):
    k = np.arange(32, dtype=np.float64)
    ang = np.asarray(pos, np.float64).reshape(-1, 1) * 10000.0 ** (-2.0 * k / 64.0)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


@pytest.mark.parametrize("rows,weighted", [(1, False), (37, True), (64, False), (1000, True), (5000, False)])
def test_front_end_bit_exact(csa, rows, weighted):
    """RMSNorm + RoPE + bf16 + NVFP4 + indexer-K in one launch: every byte equals the oracle's
    front end followed by its quantiser and projection (rows past a multiple of 64: ragged CTA)."""
    x = (synth.normal(synth.seed_of("front", rows), (rows, 512), "cuda") * 1.7).to(torch.bfloat16)
    pos = np.arange(rows) * 131 + 7
    cos, sin = _rope_tables(pos)
    w = (0.25 + synth.uniform(synth.seed_of("front-w", rows), 512).to(torch.float32)).cuda() if weighted else None
    W = synth.proj_w(rows).cuda()
    out_rows = (2 * rows + 128) // 128 * 128
    dst = torch.arange(rows, device="cuda", dtype=torch.int64) * 2 + 1
    lc = torch.zeros((out_rows, 256), dtype=torch.uint8, device="cuda")
    ls = torch.zeros((out_rows, 32), dtype=torch.uint8, device="cuda")
    kc = torch.zeros((out_rows, 32), dtype=torch.uint8, device="cuda")
    ks = torch.zeros((out_rows, 4), dtype=torch.uint8, device="cuda")
    y = torch.zeros((rows, 512), dtype=torch.bfloat16, device="cuda")
    csa.csa2_front_end(x, torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda(), W, (lc, ls, kc, ks), dst,
                       norm_w=w, y_out=y)
    oy = oracle.front_end(bits(x), cos, sin, None if w is None else np_(w))
    assert np.array_equal(bits(y), oy)
    olc, ols = oracle.quant_nvfp4(oy)
    okc, oks = oracle.index_k_proj(oy, np_(W))
    assert np.array_equal(np_(lc)[1::2][:rows], olc) and np.array_equal(np_(ls)[1::2][:rows], ols)
    gkc, gks = ik_untile(np_(kc), np_(ks))
    assert np.array_equal(gkc[1::2][:rows], okc) and np.array_equal(gks[1::2][:rows], oks)
    assert not np_(lc)[0::2].any() and not gkc[0::2].any()


def test_front_end_hand_worked_cases(csa):
    import test_oracle_front as tf
    for case in tf.CASES:
        x = torch.from_numpy(tf._bits(case["x"]).view(np.int16)).view(torch.bfloat16).reshape(1, 512).cuda()
        cos = torch.from_numpy(case["cos"]).cuda()
        sin = torch.from_numpy(case["sin"]).cuda()
        w = None if case["w"] is None else torch.from_numpy(case["w"]).cuda()
        outs = tuple(torch.zeros((128, n), dtype=torch.uint8, device="cuda") for n in (256, 32, 32, 4))
        y = torch.zeros((1, 512), dtype=torch.bfloat16, device="cuda")
        csa.csa2_front_end(x, cos, sin, synth.proj_w(0).cuda(), outs, norm_w=w, y_out=y)
        assert np.array_equal(bits(y)[0], tf._bits(case["out"])), case["name"]
