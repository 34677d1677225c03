"""GPU parity at the full sizes of the five synthetic workloads, on sampled outputs.

The CUDA path runs each call at full size in the launch configuration the
benchmark uses.  The oracle recomputes sampled outputs from the same generator
bytes (it quantises and projects the rows it needs itself); where a full
recomputation would be too slow, properties that hold at any size are checked
instead (selected entries score at least as well as any sampled unselected one,
under the tie rule).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import SM_SCALE, attn_close, bits, index_query, np_, swa_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    import sparse_attention_fp4_quant_b200 as m
    m.lib()
    return m


class BigGroup:
    """A [B][cap] cache built on the GPU by the CUDA path; bf16 latents kept for `keep` rows."""

    def __init__(self, csa, seed, B, cap, n_entries, m=1, keep=()):
        self.B, self.cap, self.m, self.seed = B, cap, m, seed
        self.kv = csa.KV(B, cap, m, "cuda")
        self.W = synth.proj_w(seed).cuda()
        self.latent = {}
        for b in range(B):
            lat = synth.latent(synth.seed_of("big", seed, b), cap, 0, "cuda")
            csa.csa2_quant_nvfp4(lat, self.kv.lat[b].view(-1, 256), self.kv.lat_sc[b].view(-1, 32))
            csa.csa2_index_k_proj(lat, self.W, self.kv.ik[b].view(-1, 32), self.kv.ik_sc[b].view(-1, 4))
            if b in keep:
                self.latent[b] = lat
            else:
                # keep a few rows of every batch row for quantiser spot checks
                self.latent.setdefault("spot", {})[b] = (lat[::4099].clone(), torch.arange(0, cap, 4099))
            del lat
        self.n_entries = np.array(n_entries, np.int32)
        self.kv.n_entries.copy_(torch.from_numpy(self.n_entries))
        self._ocache = {}

    def oracle_k(self, b):
        """The oracle's own indexer K of batch row b (all cap rows)."""
        if b not in self._ocache:
            ik, iks = oracle.index_k_proj(bits(self.latent[b]), np_(self.W))
            self._ocache[b] = (ik.reshape(1, self.cap, 32), iks.reshape(1, self.cap, 4))
        return self._ocache[b]

    def oracle_rows(self, b, rows):
        """The oracle's own quantised latent rows of batch row b at the given positions."""
        lb = bits(self.latent[b][torch.as_tensor(rows, dtype=torch.long, device="cuda")])
        return oracle.quant_nvfp4(lb)


def _check_spots(grp):
    for b, lat in grp.latent.items():
        if b == "spot":
            continue
        pos = torch.arange(0, grp.cap, 4099)
        c, s = oracle.quant_nvfp4(bits(lat[pos.cuda()]))
        assert np.array_equal(np_(grp.kv.lat[b, pos.cuda()]), c.reshape(-1, 256))
        assert np.array_equal(np_(grp.kv.lat_sc[b, pos.cuda()]), s.reshape(-1, 32))
    for b, (rows, pos) in grp.latent.get("spot", {}).items():
        c, s = oracle.quant_nvfp4(bits(rows))
        assert np.array_equal(np_(grp.kv.lat[b, pos.cuda()]), c.reshape(-1, 256))
        assert np.array_equal(np_(grp.kv.lat_sc[b, pos.cuda()]), s.reshape(-1, 32))


def _index_ref(grp, b, oiq, oiqs, ow, q_pos_row, k, blockmax=False):
    ik, iks = grp.oracle_k(b)
    return oracle.index_topk(oiq[b:b + 1], oiqs[b:b + 1], ow[b:b + 1], ik, iks, grp.n_entries[b:b + 1], grp.m,
                             np.asarray(q_pos_row, np.int32).reshape(1, -1), k, blockmax=blockmax)


def _attn_ref(grp, b, q_bits, idx_row, swa, swa_sc, pos0, q_pos, window=128, replay=None):
    """Oracle attention for batch row b's queries on a compact cache of the selected rows."""
    sel = np.unique(idx_row[idx_row >= 0])
    lat, lsc = grp.oracle_rows(b, sel)
    remap = {int(e): i for i, e in enumerate(sel)}
    idx_c = np.vectorize(lambda e: remap.get(int(e), -1))(idx_row).astype(np.int32)
    return oracle.sparse_attn(q_bits, lat.reshape(1, -1, 256), lsc.reshape(1, -1, 32),
                              np.array([len(sel)], np.int32), idx_c, swa, swa_sc, np.array([pos0], np.int32),
                              window, None if replay is None else np.array([replay], np.int32),
                              np.asarray(q_pos, np.int32).reshape(1, -1), SM_SCALE)


def _score_property(grp, b, sel, oiq_b, oiqs_b, ow_b, nvis, rng, n_sample=2000):
    """Selected entries beat every sampled unselected visible entry (score desc, position asc)."""
    sel = np.asarray([e for e in sel if e >= 0])
    cand = np.setdiff1d(rng.integers(0, nvis, n_sample), sel)
    rows = np.concatenate([sel, cand])
    lb = bits(grp.latent[b][torch.as_tensor(rows, dtype=torch.long, device="cuda")])
    ik, iks = oracle.index_k_proj(lb, np_(grp.W))
    sc = [oracle.index_score(oiq_b, oiqs_b, ow_b, ik[i], iks[i]) for i in range(len(rows))]
    worst = min(zip(sc[:len(sel)], -sel), key=lambda t: (t[0], t[1]))   # lowest (score, -pos)
    for s_, e in zip(sc[len(sel):], cand):
        assert (s_, -e) < worst, (s_, e, worst)


def test_c0_full_layer_small(csa):
    B, n = 1, 4096
    grp = BigGroup(csa, 100, B, n, [n], keep=(0,))
    iq, iqs, w, oiq, oiqs, ow = index_query(101, B, 1)
    qp = np.full((B, 1), n - 1, np.int32)
    idx = csa.csa2_index_topk(iq, iqs, w, grp.kv, torch.from_numpy(qp).cuda(), 512)
    ridx = _index_ref(grp, 0, oiq, oiqs, ow, qp[0], 512)
    assert np.array_equal(np_(idx), ridx)
    q = synth.attn_q(102, B, 1, "cuda")
    swa, swa_sc = swa_for(103, B, 128, [n - 128])
    out = csa.csa2_sparse_attn(q, grp.kv, idx, swa, swa_sc, torch.tensor([n - 128], dtype=torch.int32, device="cuda"),
                               torch.from_numpy(qp).cuda())
    ref, _ = _attn_ref(grp, 0, bits(q), ridx[0], np_(swa), np_(swa_sc), n - 128, qp[0])
    ok, st = attn_close(out, ref)
    assert ok, st


def test_c1_decode_group_b32_131k(csa):
    """B=32, 131,072 entries, 1 Full + 3 Reuse, in the benchmark's launch configuration."""
    B, n = 32, 131072
    grp = BigGroup(csa, 110, B, n, [n] * B, keep=(0, 31))
    _check_spots(grp)
    iq, iqs, w, oiq, oiqs, ow = index_query(111, B, 1)
    qp_np = np.full((B, 1), n - 1, np.int32)
    qp = torch.from_numpy(qp_np).cuda()
    ws = torch.zeros(max(csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, B, 1, n, 512),
                         csa.csa2_workspace_bytes(csa.OP_SPARSE_ATTN, B, 1, n, 512)), dtype=torch.uint8, device="cuda")
    idx = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, 512, ws=ws)
    gi = np_(idx)
    for b in (0, 31):
        assert np.array_equal(gi[b], _index_ref(grp, b, oiq, oiqs, ow, qp_np[b], 512)[0]), b
    assert np.all(np.diff(gi, axis=-1) > 0) and gi.min() >= 0 and gi.max() < n
    pos0 = np.full(B, n - 128, np.int32)
    for layer in range(4):
        q = synth.attn_q(synth.seed_of("c1q", layer), B, 1, "cuda")
        swa, swa_sc = swa_for(synth.seed_of("c1swa", layer), B, 128, pos0)
        out = csa.csa2_sparse_attn(q, grp.kv, idx, swa, swa_sc, torch.from_numpy(pos0).cuda(), qp, ws=ws)
        for b in (0, 31):
            ref, _ = _attn_ref(grp, b, bits(q[b:b + 1]), gi[b:b + 1], np_(swa)[b:b + 1], np_(swa_sc)[b:b + 1], n - 128,
                               qp_np[b])
            ok, st = attn_close(out[b:b + 1], ref)
            assert ok, (layer, b, st)


def test_index_keys_in_workspace_b2_640k(csa):
    """B=2 at 655,360 entries: more than 16 CTAs hold in TMEM, so the cluster index keeps its
    keys in the workspace (csa2_workspace_bytes counts them); both rows equal the oracle's
    Top-512, and the same call with only the minimum workspace (the per-share select) agrees."""
    B, n = 2, 655360
    nv = [n, n - 4321]
    grp = BigGroup(csa, 125, B, n, nv, keep=(0, 1))
    iq, iqs, w, oiq, oiqs, ow = index_query(126, B, 1)
    qp_np = np.array([[nv[0] - 1], [nv[1] - 1]], np.int32)
    qp = torch.from_numpy(qp_np).cuda()
    full = csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, B, 1, n, 512)
    assert full >= B * n * 4   # the keys' room
    idx = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, 512,
                              ws=torch.zeros(full, dtype=torch.uint8, device="cuda"))
    for b in range(B):
        ridx = _index_ref(grp, b, oiq, oiqs, ow, qp_np[b], 512)
        assert np.array_equal(np_(idx)[b], ridx[0]), b
    small = full - B * n * 4   # the minimum the call accepts
    idx2 = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, 512,
                               ws=torch.zeros(max(small, 1), dtype=torch.uint8, device="cuda"))
    assert np.array_equal(np_(idx2), np_(idx))


def test_c2_hierarchical_b8_1m(csa):
    """B=8, 1,048,576 entries: Full (Top-512 + block maxima) -> pool of 2,048 blocks -> Reindex Top-512."""
    B, n = 8, 1 << 20
    grp = BigGroup(csa, 120, B, n, [n] * B, keep=(0, 5))
    iq, iqs, w, oiq, oiqs, ow = index_query(121, B, 1)
    qp_np = np.full((B, 1), n - 1, np.int32)
    qp = torch.from_numpy(qp_np).cuda()
    _check_spots(grp)
    idx, bm = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, 512, blockmax=True)
    ridx, rbm = _index_ref(grp, 0, oiq, oiqs, ow, qp_np[0], 512, blockmax=True)
    assert np.array_equal(np_(idx)[0], ridx[0])
    assert np.array_equal(np_(bm)[0], rbm[0])
    pool = csa.csa2_pool_build(bm, grp.kv, qp, 2048)
    rpool = oracle.pool_build(rbm, grp.n_entries[:1], 1, qp_np[:1], 2048)
    assert np.array_equal(np_(pool)[0], rpool[0])
    riq, riqs, rw, roiq, roiqs, row_ = index_query(122, B, 1)
    ridx2 = csa.csa2_pool_topk(riq, riqs, rw, grp.kv, pool, qp, 512)
    ik, iks = grp.oracle_k(0)
    ref2 = oracle.pool_topk(roiq[:1], roiqs[:1], row_[:1], ik, iks, grp.n_entries[:1], 1, rpool, qp_np[:1], 512)
    assert np.array_equal(np_(ridx2)[0], ref2[0])
    # other batch rows: property check of the Full-layer selection
    rng = np.random.default_rng(0)
    gi = np_(idx)
    _score_property(grp, 5, gi[5, 0], oiq[5, 0], oiqs[5, 0], ow[5, 0], n, rng)
    q = synth.attn_q(123, B, 1, "cuda")
    swa, swa_sc = swa_for(124, B, 128, [n - 128] * B)
    out = csa.csa2_sparse_attn(q, grp.kv, ridx2, swa, swa_sc, torch.full((B,), n - 128, dtype=torch.int32, device="cuda"),
                               qp)
    ref, _ = _attn_ref(grp, 0, bits(q[:1]), ref2[:1], np_(swa)[:1], np_(swa_sc)[:1], n - 128, qp_np[0])
    ok, st = attn_close(out[:1], ref)
    assert ok, st


def test_c3_prefill_chunk_m2(csa):
    """m=2: 65,536 tokens -> 32,768 entries; 4,096 queries at the end of the prompt."""
    B, n, Q, tokens = 1, 32768, 4096, 65536
    grp = BigGroup(csa, 130, B, n, [n], m=2, keep=(0,))
    iq, iqs, w, oiq, oiqs, ow = index_query(131, B, Q)
    qp_np = (tokens - Q + np.arange(Q, dtype=np.int32)).reshape(1, Q)
    qp = torch.from_numpy(qp_np).cuda()
    idx = csa.csa2_index_topk(iq, iqs, w, grp.kv, qp, 512)
    gi = np_(idx)
    sample = [0, 1, 777, 2048, 4095]
    ik, iks = grp.oracle_k(0)
    ridx = oracle.index_topk(oiq[:, sample], oiqs[:, sample], ow[:, sample], ik, iks, grp.n_entries, 2,
                             qp_np[:, sample], 512)
    assert np.array_equal(gi[:, sample], ridx)
    # causality for every query: m=2 entry e visible iff 2e+1 <= p
    assert np.all(gi[0] * 2 + 1 <= qp_np[0][:, None]) and np.all(gi >= 0)
    T = Q + 127
    pos0 = tokens - Q - 127
    q = synth.attn_q(132, B, Q, "cuda")
    swa, swa_sc = swa_for(133, B, T, [pos0])
    out = csa.csa2_sparse_attn(q, grp.kv, idx, swa, swa_sc, torch.tensor([pos0], dtype=torch.int32, device="cuda"), qp)
    for qi in (0, 2048, 4095):
        ref, _ = _attn_ref(grp, 0, bits(q[:, qi:qi + 1]), ridx[:, sample.index(qi):sample.index(qi) + 1],
                           np_(swa), np_(swa_sc), pos0, qp_np[:, qi])
        ok, st = attn_close(out[:, qi:qi + 1], ref)
        assert ok, (qi, st)


def test_c4_replay_and_decoder_step(csa):
    """B=4, 262,144 entries: SWA Bounded Replay of the last 128 tokens (s = ctx - 128) through
    the 20-layer decoder pattern (fresh FP8 SWA KV per layer; Reuse layers borrow the indices,
    Reindex layers search the Full layer's pool), then one decode step through the same 20
    layers with the append.  Sampled queries of batch row 2 are checked at every indexing
    layer (indices, pool) and at several attention layers."""
    B, n = 4, 262144
    grp = BigGroup(csa, 140, B, n + 128, [n] * B, keep=(2,))
    s = n - 128
    Q = 128
    sample = [0, 64, 127]
    qp_np = np.tile(s + np.arange(Q, dtype=np.int32), (B, 1))
    qp = torch.from_numpy(qp_np).cuda()
    rs = torch.full((B,), s, dtype=torch.int32, device="cuda")
    ridx_q = torch.zeros((B, Q, 512), dtype=torch.int32, device="cuda")
    rpool = torch.zeros((B, Q, 2048), dtype=torch.int32, device="cuda")
    rbm = torch.zeros((B, Q, (grp.cap + 7) // 8), dtype=torch.float32, device="cuda")
    rik, riks = grp.oracle_k(2)
    pool_ref = cur = None
    for li, mode in enumerate(oracle.DECODER_PATTERN):
        lq = synth.attn_q(synth.seed_of("c4rq", li), B, Q, "cuda")
        lswa, lswa_sc = swa_for(synth.seed_of("c4rswa", li), B, 128, [s] * B)
        liq = liqs = lw = loiq = loiqs = low = None
        if mode != "reuse":
            liq, liqs, lw, loiq, loiqs, low = index_query(synth.seed_of("c4riq", li), B, Q)
        out = csa.csa2_layer_step(mode, grp.kv, qp, lq, lswa, lswa_sc, rs, ridx_q, 512, liq, liqs, lw, pool=rpool,
                                  blockmax=rbm, k_proj=grp.W, replay_start=rs)
        if mode == "full":
            cur, bm_ref = oracle.index_topk(loiq[2:3, sample], loiqs[2:3, sample], low[2:3, sample], rik, riks,
                                            grp.n_entries[2:3], 1, qp_np[2:3, sample], 512, blockmax=True)
            pool_ref = oracle.pool_build(bm_ref, grp.n_entries[2:3], 1, qp_np[2:3, sample], 2048)
            assert np.array_equal(np_(rpool)[2:3, sample], pool_ref)
        elif mode == "reindex":
            cur = oracle.pool_topk(loiq[2:3, sample], loiqs[2:3, sample], low[2:3, sample], rik, riks,
                                   grp.n_entries[2:3], 1, pool_ref, qp_np[2:3, sample], 512)
        assert np.array_equal(np_(ridx_q)[2:3, sample], cur), (li, mode)
        if li in (0, 1, 4, 7, 12, 19):
            for j, qi in enumerate(sample):
                ref, _ = _attn_ref(grp, 2, bits(lq[2:3, qi:qi + 1]), cur[:, j:j + 1], np_(lswa)[2:3],
                                   np_(lswa_sc)[2:3], s, qp_np[2, qi], replay=s)
                ok, st = attn_close(out[2:3, qi:qi + 1], ref)
                assert ok, (li, mode, qi, st)
    # ---- decode step: the new token (position n) is appended by the Full layer
    new_lat = torch.stack([synth.latent(synth.seed_of("c4new", b), 1, n, "cuda")[0] for b in range(B)])
    new_rows = torch.tensor([b * grp.cap + n for b in range(B)], dtype=torch.int64, device="cuda")
    grp.latent[2] = torch.cat([grp.latent[2][:n], new_lat[2:3], grp.latent[2][n + 1:]])
    grp._ocache.clear()
    grp.n_entries[:] = n + 1
    grp.kv.n_entries.fill_(n + 1)
    dqp_np = np.full((B, 1), n, np.int32)
    dqp = torch.from_numpy(dqp_np).cuda()
    idx1 = torch.zeros((B, 1, 512), dtype=torch.int32, device="cuda")
    pool = torch.zeros((B, 1, 2048), dtype=torch.int32, device="cuda")
    bm = torch.zeros((B, 1, (grp.cap + 7) // 8), dtype=torch.float32, device="cuda")
    pos0 = np.full(B, n - 127, np.int32)
    pool_ref = None
    for li, mode in enumerate(oracle.DECODER_PATTERN):
        lq = synth.attn_q(synth.seed_of("c4q", li), B, 1, "cuda")
        lswa, lswa_sc = swa_for(synth.seed_of("c4swa", li), B, 128, pos0)
        liq = liqs = lw = loiq = loiqs = low = None
        if mode != "reuse":
            liq, liqs, lw, loiq, loiqs, low = index_query(synth.seed_of("c4iq", li), B, 1)
        out = csa.csa2_layer_step(mode, grp.kv, dqp, lq, lswa, lswa_sc, torch.from_numpy(pos0).cuda(), idx1, 512,
                                  liq, liqs, lw, pool=pool, blockmax=bm, new_latent=new_lat if li == 0 else None,
                                  new_rows=new_rows if li == 0 else None, k_proj=grp.W)
        g1 = np_(idx1)
        if mode == "full":
            rik, riks = grp.oracle_k(2)
            r1, rbm = oracle.index_topk(loiq[2:3], loiqs[2:3], low[2:3], rik, riks, grp.n_entries[2:3], 1,
                                        dqp_np[2:3], 512, blockmax=True)
            pool_ref = oracle.pool_build(rbm, grp.n_entries[2:3], 1, dqp_np[2:3], 2048)
            assert np.array_equal(np_(pool)[2], pool_ref[0])
            cur = r1
        elif mode == "reindex":
            rik, riks = grp.oracle_k(2)
            cur = oracle.pool_topk(loiq[2:3], loiqs[2:3], low[2:3], rik, riks, grp.n_entries[2:3], 1, pool_ref,
                                   dqp_np[2:3], 512)
        assert np.array_equal(g1[2], cur[0]), (li, mode)
        if li in (0, 1, 4, 19):
            ref, _ = _attn_ref(grp, 2, bits(lq[2:3]), cur, np_(lswa)[2:3], np_(lswa_sc)[2:3], int(pos0[2]), dqp_np[2])
            ok, st = attn_close(out[2:3], ref)
            assert ok, (li, mode, st)
