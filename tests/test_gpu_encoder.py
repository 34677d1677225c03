"""The encoder side of CSA2 at full size, through the layer dispatcher (csa2_layer_step).

Encoder ([Blog] "CSA2：跨层复用，能借就不自己算"): 18 CSA2 layers at compression m = 2 in
three groups of 1 Full + 5 Reuse; each group's Full layer writes the group's own global
KV (FP4 main latent + FP4 indexer K) for the new entries and takes a fresh Top-512 with
m = 2 causal visibility, its Reuse layers borrow the indices; every layer has its own
query and its own FP8 sliding window.  The entries arrive already compressed (the
compressor's formula is not on the pages).

- The whole 65,536-token prompt as 16 chunks of 4,096 queries (2,048 new entries each).
- SWA Bounded Replay on a prefix-cache miss ([Blog] "FP4 与 SWA Bounded Replay：另外两刀",
  encoder side): the global KV of a 61,440-token prefix is cached, its sliding windows are
  not; the last 128 prefix tokens are replayed from s = 61,440 - 128 through the 18 layers
  against the cached global KV, then the 4,096-token suffix chunk runs.

Sampled queries are compared with the oracle's layer composition (oracle.layer_step):
indices bit for bit, attention within the tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import SM_SCALE, attn_close, bits, np_

pytestmark = pytest.mark.gpu

TOKENS, CHUNK, M, GROUPS = 65536, 4096, 2, 3
N_ENT = TOKENS // M                       # 32,768 entries per group
PATTERN = oracle.ENCODER_CSA2_PATTERN     # (full, reuse x 5) x 3


@pytest.fixture(scope="module")
def csa():
    import sparse_attention_fp4_quant_b200 as m
    m.lib()
    return m


class Encoder:
    """The three groups' caches (device, written by the Full layers) and the generator's
    bf16 entry latents (the oracle quantises and projects them itself)."""

    def __init__(self, csa, seed):
        self.csa, self.seed = csa, seed
        self.kv = [csa.KV(1, N_ENT, M, "cuda") for _ in range(GROUPS)]
        self.W = [synth.proj_w(synth.seed_of("enc-W", seed, g)).cuda() for g in range(GROUPS)]
        self.lat = [synth.latent(synth.seed_of("enc-ent", seed, g), N_ENT, 0, "cuda") for g in range(GROUPS)]
        self.idx = torch.zeros((1, CHUNK, 512), dtype=torch.int32, device="cuda")
        self._ok = {}

    def layer_inputs(self, tag, li, q_pos, pos0, T, with_iq):
        Q = q_pos.shape[1]
        q = synth.attn_q(synth.seed_of("enc-q", self.seed, tag, li), 1, Q, "cuda")
        c, sc = synth.swa_kv(synth.seed_of("enc-swa", self.seed, tag, li), T, pos0, "cuda")
        iq = iqs = None
        if with_iq:
            ib = synth.index_q(synth.seed_of("enc-iq", self.seed, tag, li), 1, Q, "cuda")
            iq, iqs = self.csa.csa2_quant_nvfp4(ib.reshape(-1, 64))
            iq, iqs = iq.view(1, Q, 128), iqs.view(1, Q, 16)
            ib = bits(ib.reshape(-1, 64))
            oiq, oiqs = oracle.quant_nvfp4(ib)
            iq_o = (oiq.reshape(1, Q, 128), oiqs.reshape(1, Q, 16))
        else:
            iq_o = None
        return q, c.unsqueeze(0), sc.unsqueeze(0), iq, iqs, iq_o

    def run_layers(self, tag, q_pos, pos0, T, append_rows, replay_start, keep):
        """The 18 layers for queries q_pos [1, Q]; `append_rows` = (e0, e1) entries each Full
        layer appends first.  Returns {li: (out, inputs)} for the layers in `keep`."""
        c = self.csa
        Q = q_pos.shape[1]
        qp = torch.from_numpy(q_pos).cuda()
        p0 = torch.tensor([pos0], dtype=torch.int32, device="cuda")
        rs = None if replay_start is None else torch.tensor([replay_start], dtype=torch.int32, device="cuda")
        idx = self.idx[:, :Q].contiguous() if Q != CHUNK else self.idx
        kept = {}
        for li, mode in enumerate(PATTERN):
            g = li // 6
            q, swa, swa_sc, iq, iqs, iq_o = self.layer_inputs(tag, li, q_pos, pos0, T, mode == "full")
            w = synth.index_w(1, Q, "cuda") if mode == "full" else None
            new = rows = None
            if mode == "full" and append_rows is not None:
                e0, e1 = append_rows
                new = self.lat[g][e0:e1].contiguous()
                rows = torch.arange(e0, e1, dtype=torch.int64, device="cuda")
                self.kv[g].n_entries.fill_(e1)
            out = c.csa2_layer_step(mode, self.kv[g], qp, q, swa, swa_sc, p0, idx, 512, iq, iqs, w,
                                    new_latent=new, new_rows=rows, k_proj=self.W[g], replay_start=rs)
            if li in keep:
                kept[li] = (out.clone(), q, swa, swa_sc, iq_o, idx.clone())
        return kept

    def oracle_group(self, g, n):
        """The oracle's own cache of group g's first n entries."""
        if (g, n) not in self._ok:
            lb = bits(self.lat[g][:n])
            lat, lsc = oracle.quant_nvfp4(lb)
            ik, iks = oracle.index_k_proj(lb, np_(self.W[g]))
            self._ok[(g, n)] = dict(lat=lat.reshape(1, n, 256), lat_sc=lsc.reshape(1, n, 32),
                                    ik=ik.reshape(1, n, 32), iks=iks.reshape(1, n, 4))
        return self._ok[(g, n)]


def _check_layers(enc, kept, q_pos, sel, n_vis_entries, pos0, replay_start):
    """Oracle layer composition for the queries `sel` of one chunk, group by group."""
    st = None
    for li, mode in enumerate(PATTERN):
        g = li // 6
        if mode == "full":
            oc = enc.oracle_group(g, n_vis_entries)
            st = dict(lat=oc["lat"], lat_sc=oc["lat_sc"], ik=oc["ik"], iks=oc["iks"],
                      n_entries=np.array([n_vis_entries], np.int32), m=M, k=512)
        if li not in kept:
            continue
        out, q, swa, swa_sc, iq_o, idx = kept[li]
        layer = dict(q=bits(q)[:, sel], swa=np_(swa), swa_sc=np_(swa_sc), swa_pos0=np.array([pos0], np.int32),
                     window=128, q_pos=q_pos[:, sel], sm_scale=SM_SCALE)
        if replay_start is not None:
            layer["replay_start"] = np.array([replay_start], np.int32)
        if mode == "full":
            layer.update(iq=iq_o[0][:, sel], iqs=iq_o[1][:, sel], w=np.full((1, len(sel), 4), 0.25, np.float32))
        ref, _ = oracle.layer_step(mode, st, layer)
        assert np.array_equal(np_(idx)[:, sel], st["idx"]), (li, mode)
        ok, stats = attn_close(out[:, sel], ref)
        assert ok, (li, mode, stats)


def test_encoder_prefill_whole_prompt_m2(csa):
    """f1: 16 chunks of 4,096 queries through 3 x (1 Full + 5 Reuse); queries of the first,
    a middle and the last chunk checked in every group (Full and two Reuse layers each)."""
    enc = Encoder(csa, 7)
    keep = {0, 1, 5, 6, 9, 12, 17}
    checks = {0: [0, 1, 2047, 4095], 7: [0, 3000], 15: [5, 4095]}
    for c in range(TOKENS // CHUNK):
        p_start = c * CHUNK
        q_pos = (p_start + np.arange(CHUNK, dtype=np.int32)).reshape(1, -1)
        pos0 = max(0, p_start - 127)
        T = p_start + CHUNK - pos0
        e0, e1 = p_start // M, (p_start + CHUNK) // M
        kept = enc.run_layers(f"chunk{c}", q_pos, pos0, T, (e0, e1), None, keep if c in checks else set())
        if c in checks:
            torch.cuda.synchronize()
            # causality: a query at token p sees entry e iff 2e + 1 <= p
            for li, (_, _, _, _, _, idx) in kept.items():
                gi = np_(idx)[0]
                assert np.all((gi < 0) | (2 * gi + 1 <= q_pos[0][:, None])), li
            _check_layers(enc, kept, q_pos, checks[c], e1, pos0, None)


def test_encoder_replay_on_prefix_cache_miss(csa):
    """f2: the global KV of a 61,440-token prefix is cached (written by earlier chunks); its
    sliding windows are gone.  Replay the last 128 prefix tokens from s = prefix - 128
    through the 18 layers (mask [max(s, i - 127), i], no append), then the suffix chunk."""
    enc = Encoder(csa, 8)
    prefix = TOKENS - CHUNK
    n_pre = prefix // M
    for g in range(GROUPS):   # the cached prefix: written once by the library's own append
        csa.csa2_append_tokens(enc.lat[g][:n_pre].contiguous(), enc.W[g], enc.kv[g],
                               torch.arange(0, n_pre, dtype=torch.int64, device="cuda"))
        enc.kv[g].n_entries.fill_(n_pre)
    s = prefix - 128
    rq = (s + np.arange(128, dtype=np.int32)).reshape(1, -1)
    keep = {0, 3, 6, 11, 12, 16}
    kept = enc.run_layers("replay", rq, s, 128, None, s, keep)
    torch.cuda.synchronize()
    _check_layers(enc, kept, rq, [0, 1, 64, 127], n_pre, s, s)
    # the suffix chunk: queries prefix .. 65,535, window back to prefix - 127
    q_pos = (prefix + np.arange(CHUNK, dtype=np.int32)).reshape(1, -1)
    pos0 = prefix - 127
    kept = enc.run_layers("suffix", q_pos, pos0, TOKENS - pos0, (n_pre, N_ENT), None, keep)
    torch.cuda.synchronize()
    _check_layers(enc, kept, q_pos, [0, 1, 2048, 4095], N_ENT, pos0, None)
