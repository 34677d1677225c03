"""csa2_index_topk_noalloc: the index + Top-K call for callers that cannot
allocate device memory (their device memory belongs to their own pool, or a
cudaMalloc, which can synchronise the device, is not allowed on their path).
It must give the oracle's indices and block maxima, and the same results as
csa2_index_topk with a caller workspace, call after call and whatever the
previous call left in the library's static scratch array.  Collected last on
purpose, so that a run stopping at the first failure has run everything else."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import np_, set_kv_ik_rows

pytestmark = pytest.mark.gpu


def _case(seed, B, Q, cap):
    import sparse_attention_fp4_quant_b200 as csa
    import synth
    kv = csa.KV(B, cap, 1, "cuda")
    W = synth.proj_w(seed).cuda()
    for b in range(B):
        lat = synth.latent(synth.seed_of("noalloc", seed, b), cap, 0, "cuda")
        csa.csa2_quant_nvfp4(lat, kv.lat[b].view(-1, 256), kv.lat_sc[b].view(-1, 32))
        csa.csa2_index_k_proj(lat, W, kv.ik[b].view(-1, 32), kv.ik_sc[b].view(-1, 4))
    kv.n_entries.copy_(torch.tensor([cap - 13 * b for b in range(B)], dtype=torch.int32))
    iq, iqs = csa.csa2_quant_nvfp4(synth.index_q(seed, B, Q, "cuda").view(-1, 64))
    w = synth.index_w(B, Q, "cuda")
    q_pos = torch.tensor([[cap - 1 - 1000 * q for q in range(Q)] for _ in range(B)], dtype=torch.int32,
                         device="cuda")
    return csa, kv, iq.view(B, Q, 128), iqs.view(B, Q, 16), w, q_pos


def _random_fp4_case(seed, B, Q, cap, m=1):
    """Seeded random FP4 indexer keys and queries, written to the device cache and kept
    row-major for the oracle (the oracle receives the generator's bytes, not the GPU's)."""
    import sparse_attention_fp4_quant_b200 as csa
    rng = np.random.default_rng(seed)
    ik = rng.integers(0, 256, (B, cap, 32), dtype=np.uint8)
    iks = rng.integers(0x20, 0x50, (B, cap, 4), dtype=np.uint8)
    q = rng.integers(0, 256, (B, Q, 128), dtype=np.uint8)
    qs = rng.integers(0x20, 0x50, (B, Q, 16), dtype=np.uint8)
    w = np.full((B, Q, 4), 0.25, np.float32)
    n_entries = np.array([cap - 7 * b for b in range(B)], np.int32)
    step = m * (cap - 7 * (B - 1)) // (Q + 1)   # queries spread over the visible range
    q_pos = np.array([[m * int(n_entries[b]) - 1 - step * qi for qi in range(Q)] for b in range(B)], np.int32)
    kv = csa.KV(B, cap, m, "cuda")
    set_kv_ik_rows(kv, ik, iks)
    kv.n_entries.copy_(torch.from_numpy(n_entries))
    dev = dict(q=torch.from_numpy(q).cuda(), qs=torch.from_numpy(qs).cuda(), w=torch.from_numpy(w).cuda(),
               q_pos=torch.from_numpy(q_pos).cuda())
    host = dict(q=q, qs=qs, w=w, ik=ik, iks=iks, n_entries=n_entries, q_pos=q_pos, m=m)
    return csa, kv, dev, host


def test_noalloc_matches_workspace_call_twice():
    # 8 queries: the cluster kernel, which needs only the scratch's error flag
    csa, kv, iq, iqs, w, q_pos = _case(5, 4, 2, 40064)
    assert "csa2_index_topk_noalloc" in csa.EXPORTS
    for k in (512, 2048):
        ref, ref_bm = csa.csa2_index_topk(iq, iqs, w, kv, q_pos, k, blockmax=True)
        for _ in range(2):
            got, bm = csa.csa2_index_topk_noalloc(iq, iqs, w, kv, q_pos, k, blockmax=True)
            torch.cuda.synchronize()
            assert torch.equal(got, ref)
            assert torch.equal(bm, ref_bm)
    csa.csa2_index_topk_noalloc_status()


def test_noalloc_per_share_path_matches_oracle_across_alternating_calls():
    # one query over 524,416 entries is too long for one cluster: the per-share kernel
    # runs it as 257 shares whose candidate lists and merge counters live in the static
    # array.  Alternating it with a cluster-path call of another shape shows that what
    # one call leaves in the array does not leak into the next.
    k = 512
    csa, kv_a, da, ha = _random_fp4_case(71, 1, 1, 524416)
    assert csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, 1, 1, kv_a.cap, k) > 1 << 20   # many shares
    want_a, want_a_bm = oracle.index_topk(ha["q"], ha["qs"], ha["w"], ha["ik"], ha["iks"], ha["n_entries"], 1,
                                          ha["q_pos"], k, blockmax=True)
    csa, kv_b, iq, iqs, w, q_pos = _case(72, 4, 2, 40064)
    ref_b = csa.csa2_index_topk(iq, iqs, w, kv_b, q_pos, k)
    ref_a = csa.csa2_index_topk(da["q"], da["qs"], da["w"], kv_a, da["q_pos"], k)
    assert np.array_equal(np_(ref_a), want_a)
    for _ in range(2):
        got_a, bm_a = csa.csa2_index_topk_noalloc(da["q"], da["qs"], da["w"], kv_a, da["q_pos"], k, blockmax=True)
        assert np.array_equal(np_(got_a), want_a)
        assert np.array_equal(np_(bm_a).view(np.uint32), want_a_bm.view(np.uint32))
        csa.csa2_index_topk_noalloc_status()
        got_b = csa.csa2_index_topk_noalloc(iq, iqs, w, kv_b, q_pos, k)
        assert torch.equal(got_b, ref_b)
        csa.csa2_index_topk_noalloc_status()


def test_noalloc_prefill_sized_request_matches_workspace_call():
    # 150 queries of one batch row at m = 2: the workspace call takes the many-query
    # kernels, the no-allocation call the per-share ones; the results are the same
    csa, kv, dev, host = _random_fp4_case(73, 1, 150, 3072, m=2)
    ref = csa.csa2_index_topk(dev["q"], dev["qs"], dev["w"], kv, dev["q_pos"], 512)
    want = oracle.index_topk(host["q"], host["qs"], host["w"], host["ik"], host["iks"], host["n_entries"], 2,
                             host["q_pos"], 512)
    assert np.array_equal(np_(ref), want)
    for _ in range(2):
        got = csa.csa2_index_topk_noalloc(dev["q"], dev["qs"], dev["w"], kv, dev["q_pos"], 512)
        assert np.array_equal(np_(got), want)
    csa.csa2_index_topk_noalloc_status(clear=True)


def test_noalloc_rejects_requests_beyond_its_scratch():
    csa, kv, iq, iqs, w, q_pos = _case(6, 1, 1, 1 << 20)
    need = csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, 1, 1, kv.cap, 2048)
    assert need > csa.NOALLOC_SCRATCH_BYTES
    with pytest.raises(csa.CSA2Error, match="WORKSPACE"):
        csa.csa2_index_topk_noalloc(iq, iqs, w, kv, q_pos, 2048)
    # the same query within the limit still works and agrees with the workspace call
    got = csa.csa2_index_topk_noalloc(iq, iqs, w, kv, q_pos, 512)
    ref = csa.csa2_index_topk(iq, iqs, w, kv, q_pos, 512)
    assert np.array_equal(got.cpu().numpy(), ref.cpu().numpy())
    csa.csa2_index_topk_noalloc_status()
