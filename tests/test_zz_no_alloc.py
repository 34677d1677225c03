"""csa2_index_topk_noalloc: the index + Top-K call for callers that cannot
allocate device memory (their device memory belongs to their own pool, or a
cudaMalloc is not allowed on their path).  It must give the same indices and
block maxima as csa2_index_topk with a caller workspace, call after call, while
using only the library's static scratch array.  Collected last on purpose."""
import numpy as np
import pytest
import torch

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


def test_noalloc_matches_workspace_call_twice():
    csa, kv, iq, iqs, w, q_pos = _case(5, 4, 2, 40064)
    assert "csa2_index_topk_noalloc" in csa.EXPORTS
    for k in (512, 2048):
        ref, ref_bm = csa.csa2_index_topk(iq, iqs, w, kv, q_pos, k, blockmax=True)
        assert csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, 4, 2, kv.cap, k) > 4 * 2 * 4  # several shares per query
        for _ in range(2):
            got, bm = csa.csa2_index_topk_noalloc(iq, iqs, w, kv, q_pos, k, blockmax=True)
            torch.cuda.synchronize()
            assert torch.equal(got, ref)
            assert torch.equal(bm, ref_bm)


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
