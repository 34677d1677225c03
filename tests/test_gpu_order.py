"""The hand-worked order cases (tests/golden/index_order_cases.txt) on every
scoring kernel: the decode cluster kernel, the many-query kernels, the
per-share kernel, the Reindex pool search and the no-allocation call; and the
indexer-K chain case on the projection and append kernels.

The expected values are the file's hand-worked ones, not the oracle's, so a
misreading of the order shared by the oracle and the kernels fails here too.
"""
import numpy as np
import pytest
import torch

from gpu_common import ik_untile, np_, set_kv_ik_rows
from order_cases import bf16_bits_of, keys_array, load

pytestmark = pytest.mark.gpu

SCORE_CASES, KPROJ_CASES = load()
STRIDE = 8   # entry i of a case sits at position 8 i: one entry per block of 8


@pytest.fixture(scope="module")
def csa():
    import sparse_attention_fp4_quant_b200 as m
    m.lib()
    return m


def _setup(csa, B, Q, cap=128):
    """Batch row b holds case b % 3 (its keys at stride 8; every query of the row is the case's)."""
    n = len(SCORE_CASES[0]["entries"]) * STRIDE
    kv = csa.KV(B, cap, 1, "cuda")
    codes = np.zeros((B, cap, 32), np.uint8)
    scales = np.full((B, cap, 4), 0x38, np.uint8)
    q = np.zeros((B, Q, 128), np.uint8)
    qs = np.zeros((B, Q, 16), np.uint8)
    w = np.zeros((B, Q, 4), np.float32)
    want_top1 = np.zeros((B, Q), np.int32)
    for b in range(B):
        case = SCORE_CASES[b % len(SCORE_CASES)]
        k, ks = keys_array(case, n, STRIDE)
        codes[b, :n], scales[b, :n] = k, ks
        q[b, :], qs[b, :], w[b, :] = case["q"], case["qs"], case["w"]
        want_top1[b, :] = case["top1"] * STRIDE
    set_kv_ik_rows(kv, codes, scales)
    kv.n_entries.fill_(n)
    q_pos = torch.full((B, Q), n - 1, dtype=torch.int32, device="cuda")
    t = lambda a: torch.from_numpy(a).cuda()
    return kv, t(q), t(qs), t(w), q_pos, want_top1


def _check_blockmax(bm, B, Q):
    bm = np_(bm)
    for b in range(B):
        case = SCORE_CASES[b % len(SCORE_CASES)]
        for e in case["entries"]:
            got = bm[b, :, e["pos"]]
            assert np.all(got.view(np.uint32) == e["score"].view(np.uint32)), (case["name"], e["pos"], got[:4])


@pytest.mark.parametrize("B,Q", [(3, 1), (3, 16), (150, 1)], ids=["cluster", "cluster_q16", "per_share"])
def test_order_cases_index_topk(csa, B, Q):
    kv, q, qs, w, q_pos, want = _setup(csa, B, Q)
    idx, bm = csa.csa2_index_topk(q, qs, w, kv, q_pos, 1, blockmax=True)
    assert np.array_equal(np_(idx)[..., 0], want)
    _check_blockmax(bm, B, Q)


def test_order_cases_many_query_path(csa):
    """192 queries, 64 per batch row: the many-query scoring + selection kernels."""
    B, Q = 3, 64
    kv, q, qs, w, q_pos, want = _setup(csa, B, Q)
    idx = csa.csa2_index_topk(q, qs, w, kv, q_pos, 1)
    assert np.array_equal(np_(idx)[..., 0], want)
    idx2 = csa.csa2_index_topk(q, qs, w, kv, q_pos, 2)
    assert np.array_equal(np_(idx2), np.broadcast_to(np.array([0, STRIDE], np.int32), (B, Q, 2)))


def test_order_cases_pool_topk(csa):
    B, Q = 3, 2
    kv, q, qs, w, q_pos, want = _setup(csa, B, Q)
    pool = torch.full((B, Q, 16), -1, dtype=torch.int32, device="cuda")
    pool[..., 0], pool[..., 1] = 1, 0   # the two blocks holding the entries, in any order
    idx = csa.csa2_pool_topk(q, qs, w, kv, pool, q_pos, 1)
    assert np.array_equal(np_(idx)[..., 0], want)


def test_order_cases_noalloc(csa):
    B, Q = 3, 1
    kv, q, qs, w, q_pos, want = _setup(csa, B, Q)
    idx, bm = csa.csa2_index_topk_noalloc(q, qs, w, kv, q_pos, 1, blockmax=True)
    assert np.array_equal(np_(idx)[..., 0], want)
    _check_blockmax(bm, B, Q)


@pytest.mark.parametrize("case", KPROJ_CASES, ids=lambda c: c["name"])
def test_order_case_index_k_proj(csa, case):
    x = torch.from_numpy(bf16_bits_of(case["x"]).view(np.int16)).view(torch.bfloat16).reshape(1, 512).cuda()
    W = torch.from_numpy(case["W"]).cuda()
    kc, ks = csa.csa2_index_k_proj(x, W)
    gc, gs = ik_untile(np_(kc), np_(ks))
    assert np.array_equal(gc[0, :8], case["kcodes"]) and gs[0, 0] == case["kscale0"]
    assert not gc[0, 8:].any() and not gs[0, 1:].any()
    # the decode append runs its own projection code: same bytes
    lc = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    ls = torch.zeros((128, 32), dtype=torch.uint8, device="cuda")
    kc2 = torch.zeros((128, 32), dtype=torch.uint8, device="cuda")
    ks2 = torch.zeros((128, 4), dtype=torch.uint8, device="cuda")
    csa.csa2_append_tokens(x, W, (lc, ls, kc2, ks2))
    gc2, gs2 = ik_untile(np_(kc2), np_(ks2))
    assert np.array_equal(gc2[0], gc[0]) and np.array_equal(gs2[0], gs[0])
