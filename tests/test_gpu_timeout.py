"""The device-side timeout path, run without any fault: a test hook
(csa2_test_starve_copies) makes the per-share scoring kernel announce its first
copy stage but issue no copy, so every CTA's bounded wait (2 s) runs out.  The
call must report CSA2_ERR_TIMEOUT through its sticky flag (csa2_device_status for a
workspace call, csa2_index_topk_noalloc_status for the no-allocation call), the
context must stay usable, and the next normal call must be bit-exact with the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import np_, set_kv_ik_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    import sparse_attention_fp4_quant_b200 as m
    m.lib()
    return m


def _case(csa, seed, B=150, cap=1024):
    # 150 queries, one per batch row: more than one wave of clusters, fewer than 8 per
    # row, so the per-share kernel (one CTA per query here) runs them
    rng = np.random.default_rng(seed)
    ik = rng.integers(0, 256, (B, cap, 32), dtype=np.uint8)
    iks = rng.integers(0x20, 0x50, (B, cap, 4), dtype=np.uint8)
    q = rng.integers(0, 256, (B, 1, 128), dtype=np.uint8)
    qs = rng.integers(0x20, 0x50, (B, 1, 16), dtype=np.uint8)
    w = np.full((B, 1, 4), 0.25, np.float32)
    ne = np.full(B, cap - 24, np.int32)
    q_pos = np.full((B, 1), cap - 25, np.int32)
    kv = csa.KV(B, cap, 1, "cuda")
    set_kv_ik_rows(kv, ik, iks)
    kv.n_entries.copy_(torch.from_numpy(ne))
    dev = [torch.from_numpy(a).cuda() for a in (q, qs, w, q_pos)]
    want = oracle.index_topk(q, qs, w, ik, iks, ne, 1, q_pos, 64)
    return kv, dev, want


def test_timeout_reported_then_recovered(csa):
    kv, (q, qs, w, qp), want = _case(csa, 3)
    B = qp.shape[0]
    ws = torch.zeros(csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, B, 1, kv.cap, 64), dtype=torch.uint8, device="cuda")
    csa.csa2_device_status(ws, B, 1)   # clear to start with
    csa.lib().csa2_test_starve_copies(1)
    try:
        csa.csa2_index_topk(q, qs, w, kv, qp, 64, ws=ws)
        with pytest.raises(csa.CSA2Error, match="TIMEOUT"):
            csa.csa2_device_status(ws, B, 1, clear=True)
    finally:
        csa.lib().csa2_test_starve_copies(0)
    csa.csa2_device_status(ws, B, 1)   # cleared
    got = csa.csa2_index_topk(q, qs, w, kv, qp, 64, ws=ws)
    assert np.array_equal(np_(got), want)
    csa.csa2_device_status(ws, B, 1)


def test_timeout_on_the_no_allocation_call(csa):
    kv, (q, qs, w, qp), want = _case(csa, 4)
    csa.lib().csa2_test_starve_copies(1)
    try:
        csa.csa2_index_topk_noalloc(q, qs, w, kv, qp, 64)
        with pytest.raises(csa.CSA2Error, match="TIMEOUT"):
            csa.csa2_index_topk_noalloc_status()
    finally:
        csa.lib().csa2_test_starve_copies(0)
    got = csa.csa2_index_topk_noalloc(q, qs, w, kv, qp, 64)   # clears the flag, then runs normally
    assert np.array_equal(np_(got), want)
    csa.csa2_index_topk_noalloc_status()
