"""Pins of the oracle's fixed fp32 orders against hand-worked values (CPU only).

The cases in tests/golden/index_order_cases.txt were derived by hand from the
defined order of the index score (blocks ascending, heads ascending, products
rounded before each add) and of the indexer-K projection (fused multiply-add
chain over the channels in ascending order).  Each case is built so that the
plausible other orders -- pairwise or descending sums, a fused multiply-add,
an exact sum rounded once -- give a different fp32 result, so a change of
order in the oracle fails here.
"""
import numpy as np
import pytest

import oracle
from order_cases import bf16_bits_of, keys_array, load

SCORE_CASES, KPROJ_CASES = load()


def test_golden_file_has_the_cases():
    assert {c["name"] for c in SCORE_CASES} == {"block_order", "head_order", "rounded_products"}
    assert [c["name"] for c in KPROJ_CASES] == ["kproj_chain"]


@pytest.mark.parametrize("case", SCORE_CASES, ids=lambda c: c["name"])
def test_index_score_hand_worked(case):
    for e in case["entries"]:
        got = np.float32(oracle.index_score(case["q"], case["qs"], case["w"], e["k"], e["ks"]))
        assert got.view(np.uint32) == e["score"].view(np.uint32), (case["name"], e["pos"], float(got))


@pytest.mark.parametrize("case", SCORE_CASES, ids=lambda c: c["name"])
@pytest.mark.parametrize("stride", [1, 8])
def test_index_topk_hand_worked(case, stride):
    """The whole selection: Top-1 returns the entry the defined order ranks first,
    and block maxima carry the hand-worked scores."""
    n = 2 * stride
    k, ks = keys_array(case, n, stride)
    q = case["q"].reshape(1, 1, 128)
    qs = case["qs"].reshape(1, 1, 16)
    w = case["w"].reshape(1, 1, 4)
    idx, bm = oracle.index_topk(q, qs, w, k[None], ks[None], np.array([n], np.int32), 1,
                                np.array([[n - 1]], np.int32), 1, blockmax=True)
    assert idx[0, 0, 0] == case["top1"] * stride
    if stride == 8:
        for e in case["entries"]:
            assert bm[0, 0, e["pos"]].view(np.uint32) == e["score"].view(np.uint32)


@pytest.mark.parametrize("case", KPROJ_CASES, ids=lambda c: c["name"])
def test_index_k_proj_hand_worked(case):
    x = bf16_bits_of(case["x"]).reshape(1, 512)
    got = oracle.index_k_proj_f32(x, case["W"])[0]
    want = np.zeros(64, np.float32)
    for j, v in case["out"].items():
        want[j] = v
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), got[[0, 7]]
    codes, scales = oracle.index_k_proj(x, case["W"])
    assert np.array_equal(codes[0, :8], case["kcodes"]) and scales[0, 0] == case["kscale0"]
    assert not codes[0, 8:].any() and not scales[0, 1:].any()
