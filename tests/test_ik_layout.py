"""The indexer-K cache order (codes in 128-entry tiles, the tensor cores' operand
image; scales row-major) as the C header states it, checked against the test
helpers that convert to rows."""
import numpy as np

from gpu_common import ik_tile, ik_untile


def _code_off(e, h):
    return 4096 * (e // 128) + 256 * ((e // 8) % 16) + 128 * h + 16 * (e % 8)


def _scale_off(e):
    return 4 * e


def test_tiled_order_matches_the_header_formula():
    n = 384
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 256, (n, 32), dtype=np.uint8)
    scales = rng.integers(0, 256, (n, 4), dtype=np.uint8)
    tc, ts = ik_tile(codes, scales)
    ref_c = np.zeros(n * 32, np.uint8)
    ref_s = np.zeros(n * 4, np.uint8)
    for e in range(n):
        for h in range(2):
            o = _code_off(e, h)
            ref_c[o:o + 16] = codes[e, 16 * h:16 * h + 16]
        ref_s[_scale_off(e):_scale_off(e) + 4] = scales[e]
    assert np.array_equal(tc, ref_c) and np.array_equal(ts, ref_s)
    # a permutation: every byte lands once, and the inverse restores the rows
    offs = sorted(_code_off(e, h) + j for e in range(n) for h in range(2) for j in range(16))
    assert offs == list(range(n * 32))
    uc, us = ik_untile(tc, ts)
    assert np.array_equal(uc, codes) and np.array_equal(us, scales)


def test_a_pool_block_is_256_contiguous_bytes():
    # 8 consecutive entries starting at a multiple of 8 occupy one 256-byte span
    for e0 in range(0, 512, 8):
        offs = {_code_off(e, h) + j for e in range(e0, e0 + 8) for h in range(2) for j in range(16)}
        base = _code_off(e0, 0)
        assert offs == set(range(base, base + 256))
