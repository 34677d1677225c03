"""The C-ABI library loads, exports every symbol include/csa2.h declares, and
rejects invalid arguments on the host before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "csa2.h")).read()
    return sorted(set(re.findall(r"CSA2_API\s+[\w\s\*]+?\b(csa2_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from sparse_attention_fp4_quant_b200 import build
    import sparse_attention_fp4_quant_b200 as csa
    build.build()
    return csa.lib()


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 10
    import sparse_attention_fp4_quant_b200 as csa
    assert sorted(csa.EXPORTS) == names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    assert L.csa2_status_str(0) == b"CSA2_OK"
    assert L.csa2_status_str(1) == b"CSA2_ERR_INVALID_ARG"
    assert L.csa2_status_str(4) == b"CSA2_ERR_CUDA"
    assert L.csa2_status_str(5) == b"CSA2_ERR_TIMEOUT"


def test_workspace_sizes_are_host_only(L):
    import sparse_attention_fp4_quant_b200 as csa
    for op in range(5):
        assert L.csa2_workspace_bytes(op, 32, 1, 131072, 512, 2048) >= 256
    assert L.csa2_workspace_bytes(0, 0, 1, 10, 512, 0) == 0
    # one share per query needs only the counters
    assert L.csa2_workspace_bytes(csa.OP_INDEX_TOPK, 4096, 1, 1000, 512, 0) == 4096 * 4 + 256  # counters + status word
    # many queries per batch row (a prefill chunk): the workspace also holds every query's
    # 16-bit key prefixes and its 2,048-bin histogram for the many-query path
    many = L.csa2_workspace_bytes(csa.OP_INDEX_TOPK, 1, 4096, 32768, 512, 0)
    assert many >= 4096 * 32768 * 2 + 4096 * 2048 * 4
    # up to 262,144 entries (a replay through a long decoder context) too
    assert L.csa2_workspace_bytes(csa.OP_INDEX_TOPK, 4, 128, 262144, 512, 0) >= 512 * 262144 * 2 + 512 * 2048 * 4
    # beyond that the path is not taken, and nothing is reserved for it
    assert L.csa2_workspace_bytes(csa.OP_INDEX_TOPK, 1, 4096, 524288, 512, 0) < 4096 * 524288 * 2
    # a layer whose Reindex runs one CTA per query also keeps the pool search's order keys:
    # 4 B per pool entry, the pool's slots rounded up to whole 128-entry tiles
    for P in (2048, 300):
        layer = L.csa2_workspace_bytes(csa.OP_LAYER, 2, 80, 30080, 512, P)
        pool = L.csa2_workspace_bytes(csa.OP_POOL_TOPK, 2, 80, 30080, 512, P)
        assert layer >= pool + 160 * ((P + 15) // 16) * 128 * 4
    # a decode group above 16 x 32,768 entries keeps the index's order keys (4 B per entry)
    assert L.csa2_workspace_bytes(csa.OP_INDEX_TOPK, 8, 1, 1048576, 512, 0) >= 8 * 1048576 * 4


def test_invalid_arguments_rejected_before_launch(L):
    P = ctypes.c_void_p
    fake = P(0x1000)
    # channel count not a multiple of 16
    assert L.csa2_quant_nvfp4(fake, 4, 15, fake, fake, None, 4, None) == 1
    # misaligned input
    assert L.csa2_quant_nvfp4(P(0x1001), 4, 16, fake, fake, None, 4, None) == 1
    # output smaller than the input without a row map
    assert L.csa2_quant_nvfp4(fake, 4, 16, fake, fake, None, 3, None) == 1
    # rows == 0 is a no-op
    assert L.csa2_quant_nvfp4(None, 0, 16, None, None, None, 0, None) == 0
    # projection matrix not 16-byte aligned
    assert L.csa2_index_k_proj(fake, 4, P(0x1004), fake, fake, None, 4, None) == 1
    import sparse_attention_fp4_quant_b200 as csa
    # indexer-K output rows that are not whole 128-entry tiles
    assert L.csa2_index_k_proj(fake, 4, fake, fake, fake, None, 100, None) == 1
    assert L.csa2_append_tokens(fake, 4, fake, fake, fake, fake, fake, None, 100, None) == 1
    kv = csa.csa2_kv(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 128, 3)  # m = 3 is invalid
    assert L.csa2_index_topk(fake, fake, fake, ctypes.byref(kv), fake, 1, 1, 512, fake, None, fake, 1 << 20,
                             None) == 1
    kv.m = 1
    kv.cap = 1000   # not whole tiles of the indexer-K order
    assert L.csa2_index_topk(fake, fake, fake, ctypes.byref(kv), fake, 1, 1, 512, fake, None, fake, 1 << 20,
                             None) == 1
    kv.cap = 128
    assert L.csa2_index_topk(fake, fake, fake, ctypes.byref(kv), fake, 1, 1, 4096, fake, None, fake, 1 << 20,
                             None) == 1   # k > CSA2_MAX_K
    assert L.csa2_index_topk(fake, fake, fake, ctypes.byref(kv), fake, 1, 1, 512, fake, None, fake, 0,
                             None) == 3   # workspace too small
    assert L.csa2_sparse_attn(fake, ctypes.byref(kv), fake, 512, fake, fake, fake, 128, 129, None, fake, 1, 1,
                              ctypes.c_float(0.04), fake, None, fake, 1 << 20, None) == 1   # window > 128
    assert L.csa2_layer_step(None, None) == 1
    assert L.csa2_device_status(None, 1, 1, 0, None) == 1   # no workspace
