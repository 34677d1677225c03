"""CPU oracle for the CSA2 hot path (ctypes wrapper around ``csa2_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``.  The CUDA library and
its binding never import this package, and this package imports nothing from
them.  All arrays are numpy; bf16 tensors are passed as their uint16 bit
patterns.

Sources: the three public pages on DeepSeek-V4.1-Flash -- the shibing624 blog
"一个 token 只花 890 字节" (sections "CSA2：跨层复用", "分层稀疏索引器" Fig. 5,
"FP4 与 SWA Bounded Replay"), the jdon.com article ("缓存压缩真的是越大越好吗")
and m.lsln.cn news 211874 (§4.3 消融实验).
"""
import ctypes
import math

import numpy as np

from . import build as _build

D, H, IH, ID, BLK = 512, 16, 4, 64, 8

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.orc_e2m1_value.restype = dbl
        L.orc_e2m1_value.argtypes = [ctypes.c_uint]
        L.orc_e4m3_value.restype = dbl
        L.orc_e4m3_value.argtypes = [ctypes.c_uint]
        L.orc_e4m3_encode.restype = ctypes.c_uint
        L.orc_e4m3_encode.argtypes = [dbl]
        L.orc_quant_nvfp4_f32.argtypes = [P, i64, i32, P, P]
        L.orc_quant_nvfp4_bf16.argtypes = [P, i64, i32, P, P]
        L.orc_dequant_nvfp4.argtypes = [P, P, i64, i32, P]
        L.orc_index_k_proj_f32.argtypes = [P, i64, P, P]
        L.orc_index_k_proj.argtypes = [P, i64, P, P, P]
        L.orc_index_score.restype = ctypes.c_float
        L.orc_index_score.argtypes = [P, P, P, P, P]
        L.orc_n_visible.restype = i64
        L.orc_n_visible.argtypes = [i64, i64, i32]
        L.orc_index_topk.argtypes = [P, P, P, P, P, P, i64, i32, P, i32, i32, i32, P, P, i64]
        L.orc_pool_build.argtypes = [P, i64, P, i32, P, i32, i32, i32, P]
        L.orc_pool_topk.argtypes = [P, P, P, P, P, P, i64, i32, P, i32, P, i32, i32, i32, P]
        L.orc_sparse_attn.argtypes = [P, P, P, P, i64, P, i32, P, P, P, i32, i32, P, P,
                                      i32, i32, dbl, P, P]
        L.orc_front_end_f32.argtypes = [P, i64, P, P, P, ctypes.c_float, P]
        L.orc_front_end.argtypes = [P, i64, P, P, P, ctypes.c_float, P]
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- formats
def e2m1_value(code):
    return lib().orc_e2m1_value(int(code))


def e4m3_value(byte):
    return lib().orc_e4m3_value(int(byte))


def e4m3_encode(v):
    return lib().orc_e4m3_encode(float(v))


def quant_nvfp4(x):
    """x: float32 [rows, ch] or uint16 bf16 bits [rows, ch] -> (codes u8 [rows, ch/2], scales u8 [rows, ch/16])."""
    x = np.asarray(x)
    rows, ch = x.shape
    assert ch % 16 == 0
    packed = np.zeros((rows, ch // 2), np.uint8)
    scales = np.zeros((rows, ch // 16), np.uint8)
    if x.dtype == np.uint16:
        xc = _c(x, np.uint16)
        lib().orc_quant_nvfp4_bf16(_p(xc), rows, ch, _p(packed), _p(scales))
    else:
        xc = _c(x, np.float32)
        lib().orc_quant_nvfp4_f32(_p(xc), rows, ch, _p(packed), _p(scales))
    return packed, scales


def dequant_nvfp4(packed, scales):
    packed = _c(packed, np.uint8)
    scales = _c(scales, np.uint8)
    rows = packed.shape[0]
    ch = packed.shape[-1] * 2
    out = np.zeros((rows, ch), np.float64)
    lib().orc_dequant_nvfp4(_p(packed), _p(scales), rows, ch, _p(out))
    return out


# ---------------------------------------------------------------- front end
def front_end(x_bf16, cos, sin, w=None, eps=1e-6, f32=False):
    """RMSNorm (eps, optional per-channel weight) then RoPE on channels 448..511 (pairs
    (448 + 2k, 449 + 2k) with the caller's cos/sin [rows, 32]) of bf16 latents [rows, 512]:
    bf16 bits [rows, 512] (or the fp32 values before the bf16 rounding with f32=True)."""
    x = _c(x_bf16, np.uint16).reshape(-1, D)
    rows = x.shape[0]
    cos = _c(cos, np.float32).reshape(rows, 32)
    sin = _c(sin, np.float32).reshape(rows, 32)
    wv = None if w is None else _c(w, np.float32).reshape(D)
    if f32:
        out = np.zeros((rows, D), np.float32)
        lib().orc_front_end_f32(_p(x), rows, _p(cos), _p(sin), _p(wv), float(eps), _p(out))
    else:
        out = np.zeros((rows, D), np.uint16)
        lib().orc_front_end(_p(x), rows, _p(cos), _p(sin), _p(wv), float(eps), _p(out))
    return out


# ---------------------------------------------------------------- indexer
def index_k_proj_f32(x_bf16, W):
    x = _c(x_bf16, np.uint16).reshape(-1, D)
    W = _c(W, np.float32)
    out = np.zeros((x.shape[0], ID), np.float32)
    lib().orc_index_k_proj_f32(_p(x), x.shape[0], _p(W), _p(out))
    return out


def index_k_proj(x_bf16, W):
    x = _c(x_bf16, np.uint16).reshape(-1, D)
    W = _c(W, np.float32)
    codes = np.zeros((x.shape[0], ID // 2), np.uint8)
    scales = np.zeros((x.shape[0], ID // 16), np.uint8)
    lib().orc_index_k_proj(_p(x), x.shape[0], _p(W), _p(codes), _p(scales))
    return codes, scales


def index_score(q, qs, w, k, ks):
    q, qs, k, ks = (_c(a, np.uint8) for a in (q, qs, k, ks))
    w = _c(w, np.float32)
    return lib().orc_index_score(_p(q), _p(qs), _p(w), _p(k), _p(ks))


def n_visible(q_pos, n_entries, m):
    return lib().orc_n_visible(int(q_pos), int(n_entries), int(m))


def index_topk(q, qs, w, ik, iks, n_entries, m, q_pos, k, blockmax=False):
    """q [B,Q,128] u8, qs [B,Q,16] u8, w [B,Q,4] f32, ik [B,cap,32] u8, iks [B,cap,4] u8,
    n_entries [B] i32, q_pos [B,Q] i32 -> idx [B,Q,k] i32 (and blockmax [B,Q,ceil(cap/8)] f32)."""
    q, qs, ik, iks = (_c(a, np.uint8) for a in (q, qs, ik, iks))
    w = _c(w, np.float32)
    n_entries = _c(n_entries, np.int32)
    q_pos = _c(q_pos, np.int32)
    B, Q = q_pos.shape
    cap = ik.shape[1]
    nb_cap = (cap + BLK - 1) // BLK
    idx = np.zeros((B, Q, k), np.int32)
    bm = np.zeros((B, Q, nb_cap), np.float32) if blockmax else None
    lib().orc_index_topk(_p(q), _p(qs), _p(w), _p(ik), _p(iks), _p(n_entries), cap, m,
                         _p(q_pos), B, Q, k, _p(idx), _p(bm), nb_cap)
    return (idx, bm) if blockmax else idx


def pool_build(blockmax, n_entries, m, q_pos, max_blocks):
    bm = _c(blockmax, np.float32)
    n_entries = _c(n_entries, np.int32)
    q_pos = _c(q_pos, np.int32)
    B, Q = q_pos.shape
    pool = np.zeros((B, Q, max_blocks), np.int32)
    lib().orc_pool_build(_p(bm), bm.shape[-1], _p(n_entries), m, _p(q_pos), B, Q, max_blocks, _p(pool))
    return pool


def pool_topk(q, qs, w, ik, iks, n_entries, m, pool, q_pos, k):
    q, qs, ik, iks = (_c(a, np.uint8) for a in (q, qs, ik, iks))
    w = _c(w, np.float32)
    n_entries = _c(n_entries, np.int32)
    pool = _c(pool, np.int32)
    q_pos = _c(q_pos, np.int32)
    B, Q = q_pos.shape
    cap = ik.shape[1]
    idx = np.zeros((B, Q, k), np.int32)
    lib().orc_pool_topk(_p(q), _p(qs), _p(w), _p(ik), _p(iks), _p(n_entries), cap, m,
                        _p(pool), pool.shape[-1], _p(q_pos), B, Q, k, _p(idx))
    return idx


# ---------------------------------------------------------------- attention
def sparse_attn(q_bf16, lat, lat_sc, n_entries, idx, swa, swa_sc, swa_pos0, window,
                replay_start, q_pos, sm_scale=1.0 / math.sqrt(D)):
    """q_bf16 u16 [B,Q,16,512]; lat u8 [B,cap,256]; lat_sc u8 [B,cap,32]; idx i32 [B,Q,k];
    swa u8 [B,T,512]; swa_sc f32 [B,T]; swa_pos0 i32 [B]; replay_start i32 [B] or None;
    q_pos i32 [B,Q]  ->  out f64 [B,Q,16,512], lse f64 [B,Q,16]."""
    q = _c(q_bf16, np.uint16)
    lat, lat_sc, swa = (_c(a, np.uint8) for a in (lat, lat_sc, swa))
    n_entries = _c(n_entries, np.int32)
    idx = _c(idx, np.int32)
    swa_sc = _c(swa_sc, np.float32)
    swa_pos0 = _c(swa_pos0, np.int32)
    rs = None if replay_start is None else _c(replay_start, np.int32)
    q_pos = _c(q_pos, np.int32)
    B, Q = q_pos.shape
    cap = lat.shape[1]
    T = swa.shape[1]
    k = idx.shape[-1]
    out = np.zeros((B, Q, H, D), np.float64)
    lse = np.zeros((B, Q, H), np.float64)
    lib().orc_sparse_attn(_p(q), _p(lat), _p(lat_sc), _p(n_entries), cap, _p(idx), k,
                          _p(swa), _p(swa_sc), _p(swa_pos0), T, window, _p(rs), _p(q_pos),
                          B, Q, float(sm_scale), _p(out), _p(lse))
    return out, lse


# ---------------------------------------------------------------- layer modes
# [Blog] "CSA2：跨层复用" (Fig. 4): Full computes main KV + indexer K and a
# fresh Top-K; Reindex borrows the global KV and re-scores with its own
# indexer Q; Reuse borrows the indices too.  Every mode keeps its own global Q
# and SWA KV.  Decoder: 1 Full + 3 Reuse, then 4 x (1 Reindex + 3 Reuse).
# Encoder: 3 groups of 1 Full + 5 Reuse (after 2 pure-SWA layers).
DECODER_PATTERN = ["full", "reuse", "reuse", "reuse"] + ["reindex", "reuse", "reuse", "reuse"] * 4
ENCODER_CSA2_PATTERN = (["full"] + ["reuse"] * 5) * 3


def layer_step(mode, st, layer):
    """One CSA2 layer on the oracle.

    ``st`` is a dict holding the shared state of a layer group (the quantised
    main KV and indexer K, the current indices and pool) and ``layer`` the
    layer's own inputs: attention Q (bf16 bits), indexer Q codes/scales/w,
    SWA KV and mask parameters.  Returns (out, lse)."""
    if mode == "full":
        idx, bm = index_topk(layer["iq"], layer["iqs"], layer["w"], st["ik"], st["iks"],
                             st["n_entries"], st["m"], layer["q_pos"], st["k"], blockmax=True)
        st["idx"] = idx
        if st.get("build_pool"):
            st["pool"] = pool_build(bm, st["n_entries"], st["m"], layer["q_pos"], st["pool_blocks"])
    elif mode == "reindex":
        st["idx"] = pool_topk(layer["iq"], layer["iqs"], layer["w"], st["ik"], st["iks"],
                              st["n_entries"], st["m"], st["pool"], layer["q_pos"], st["k"])
    elif mode != "reuse":
        raise ValueError(mode)
    return sparse_attn(layer["q"], st["lat"], st["lat_sc"], st["n_entries"], st["idx"],
                       layer["swa"], layer["swa_sc"], layer["swa_pos0"], layer["window"],
                       layer.get("replay_start"), layer["q_pos"], layer.get("sm_scale", 1.0 / math.sqrt(D)))
