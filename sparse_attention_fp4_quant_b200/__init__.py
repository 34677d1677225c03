"""Python binding of libcsa2.so (include/csa2.h): argument marshalling only.

Every function has the name of the C entry point it calls and takes torch
tensors resident on the current CUDA device; outputs that are not passed in
are allocated with torch (device memory is the only thing torch provides here).
All work runs in the library's CUDA kernels on torch's current stream.  There
is no fallback: if the library is missing or its call fails, an exception is
raised.
"""
import ctypes
import math
import os

import torch

D, H, IH, ID, BLOCK, MAX_K, MAX_WINDOW = 512, 16, 4, 64, 8, 2048, 128
IK_TILE = 128   # entries per tile of the indexer-K cache order
TOPK, POOL_BLOCKS, WINDOW = 512, 2048, 128

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

OP_INDEX_TOPK, OP_POOL_BUILD, OP_POOL_TOPK, OP_SPARSE_ATTN, OP_LAYER = range(5)
MODE_FULL, MODE_REINDEX, MODE_REUSE = range(3)
MODES = {"full": MODE_FULL, "reindex": MODE_REINDEX, "reuse": MODE_REUSE}


class csa2_kv(ctypes.Structure):
    _fields_ = [("lat", ctypes.c_void_p), ("lat_sc", ctypes.c_void_p), ("ik", ctypes.c_void_p),
                ("ik_sc", ctypes.c_void_p), ("n_entries", ctypes.c_void_p), ("cap", ctypes.c_int64),
                ("m", ctypes.c_int32)]


class csa2_layer_args(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("kv", ctypes.POINTER(csa2_kv)), ("B", ctypes.c_int32),
                ("Q", ctypes.c_int32), ("q_pos", ctypes.c_void_p), ("new_latent", ctypes.c_void_p),
                ("n_new", ctypes.c_int64), ("new_rows", ctypes.c_void_p), ("k_proj", ctypes.c_void_p),
                ("iq", ctypes.c_void_p), ("iq_sc", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("idx", ctypes.c_void_p), ("k", ctypes.c_int32), ("pool", ctypes.c_void_p),
                ("pool_blocks", ctypes.c_int32), ("blockmax", ctypes.c_void_p), ("q", ctypes.c_void_p),
                ("swa", ctypes.c_void_p), ("swa_sc", ctypes.c_void_p), ("swa_pos0", ctypes.c_void_p),
                ("T", ctypes.c_int32), ("window", ctypes.c_int32), ("replay_start", ctypes.c_void_p),
                ("sm_scale", ctypes.c_float), ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("ws", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t)]


_lib = None
EXPORTS = ["csa2_status_str", "csa2_last_cuda_error", "csa2_quant_nvfp4", "csa2_index_k_proj", "csa2_append_tokens",
           "csa2_index_topk",
           "csa2_pool_build", "csa2_pool_topk", "csa2_sparse_attn", "csa2_workspace_bytes", "csa2_layer_step",
           "csa2_index_topk_noalloc", "csa2_index_topk_noalloc_status", "csa2_device_status", "csa2_front_end",
           "csa2_test_starve_copies"]
NOALLOC_SCRATCH_BYTES = 4 << 20


def lib():
    """Load libcsa2.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_attention_fp4_quant_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    KVP = ctypes.POINTER(csa2_kv)
    sig = {
        "csa2_status_str": (ctypes.c_char_p, [ctypes.c_int]),
        "csa2_last_cuda_error": (ctypes.c_int, []),
        "csa2_quant_nvfp4": (ctypes.c_int, [P, i64, i32, P, P, P, i64, P]),
        "csa2_index_k_proj": (ctypes.c_int, [P, i64, P, P, P, P, i64, P]),
        "csa2_append_tokens": (ctypes.c_int, [P, i64, P, P, P, P, P, P, i64, P]),
        "csa2_device_status": (ctypes.c_int, [P, i32, i32, i32, P]),
        "csa2_index_topk": (ctypes.c_int, [P, P, P, KVP, P, i32, i32, i32, P, P, P, sz, P]),
        "csa2_pool_build": (ctypes.c_int, [P, KVP, P, i32, i32, i32, P, P, sz, P]),
        "csa2_pool_topk": (ctypes.c_int, [P, P, P, KVP, P, i32, P, i32, i32, i32, P, P, sz, P]),
        "csa2_sparse_attn": (ctypes.c_int, [P, KVP, P, i32, P, P, P, i32, i32, P, P, i32, i32, ctypes.c_float,
                                            P, P, P, sz, P]),
        "csa2_workspace_bytes": (sz, [ctypes.c_int, i32, i32, i64, i32, i32]),
        "csa2_layer_step": (ctypes.c_int, [ctypes.POINTER(csa2_layer_args), P]),
        "csa2_index_topk_noalloc": (ctypes.c_int, [P, P, P, KVP, P, i32, i32, i32, P, P, P]),
        "csa2_index_topk_noalloc_status": (ctypes.c_int, [i32, P]),
        "csa2_test_starve_copies": (None, [i32]),
        "csa2_front_end": (ctypes.c_int, [P, i64, P, P, P, ctypes.c_float, P, P, P, P, P, P, i64, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


class CSA2Error(RuntimeError):
    pass


def _check(status):
    if status != 0:
        L = lib()
        msg = L.csa2_status_str(status).decode()
        if status == 4:
            msg += f" (cudaError {L.csa2_last_cuda_error()})"
        raise CSA2Error(msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t, dtype, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous CUDA tensor of {dtype}, got {t.dtype} on {t.device}")
    return t


def _size(t, n, name):
    if t.numel() != n:
        raise ValueError(f"{name}: expected {n} elements, got {t.numel()} (shape {tuple(t.shape)})")
    return t


def _batch(kv, B):
    if kv.B != B:
        raise ValueError(f"q_pos has {B} batch rows but the KV has {kv.B}")


class KV:
    """The shared global KV of a CSA2 layer group (device tensors) and its csa2_kv view."""

    def __init__(self, B, cap, m=1, device="cuda"):
        if cap <= 0 or cap % IK_TILE:
            raise ValueError(f"cap must be a positive multiple of {IK_TILE} (the indexer-K tile), got {cap}")
        self.B, self.cap, self.m = B, cap, m
        self.lat = torch.zeros((B, cap, D // 2), dtype=torch.uint8, device=device)
        self.lat_sc = torch.zeros((B, cap, D // 16), dtype=torch.uint8, device=device)
        self.ik = torch.zeros((B, cap, ID // 2), dtype=torch.uint8, device=device)
        self.ik_sc = torch.zeros((B, cap, ID // 16), dtype=torch.uint8, device=device)
        self.n_entries = torch.zeros((B,), dtype=torch.int32, device=device)

    def c(self):
        self._c = csa2_kv(self.lat.data_ptr(), self.lat_sc.data_ptr(), self.ik.data_ptr(), self.ik_sc.data_ptr(),
                          self.n_entries.data_ptr(), self.cap, self.m)
        return ctypes.byref(self._c)


class Workspace:
    """A zero-filled device workspace, grown on demand (the library keeps its counters at zero)."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = torch.zeros(256, dtype=torch.uint8, device=device)

    def get(self, nbytes):
        if nbytes > self.buf.numel():
            self.buf = torch.zeros(int(nbytes), dtype=torch.uint8, device=self.device)
        return self.buf


_ws = {}


def _workspace(nbytes):
    dev = torch.cuda.current_device()
    if dev not in _ws:
        _ws[dev] = Workspace(f"cuda:{dev}")
    return _ws[dev].get(nbytes)


def status_offset(B, Q):
    """Byte offset of the sticky device error flag in an index / pool workspace (CSA2_STATUS_OFFSET)."""
    return (B * Q * 4 + 255) & ~255


def device_error_flag(ws, B, Q):
    """The workspace's sticky device error flag (1 after a device-side wait ran out of time)."""
    off = status_offset(B, Q)
    return int(ws[off:off + 4].view(torch.int32).item())


def csa2_device_status(ws, B, Q, clear=False):
    """Waits for the current stream; raises CSA2Error (CSA2_ERR_TIMEOUT) if a call on this
    workspace had a device-side wait run out of time."""
    _check(lib().csa2_device_status(_ptr(ws), B, Q, 1 if clear else 0, _stream()))


def csa2_workspace_bytes(op, B, Q, cap, k, P=0):
    return int(lib().csa2_workspace_bytes(op, B, Q, cap, k, P))


def csa2_quant_nvfp4(x, codes=None, scales=None, dst_rows=None):
    """x: bf16 [rows, ch] -> (codes u8 [rows, ch/2], scales u8 [rows, ch/16]); with dst_rows, written in place."""
    _dev(x, torch.bfloat16, "x")
    rows, ch = x.reshape(-1, x.shape[-1]).shape
    if codes is None:
        codes = torch.empty((rows, ch // 2), dtype=torch.uint8, device=x.device)
        scales = torch.empty((rows, ch // 16), dtype=torch.uint8, device=x.device)
    if dst_rows is not None:
        _dev(dst_rows, torch.int64, "dst_rows")
    _check(lib().csa2_quant_nvfp4(_ptr(x), rows, ch, _ptr(codes), _ptr(scales), _ptr(dst_rows),
                                  codes.numel() // (ch // 2), _stream()))
    return codes, scales


def csa2_index_k_proj(x, W, k_codes=None, k_scales=None, dst_rows=None):
    _dev(x, torch.bfloat16, "x")
    _dev(W, torch.float32, "W")
    rows = x.reshape(-1, D).shape[0]
    if k_codes is None:   # whole tiles of the indexer-K order
        out_rows = (rows + IK_TILE - 1) // IK_TILE * IK_TILE
        k_codes = torch.empty((out_rows, ID // 2), dtype=torch.uint8, device=x.device)
        k_scales = torch.empty((out_rows, ID // 16), dtype=torch.uint8, device=x.device)
    if dst_rows is not None:
        _dev(dst_rows, torch.int64, "dst_rows")
    _check(lib().csa2_index_k_proj(_ptr(x), rows, _ptr(W), _ptr(k_codes), _ptr(k_scales), _ptr(dst_rows),
                                   k_codes.numel() // (ID // 2), _stream()))
    return k_codes, k_scales


def csa2_append_tokens(x, W, kv_or_outs, dst_rows=None):
    """Quantise new latent rows x (bf16 [rows, 512]) into the main KV and project + quantise their
    indexer K, in one launch.  kv_or_outs: a KV (rows land at dst_rows of its [B*cap] cache) or a
    tuple (lat_codes, lat_scales, k_codes, k_scales)."""
    _dev(x, torch.bfloat16, "x")
    _dev(W, torch.float32, "W")
    _size(W, D * ID, "W")
    rows = x.reshape(-1, D).shape[0]
    if isinstance(kv_or_outs, KV):
        kv = kv_or_outs
        lc, ls, kc, ks = kv.lat, kv.lat_sc, kv.ik, kv.ik_sc
        out_rows = kv.B * kv.cap
    else:
        lc, ls, kc, ks = kv_or_outs
        out_rows = lc.numel() // (D // 2)
    if dst_rows is not None:
        _dev(dst_rows, torch.int64, "dst_rows")
        _size(dst_rows, rows, "dst_rows")
    elif out_rows < rows:
        raise ValueError("outputs have fewer rows than x")
    for t, n, per in ((lc, "lat_codes", D // 2), (ls, "lat_scales", D // 16), (kc, "k_codes", ID // 2),
                      (ks, "k_scales", ID // 16)):
        _size(_dev(t, torch.uint8, n), out_rows * per, n)
    _check(lib().csa2_append_tokens(_ptr(x), rows, _ptr(W), _ptr(lc), _ptr(ls), _ptr(kc), _ptr(ks), _ptr(dst_rows),
                                    out_rows, _stream()))


def csa2_front_end(x, rope_cos, rope_sin, W, kv_or_outs, dst_rows=None, norm_w=None, eps=1e-6, y_out=None):
    """Pre-norm bf16 rows x [rows, 512] -> RMSNorm, RoPE (fp32 cos/sin [rows, 32]), bf16, then the
    append's bytes into a KV (or a tuple (lat_codes, lat_scales, k_codes, k_scales)); y_out, if given,
    receives the post-RoPE bf16 rows."""
    _dev(x, torch.bfloat16, "x")
    rows = x.numel() // D
    _size(x, rows * D, "x")
    _size(_dev(rope_cos, torch.float32, "rope_cos"), rows * 32, "rope_cos")
    _size(_dev(rope_sin, torch.float32, "rope_sin"), rows * 32, "rope_sin")
    _size(_dev(W, torch.float32, "W"), D * ID, "W")
    if norm_w is not None:
        _size(_dev(norm_w, torch.float32, "norm_w"), D, "norm_w")
    if isinstance(kv_or_outs, KV):
        lc, ls, kc, ks = kv_or_outs.lat, kv_or_outs.lat_sc, kv_or_outs.ik, kv_or_outs.ik_sc
    else:
        lc, ls, kc, ks = kv_or_outs
    out_rows = lc.numel() // (D // 2)
    for t, n, per in ((lc, "lat_codes", D // 2), (ls, "lat_scales", D // 16), (kc, "k_codes", ID // 2),
                      (ks, "k_scales", ID // 16)):
        _size(_dev(t, torch.uint8, n), out_rows * per, n)
    if dst_rows is not None:
        _size(_dev(dst_rows, torch.int64, "dst_rows"), rows, "dst_rows")
    if y_out is not None:
        _size(_dev(y_out, torch.bfloat16, "y_out"), rows * D, "y_out")
    _check(lib().csa2_front_end(_ptr(x), rows, _ptr(rope_cos), _ptr(rope_sin), _ptr(norm_w), float(eps), _ptr(W),
                                _ptr(lc), _ptr(ls), _ptr(kc), _ptr(ks), _ptr(dst_rows), out_rows, _ptr(y_out),
                                _stream()))


def csa2_index_topk(q, q_sc, w, kv, q_pos, k, idx_out=None, blockmax=False, ws=None):
    """q u8 [B,Q,128], q_sc u8 [B,Q,16], w f32 [B,Q,4], q_pos i32 [B,Q] -> idx i32 [B,Q,k] (, blockmax f32)."""
    B, Q = q_pos.shape
    for t, dt, n in ((q, torch.uint8, "q"), (q_sc, torch.uint8, "q_sc"), (w, torch.float32, "w"),
                     (q_pos, torch.int32, "q_pos")):
        _dev(t, dt, n)
    _batch(kv, B)
    _size(q, B * Q * 128, "q"), _size(q_sc, B * Q * 16, "q_sc"), _size(w, B * Q * 4, "w")
    if idx_out is None:
        idx_out = torch.empty((B, Q, k), dtype=torch.int32, device=q.device)
    _size(_dev(idx_out, torch.int32, "idx_out"), B * Q * k, "idx_out")
    bm = None
    if blockmax is not False:
        bm = blockmax if isinstance(blockmax, torch.Tensor) else torch.empty(
            (B, Q, (kv.cap + BLOCK - 1) // BLOCK), dtype=torch.float32, device=q.device)
        _size(_dev(bm, torch.float32, "blockmax"), B * Q * ((kv.cap + BLOCK - 1) // BLOCK), "blockmax")
    nbytes = csa2_workspace_bytes(OP_INDEX_TOPK, B, Q, kv.cap, k)
    ws = _workspace(nbytes) if ws is None else ws
    _check(lib().csa2_index_topk(_ptr(q), _ptr(q_sc), _ptr(w), kv.c(), _ptr(q_pos), B, Q, k, _ptr(idx_out),
                                 _ptr(bm), _ptr(ws), ws.numel(), _stream()))
    return (idx_out, bm) if bm is not None else idx_out


def csa2_index_topk_noalloc(q, q_sc, w, kv, q_pos, k, idx_out=None, blockmax=False):
    """csa2_index_topk for callers that cannot allocate device memory: the scratch is the
    library's own static device array (CSA2_NOALLOC_SCRATCH_BYTES per GPU); calls that overlap
    on the GPU race on it."""
    B, Q = q_pos.shape
    for t, dt, n in ((q, torch.uint8, "q"), (q_sc, torch.uint8, "q_sc"), (w, torch.float32, "w"),
                     (q_pos, torch.int32, "q_pos")):
        _dev(t, dt, n)
    _batch(kv, B)
    _size(q, B * Q * 128, "q"), _size(q_sc, B * Q * 16, "q_sc"), _size(w, B * Q * 4, "w")
    if idx_out is None:
        idx_out = torch.empty((B, Q, k), dtype=torch.int32, device=q.device)
    _size(_dev(idx_out, torch.int32, "idx_out"), B * Q * k, "idx_out")
    bm = None
    if blockmax is not False:
        bm = blockmax if isinstance(blockmax, torch.Tensor) else torch.empty(
            (B, Q, (kv.cap + BLOCK - 1) // BLOCK), dtype=torch.float32, device=q.device)
        _size(_dev(bm, torch.float32, "blockmax"), B * Q * ((kv.cap + BLOCK - 1) // BLOCK), "blockmax")
    _check(lib().csa2_index_topk_noalloc(_ptr(q), _ptr(q_sc), _ptr(w), kv.c(), _ptr(q_pos), B, Q, k, _ptr(idx_out),
                                         _ptr(bm), _stream()))
    return (idx_out, bm) if bm is not None else idx_out


def csa2_index_topk_noalloc_status(clear=False):
    """Waits for the current stream; raises CSA2Error (CSA2_ERR_TIMEOUT) if the last
    csa2_index_topk_noalloc call on this device had a device-side wait run out of time."""
    _check(lib().csa2_index_topk_noalloc_status(1 if clear else 0, _stream()))


def csa2_pool_build(blockmax, kv, q_pos, max_blocks=POOL_BLOCKS, pool_out=None, ws=None):
    B, Q = q_pos.shape
    _dev(blockmax, torch.float32, "blockmax")
    _dev(q_pos, torch.int32, "q_pos")
    _batch(kv, B)
    _size(blockmax, B * Q * ((kv.cap + BLOCK - 1) // BLOCK), "blockmax")
    if pool_out is None:
        pool_out = torch.empty((B, Q, max_blocks), dtype=torch.int32, device=blockmax.device)
    _size(_dev(pool_out, torch.int32, "pool_out"), B * Q * max_blocks, "pool_out")
    nbytes = csa2_workspace_bytes(OP_POOL_BUILD, B, Q, kv.cap, max_blocks)
    ws = _workspace(nbytes) if ws is None else ws
    _check(lib().csa2_pool_build(_ptr(blockmax), kv.c(), _ptr(q_pos), B, Q, max_blocks, _ptr(pool_out), _ptr(ws),
                                 ws.numel(), _stream()))
    return pool_out


def csa2_pool_topk(q, q_sc, w, kv, pool, q_pos, k, idx_out=None, ws=None):
    B, Q = q_pos.shape
    P = pool.shape[-1]
    for t, dt, n in ((q, torch.uint8, "q"), (q_sc, torch.uint8, "q_sc"), (w, torch.float32, "w"),
                     (pool, torch.int32, "pool"), (q_pos, torch.int32, "q_pos")):
        _dev(t, dt, n)
    _batch(kv, B)
    _size(q, B * Q * 128, "q"), _size(q_sc, B * Q * 16, "q_sc"), _size(w, B * Q * 4, "w")
    _size(pool, B * Q * P, "pool")
    if idx_out is None:
        idx_out = torch.empty((B, Q, k), dtype=torch.int32, device=q.device)
    _size(_dev(idx_out, torch.int32, "idx_out"), B * Q * k, "idx_out")
    nbytes = csa2_workspace_bytes(OP_POOL_TOPK, B, Q, kv.cap, k, P)
    ws = _workspace(nbytes) if ws is None else ws
    _check(lib().csa2_pool_topk(_ptr(q), _ptr(q_sc), _ptr(w), kv.c(), _ptr(pool), P, _ptr(q_pos), B, Q, k,
                                _ptr(idx_out), _ptr(ws), ws.numel(), _stream()))
    return idx_out


def csa2_sparse_attn(q, kv, idx, swa, swa_sc, swa_pos0, q_pos, window=WINDOW, replay_start=None,
                     sm_scale=1.0 / math.sqrt(D), out=None, lse=False, ws=None):
    """q bf16 [B,Q,16,512]; idx i32 [B,Q,k]; swa u8 [B,T,512]; swa_sc f32 [B,T]; swa_pos0 i32 [B]
    -> out bf16 [B,Q,16,512] (, lse f32 [B,Q,16])."""
    B, Q = q_pos.shape
    _dev(q, torch.bfloat16, "q")
    _dev(idx, torch.int32, "idx")
    _dev(swa, torch.uint8, "swa")
    _dev(swa_sc, torch.float32, "swa_sc")
    _dev(swa_pos0, torch.int32, "swa_pos0")
    _dev(q_pos, torch.int32, "q_pos")
    if replay_start is not None:
        _dev(replay_start, torch.int32, "replay_start")
    k = idx.shape[-1]
    T = swa.shape[1]
    _batch(kv, B)
    _size(q, B * Q * H * D, "q"), _size(idx, B * Q * k, "idx"), _size(swa, B * T * D, "swa")
    _size(swa_sc, B * T, "swa_sc"), _size(swa_pos0, B, "swa_pos0")
    if replay_start is not None:
        _size(replay_start, B, "replay_start")
    if out is None:
        out = torch.empty((B, Q, H, D), dtype=torch.bfloat16, device=q.device)
    _size(_dev(out, torch.bfloat16, "out"), B * Q * H * D, "out")
    lse_t = None
    if lse is not False:
        lse_t = lse if isinstance(lse, torch.Tensor) else torch.empty((B, Q, H), dtype=torch.float32,
                                                                      device=q.device)
    nbytes = csa2_workspace_bytes(OP_SPARSE_ATTN, B, Q, kv.cap, k)
    ws = _workspace(nbytes) if ws is None else ws
    _check(lib().csa2_sparse_attn(_ptr(q), kv.c(), _ptr(idx), k, _ptr(swa), _ptr(swa_sc), _ptr(swa_pos0), T, window,
                                  _ptr(replay_start), _ptr(q_pos), B, Q, float(sm_scale), _ptr(out), _ptr(lse_t),
                                  _ptr(ws), ws.numel(), _stream()))
    return (out, lse_t) if lse_t is not None else out


def csa2_layer_step(mode, kv, q_pos, q, swa, swa_sc, swa_pos0, idx, k=TOPK, iq=None, iq_sc=None, w=None,
                    pool=None, pool_blocks=POOL_BLOCKS, blockmax=None, new_latent=None, new_rows=None, k_proj=None,
                    window=WINDOW, replay_start=None, sm_scale=1.0 / math.sqrt(D), out=None, lse=None, ws=None):
    """One CSA2 layer dispatched by mode ('full' | 'reindex' | 'reuse'); returns the attention output."""
    B, Q = q_pos.shape
    _batch(kv, B)
    if out is None:
        out = torch.empty((B, Q, H, D), dtype=torch.bfloat16, device=q.device)
    P = pool.shape[-1] if pool is not None else pool_blocks
    nbytes = csa2_workspace_bytes(OP_LAYER, B, Q, kv.cap, k, P)
    ws = _workspace(nbytes) if ws is None else ws
    a = csa2_layer_args()
    a.mode = MODES[mode] if isinstance(mode, str) else int(mode)
    a.kv = ctypes.pointer(csa2_kv(kv.lat.data_ptr(), kv.lat_sc.data_ptr(), kv.ik.data_ptr(), kv.ik_sc.data_ptr(),
                                  kv.n_entries.data_ptr(), kv.cap, kv.m))
    a.B, a.Q = B, Q
    a.q_pos = q_pos.data_ptr()
    a.new_latent = new_latent.data_ptr() if new_latent is not None else None
    a.n_new = new_latent.shape[0] if new_latent is not None else 0
    a.new_rows = new_rows.data_ptr() if new_rows is not None else None
    a.k_proj = k_proj.data_ptr() if k_proj is not None else None
    a.iq = iq.data_ptr() if iq is not None else None
    a.iq_sc = iq_sc.data_ptr() if iq_sc is not None else None
    a.w = w.data_ptr() if w is not None else None
    a.idx = idx.data_ptr()
    a.k = k
    a.pool = pool.data_ptr() if pool is not None else None
    a.pool_blocks = P
    a.blockmax = blockmax.data_ptr() if blockmax is not None else None
    a.q = q.data_ptr()
    a.swa = swa.data_ptr()
    a.swa_sc = swa_sc.data_ptr()
    a.swa_pos0 = swa_pos0.data_ptr()
    a.T = swa.shape[1]
    a.window = window
    a.replay_start = replay_start.data_ptr() if replay_start is not None else None
    a.sm_scale = sm_scale
    a.out = out.data_ptr()
    a.lse = lse.data_ptr() if lse is not None else None
    a.ws = ws.data_ptr()
    a.ws_bytes = ws.numel()
    _check(lib().csa2_layer_step(ctypes.byref(a), _stream()))
    return out
