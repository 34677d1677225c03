"""Seeded synthetic inputs for the CSA2 hot path.

This module is shared by the tests, the benchmark and the smoke check; it holds
none of the method's arithmetic (no FP4 quantisation, no indexer projection, no
scoring, no selection, no attention).  It only draws the raw inputs that the
method consumes:

* main-KV latents: x ~ N(0, 1) per channel, RMSNorm (eps 1e-6, weight 1), RoPE
  on the last 64 channels (interleaved pairs, base 10000, angle = position *
  10000^(-2k/64)), rounded to bf16.  The FP4 quantisation of these rows is the
  first step of the method and is done by whoever consumes them;
* attention queries (bf16 N(0,1), 16 heads x 512) and indexer queries (bf16
  N(0,1), 4 heads x 64) before quantisation, indexer weights w_h = 0.25 and the
  indexer-K projection matrix (fp32 N(0, 1/512), 512 x 64);
* sliding-window KV in its storage format: the same latent recipe stored as
  FP8 E4M3 with one fp32 scale per token (scale = amax / 448).

Random numbers come from a counter-based generator (splitmix64 of
seed + counter, Box-Muller for normals) written with integer tensor ops, so a
tensor of a given seed and shape can be drawn on any device.  Each input is
drawn once and both the CUDA path and the oracle consume the same bytes.
"""
import hashlib
import math

import torch

D, H, IH, ID = 512, 16, 4, 64
ROPE_DIMS = 64
BASE_SEED = 20261202

_M64 = (1 << 64) - 1


def _s64(u):
    u &= _M64
    return u - (1 << 64) if u >= (1 << 63) else u


_GOLD = _s64(0x9E3779B97F4A7C15)
_MIX1 = _s64(0xBF58476D1CE4E5B9)
_MIX2 = _s64(0x94D049BB133111EB)


def seed_of(*parts):
    """A 63-bit seed from a tuple of names/numbers (stable across runs and machines)."""
    h = hashlib.blake2b(repr((BASE_SEED,) + tuple(parts)).encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 63) - 1)


def _srl(z, k):
    return (z >> k) & ((1 << (64 - k)) - 1)


def _splitmix64(x):
    z = x + _GOLD
    z = (z ^ _srl(z, 30)) * _MIX1
    z = (z ^ _srl(z, 27)) * _MIX2
    return z ^ _srl(z, 31)


def uniform(seed, n, device="cpu", offset=0):
    """n doubles in (0, 1): the top 53 bits of splitmix64(seed + 2 (offset + i) gold) + 1/2 ulp."""
    i = torch.arange(offset, offset + n, dtype=torch.int64, device=device)
    z = _splitmix64(i * _GOLD + _s64(seed))
    return (_srl(z, 11).to(torch.float64) + 0.5) * (2.0 ** -53)


def normal(seed, shape, device="cpu"):
    """Standard normals (float64) of the given shape, by Box-Muller on two counter streams."""
    n = math.prod(shape)
    u1 = uniform(seed, n, device)
    u2 = uniform(seed ^ 0x5DEECE66D, n, device)
    z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)
    return z.reshape(shape)


def _rope_rms(x, pos):
    """RMSNorm (weight 1, eps 1e-6) then RoPE on the last 64 channels; x float64 [n, 512]."""
    x = x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + 1e-6)
    k = torch.arange(ROPE_DIMS // 2, dtype=torch.float64, device=x.device)
    theta = torch.pow(torch.tensor(10000.0, dtype=torch.float64, device=x.device), -2.0 * k / ROPE_DIMS)
    ang = pos.to(torch.float64)[:, None] * theta[None, :]
    c, s = torch.cos(ang), torch.sin(ang)
    r = x[:, D - ROPE_DIMS:]
    ev, od = r[:, 0::2], r[:, 1::2]
    out = x.clone()
    out[:, D - ROPE_DIMS::2] = ev * c - od * s
    out[:, D - ROPE_DIMS + 1::2] = ev * s + od * c
    return out


def latent(seed, n, start_pos=0, device="cpu", chunk=1 << 16):
    """bf16 [n, 512] post-RoPE latents for positions start_pos .. start_pos + n - 1."""
    out = torch.empty((n, D), dtype=torch.bfloat16, device=device)
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        x = normal(seed_of("latent-rows", seed, r0), (r1 - r0, D), device)
        pos = torch.arange(start_pos + r0, start_pos + r1, device=device)
        out[r0:r1] = _rope_rms(x, pos).to(torch.bfloat16)
    return out


def swa_kv(seed, T, pos0, device="cpu"):
    """Sliding-window KV of T tokens at positions pos0 .. pos0+T-1 in its FP8 storage form:
    (E4M3 codes uint8 [T, 512], fp32 scale [T]) with scale = amax / 448 per token."""
    x = latent(seed, T, pos0, device).to(torch.float32)
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    y = (x / scale[:, None]).clamp(-448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def attn_q(seed, B, Q, device="cpu"):
    return normal(seed, (B, Q, H, D), device).to(torch.bfloat16)


def index_q(seed, B, Q, device="cpu"):
    return normal(seed, (B, Q, IH, ID), device).to(torch.bfloat16)


def index_w(B, Q, device="cpu"):
    return torch.full((B, Q, IH), 0.25, dtype=torch.float32, device=device)


def proj_w(seed=0, device="cpu"):
    """Indexer-K projection, fp32 [512, 64] with entries N(0, 1/512)."""
    return (normal(seed_of("index-k-projection", seed), (D, ID), device) / math.sqrt(D)).to(torch.float32)


def bf16_bits(t):
    """uint16 numpy view of a bf16 tensor (the oracle's bf16 input format)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


# Workloads of the pages' shapes (synthetic stand-ins; no dataset is involved).
CONFIGS = {
    "c0": dict(name="full-layer decode, B=1, 4,096 entries, m=1", B=1, n=4096, m=1, Q=1,
               layers=["full"]),
    "c1": dict(name="decode group 1 Full + 3 Reuse, B=32, 131,072 entries, m=1", B=32, n=131072, m=1, Q=1,
               layers=["full", "reuse", "reuse", "reuse"]),
    "c2": dict(name="hierarchical indexer, Full + Reindex, B=8, 1,048,576 entries, m=1", B=8, n=1048576, m=1,
               Q=1, layers=["full", "reindex"]),
    "c3": dict(name="encoder prefill chunk, B=1, m=2, 65,536 tokens -> 32,768 entries, 4,096 queries",
               B=1, n=32768, m=2, Q=4096, tokens=65536, layers=["full"]),
    "c4": dict(name="SWA Bounded Replay + 20-layer decoder step, B=4, 262,144 entries, m=1", B=4, n=262144,
               m=1, Q=1, layers=["full", "reuse", "reuse", "reuse"] + ["reindex", "reuse", "reuse", "reuse"] * 4),
}
TOPK = 512
POOL_BLOCKS = 2048
WINDOW = 128
