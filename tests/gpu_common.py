"""Shared helpers of the GPU parity tests: input builders on both sides of the boundary.

Inputs come from the seeded generator (synth); the CUDA path receives them as
device tensors and the oracle as numpy copies of the same bytes.  Nothing the
CUDA path computes is fed to the oracle.
"""
import math

import numpy as np
import torch

import oracle
import synth

TOL_ABS, TOL_REL = 2e-3, 1e-2   # attention: |gpu - ref| <= 2e-3 + 1e-2 |ref|


def np_(t):
    return t.detach().cpu().numpy()


def bits(t):
    return synth.bf16_bits(t)


def attn_close(gpu_bf16, ref):
    g = gpu_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    ok = err <= TOL_ABS + TOL_REL * np.abs(ref)
    big = np.abs(ref) > 1e-2
    stats = dict(max_abs=float(err.max()) if err.size else 0.0,
                 max_rel=float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0,
                 worst=float((err / (TOL_ABS + TOL_REL * np.abs(ref))).max()) if err.size else 0.0)
    return bool(ok.all()), stats


def ik_untile(codes, scales):
    """Row-major [n, 32] codes and [n, 4] scales from the indexer-K cache order (any
    leading shape with a multiple of 128 entries).  In a 128-entry tile, half h of
    entry e's codes sits at 256 (e // 8 % 16) + 128 h + 16 (e % 8); scales are row-major."""
    c = np.asarray(codes).reshape(-1, 16, 2, 8, 16).transpose(0, 1, 3, 2, 4).reshape(-1, 32)
    return c, np.asarray(scales).reshape(-1, 4)


def ik_tile(codes, scales):
    """Inverse of ik_untile: row-major indexer K -> the cache order (flat bytes)."""
    c = np.ascontiguousarray(np.asarray(codes).reshape(-1, 16, 8, 2, 16).transpose(0, 1, 3, 2, 4)).reshape(-1)
    return c, np.ascontiguousarray(np.asarray(scales)).reshape(-1)


def kv_ik_rows(kv):
    """The device cache's indexer K as row-major numpy [B, cap, 32] / [B, cap, 4]."""
    c, s = ik_untile(np_(kv.ik), np_(kv.ik_sc))
    return c.reshape(kv.B, kv.cap, 32), s.reshape(kv.B, kv.cap, 4)


def set_kv_ik_rows(kv, codes, scales):
    """Write row-major indexer K [B, cap, 32] / [B, cap, 4] into the device cache's tiled order."""
    c, s = ik_tile(codes, scales)
    kv.ik.copy_(torch.from_numpy(c).view(kv.B, kv.cap, 32))
    kv.ik_sc.copy_(torch.from_numpy(s).view(kv.B, kv.cap, 4))


class Group:
    """A CSA2 layer group: bf16 latent rows (generator), the oracle's quantised
    cache (numpy) and the CUDA path's own quantised cache (device)."""

    def __init__(self, seed, B, cap, n_entries, m=1, device="cuda", latent_device=None, rows=None):
        """rows (a multiple of 128, at least every n_entries): only the first rows entries of
        each batch row hold data, the rest of the capacity stays zero on both sides."""
        import sparse_attention_fp4_quant_b200 as csa
        self.B, self.cap, self.m = B, cap, m
        self.rows = cap if rows is None else rows
        assert self.rows % 128 == 0 and self.rows <= cap and max(n_entries) <= self.rows
        latent_device = latent_device or device
        self.latent = torch.stack([synth.latent(synth.seed_of("grp", seed, b), self.rows, 0, latent_device)
                                   for b in range(B)])  # [B, rows, 512] bf16
        self.W = synth.proj_w(seed).to(device)
        self.n_entries = np.array(n_entries, np.int32)
        # CUDA path: its own quantiser and projection write the cache
        self.kv = csa.KV(B, cap, m, device)
        if self.rows == cap:
            lat_dev = self.latent.to(device).reshape(-1, 512)
            csa.csa2_quant_nvfp4(lat_dev, self.kv.lat.view(-1, 256), self.kv.lat_sc.view(-1, 32))
            csa.csa2_index_k_proj(lat_dev, self.W, self.kv.ik.view(-1, 32), self.kv.ik_sc.view(-1, 4))
        else:   # per batch row: the first rows entries (whole 128-entry tiles of the indexer-K image)
            for b in range(B):
                lat_b = self.latent[b].to(device)
                csa.csa2_quant_nvfp4(lat_b, self.kv.lat[b, :self.rows], self.kv.lat_sc[b, :self.rows])
                csa.csa2_index_k_proj(lat_b, self.W, self.kv.ik[b, :self.rows], self.kv.ik_sc[b, :self.rows])
        self.kv.n_entries.copy_(torch.from_numpy(self.n_entries))
        self._oracle = None

    def oracle_cache(self):
        if self._oracle is None:
            lb = bits(self.latent.reshape(-1, 512))
            lat, lat_sc = oracle.quant_nvfp4(lb)
            ik, iks = oracle.index_k_proj(lb, np_(self.W))
            B, cap, rows = self.B, self.cap, self.rows

            def full(a, width):   # [B, rows, width] -> [B, cap, width], zero beyond rows
                out = np.zeros((B, cap, width), a.dtype)
                out[:, :rows] = a.reshape(B, rows, width)
                return out
            self._oracle = dict(lat=full(lat, 256), lat_sc=full(lat_sc, 32), ik=full(ik, 32), iks=full(iks, 4))
        return self._oracle


def index_query(seed, B, Q, device="cuda"):
    """Indexer query: bf16 from the generator, quantised by each side on its own."""
    import sparse_attention_fp4_quant_b200 as csa
    iq_bf = synth.index_q(seed, B, Q, device)
    iq_d, iqs_d = csa.csa2_quant_nvfp4(iq_bf.reshape(-1, 64))
    iq_o, iqs_o = oracle.quant_nvfp4(bits(iq_bf.reshape(-1, 64)))
    w = synth.index_w(B, Q, device)
    return (iq_d.reshape(B, Q, 128), iqs_d.reshape(B, Q, 16), w,
            iq_o.reshape(B, Q, 128), iqs_o.reshape(B, Q, 16), np_(w))


def swa_for(seed, B, T, pos0s, device="cuda"):
    codes, scs = [], []
    for b in range(B):
        c, s = synth.swa_kv(synth.seed_of("swa", seed, b), T, int(pos0s[b]), device)
        codes.append(c)
        scs.append(s)
    return torch.stack(codes), torch.stack(scs)


SM_SCALE = 1.0 / math.sqrt(512)
