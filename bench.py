"""Benchmark of the CSA2 decode hot path on synthetic inputs shaped like the pages' workloads.

Workload (one step): decode of B = 32 queries at 131,072 compressed entries
(m = 1) through one CSA2 group, 1 Full layer + 3 Reuse layers: the Full layer
appends the new token (NVFP4 latent + FP4 indexer K), quantises its indexer
query, scores every entry and keeps the Top-512; all four layers run sparse
attention (Top-512 FP4 rows + their own 128-token FP8 window) with their own
16-head queries.  Inputs are resident in HBM when timing starts; L2 is flushed
(256 MiB write) between timed steps, outside the per-step events.

`python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]`
prints one JSON line (rank 0).  Under torchrun every rank runs its own replica
(weak scaling: the batch is independent per rank; no collective on the data
path) and `value` is N * 32 / (max over ranks of the per-step time).
"""
import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "CSA2 decode queries/s @128K ctx; index+attn HBM GB/s and % of B200 roofline"
B, N_CTX, T_SWA, TOPK, LAYERS = 32, 131072, 128, 512, ["full", "reuse", "reuse", "reuse"]
WORKLOAD = "c1: decode, B=32, 131,072 entries, m=1, 1 Full + 3 Reuse, Top-512, SWA-128"

# algorithmic bytes (each byte the method must move once)
IDX_BYTES_PER_ENTRY = 36                         # 32 B FP4 indexer K + 4 B E4M3 scales
ROW_BYTES = 288                                  # 256 B FP4 latent + 32 B scales
SWA_BYTES = 516                                  # 512 B FP8 + 4 B fp32 scale
Q_OUT_BYTES = 2 * 16 * 512 * 2                   # bf16 query in + bf16 output
IDX_LIST_BYTES = TOPK * 4
ATTN_LAYER_BYTES = B * (TOPK * ROW_BYTES + T_SWA * SWA_BYTES + Q_OUT_BYTES + IDX_LIST_BYTES)


def index_launch_bytes(n_ctx):
    return B * n_ctx * IDX_BYTES_PER_ENTRY + B * (128 + 16 + 16) + B * TOPK * 4


def step_bytes(n_ctx):
    return B * n_ctx * IDX_BYTES_PER_ENTRY + len(LAYERS) * ATTN_LAYER_BYTES


def _peaks():
    """(HBM GB/s, source) from MEASURED_PEAKS.json (a copy test on this machine's B200s), else
    the profiling recipe's fallback measurement."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def _bf16_peak():
    """(dense bf16 TFLOP/s burst, source): the measured cuBLAS figure, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def max_over_ranks(x, device, world):
    """The largest x over all ranks, on every rank (x itself when world == 1).  Every
    rank must call it at the same point."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(world, ms_max):
    """Whole-job queries/s: every rank decodes its own B queries per step (weak scaling),
    and the job's step takes as long as its slowest rank."""
    return world * B / (ms_max / 1000.0)


def _kernel_hash():
    """The index kernel's translation unit: index_cluster.cu and every header it includes."""
    h = hashlib.sha256()
    for f in ("index_cluster.cu", "cluster.cuh", "index_pipe.cuh", "common.cuh", "kernels.h", "host_util.h", "tc.cuh",
              os.path.join("..", "..", "include", "csa2.h")):
        with open(os.path.join(ROOT, "sparse_attention_fp4_quant_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _ncu_traffic():
    """DRAM bytes per launch of the index kernel from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "index_topk_decode_b32_131k.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("kernel_hash") == _kernel_hash():
            return float(d["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        pass
    return None


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this GPU, read through NVML (the source
    nvidia-smi reports from) every ~0.5 ms; only samples taken between mark() and stop() count,
    so they cover the timed region, which lasts a few milliseconds (nvidia-smi's fastest loop,
    200 ms, would see it once at most)."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, device_index):
        self.device_index, self.rows, self.t0, self.handle = device_index, [], None, None
        self.stop_flag = threading.Event()

    def _open(self):
        import pynvml
        pynvml.nvmlInit()
        self.nvml = pynvml
        try:
            pr = torch.cuda.get_device_properties(self.device_index)
            bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:  # noqa: BLE001 - fall back to the CUDA ordinal
            return pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def start(self):
        try:
            self.handle = self._open()
        except Exception:  # noqa: BLE001 - no NVML: the record says so
            self.handle = None
            return
        self.max_mhz = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
        get_reasons = getattr(self.nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nvml.nvmlDeviceGetCurrentClocksThrottleReasons

        def run():
            while not self.stop_flag.is_set():
                t = time.perf_counter()
                mhz = self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
                self.rows.append((t, float(mhz), int(get_reasons(self.handle))))
                time.sleep(0.0005)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def mark(self):
        self.t0 = time.perf_counter()

    def stop(self):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["NVML unavailable"], "samples": 0}
        t1 = time.perf_counter()
        self.stop_flag.set()
        self.thread.join(timeout=2)
        rows = [r for r in self.rows if self.t0 is None or self.t0 <= r[0] <= t1]
        sm = [r[1] for r in rows]
        reasons = sorted({name for r in rows for name, bit in self.REASONS if r[2] & bit})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(rows), "source": "NVML every ~0.5 ms during the timed region"}


# ------------------------------------------------------------------ our arm
class DecodeGroup:
    """Device state and per-step inputs of the config-1 workload on one GPU."""

    def __init__(self, csa, seed, device, n_ctx=N_CTX):
        self.csa = csa
        self.device = device
        self.n_ctx = N_CTX = n_ctx
        self.kv = csa.KV(B, N_CTX, 1, device)
        self.W = synth.proj_w(seed).to(device)
        # context: N_CTX - 1 cached entries; the step appends the new token at N_CTX - 1
        for b in range(B):
            lat = synth.latent(synth.seed_of("bench-ctx", seed, b), N_CTX - 1, 0, device)
            csa.csa2_quant_nvfp4(lat, self.kv.lat[b].view(-1, 256), self.kv.lat_sc[b].view(-1, 32))
            csa.csa2_index_k_proj(lat, self.W, self.kv.ik[b].view(-1, 32), self.kv.ik_sc[b].view(-1, 4))
            del lat
        self.kv.n_entries.fill_(N_CTX)
        # the step's inputs in two contiguous buffers (so the end-to-end step copies them in with two
        # transfers): the new tokens' latents and indexer queries, then every layer's attention query
        self.in_small = torch.empty(B * 512 + B * 256, dtype=torch.bfloat16, device=device)
        self.new_lat = self.in_small[:B * 512].view(B, 512)
        self.new_lat.copy_(torch.stack([synth.latent(synth.seed_of("bench-new", seed, b), 1, N_CTX - 1, device)[0]
                                        for b in range(B)]))
        self.new_rows = (torch.arange(B, device=device, dtype=torch.int64) * N_CTX + (N_CTX - 1))
        self.iq_bf = self.in_small[B * 512:].view(B, 1, 4, 64)
        self.iq_bf.copy_(synth.index_q(synth.seed_of("bench-iq", seed), B, 1, device))
        self.w = synth.index_w(B, 1, device)
        self.q_pos = torch.full((B, 1), N_CTX - 1, dtype=torch.int32, device=device)
        self.q_all = torch.stack([synth.attn_q(synth.seed_of("bench-q", seed, li), B, 1, device)
                                  for li in range(len(LAYERS))])
        self.q = [self.q_all[li] for li in range(len(LAYERS))]
        self.swa = []
        for li in range(len(LAYERS)):
            cs = [synth.swa_kv(synth.seed_of("bench-swa", seed, li, b), T_SWA, N_CTX - T_SWA, device) for b in range(B)]
            self.swa.append((torch.stack([c[0] for c in cs]), torch.stack([c[1] for c in cs])))
        self.swa_pos0 = torch.full((B,), N_CTX - T_SWA, dtype=torch.int32, device=device)
        self.iq = torch.empty((B, 1, 128), dtype=torch.uint8, device=device)
        self.iqs = torch.empty((B, 1, 16), dtype=torch.uint8, device=device)
        self.idx = torch.empty((B, 1, TOPK), dtype=torch.int32, device=device)
        self.out_all = torch.empty((len(LAYERS), B, 1, 16, 512), dtype=torch.bfloat16, device=device)
        self.out = [self.out_all[li] for li in range(len(LAYERS))]
        nbytes = max(csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, B, 1, N_CTX, TOPK),
                     csa.csa2_workspace_bytes(csa.OP_SPARSE_ATTN, B, 1, N_CTX, TOPK))
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.side = torch.cuda.Stream(device=device)
        self.io_in = torch.cuda.Stream(device=device)
        self.io_out = torch.cuda.Stream(device=device)

    # the three segments of a step
    def front(self):
        """Append the new tokens (latent + indexer K, one launch) while, on a second
        branch, the indexer query is quantised (the two are independent)."""
        c = self.csa
        cur = torch.cuda.current_stream()
        self.side.wait_stream(cur)
        with torch.cuda.stream(self.side):
            c.csa2_quant_nvfp4(self.iq_bf.view(-1, 64), self.iq.view(-1, 32), self.iqs.view(-1, 4))
        c.csa2_append_tokens(self.new_lat, self.W, self.kv, self.new_rows)
        cur.wait_stream(self.side)

    def index(self):
        self.csa.csa2_index_topk(self.iq, self.iqs, self.w, self.kv, self.q_pos, TOPK, self.idx, ws=self.ws)

    def attention_layer(self, li):
        swa, swa_sc = self.swa[li]
        self.csa.csa2_sparse_attn(self.q[li], self.kv, self.idx, swa, swa_sc, self.swa_pos0, self.q_pos,
                                  out=self.out[li], ws=self.ws)

    def attention(self):
        for li in range(len(LAYERS)):
            self.attention_layer(li)

    def step(self):
        self.front()
        self.index()
        self.attention()

    def step_with_host_io(self, h_small, h_q_all, h_out_all):
        """One step fed from pinned host buffers and read back to them: the append and
        indexer inputs (48 KB) are copied in first; the four layers' attention queries (2 MB)
        travel as one transfer on a copy stream while the front and the index run (one large
        transfer: each transfer costs ~15 us of set-up on this link); the outputs go back two
        layers at a time, each pair as soon as its second layer is done (a transfer per layer
        queued up behind the attention; one transfer at the end left all 2 MB exposed)."""
        cur = torch.cuda.current_stream()
        self.in_small.copy_(h_small, non_blocking=True)
        self.io_in.wait_stream(cur)
        self.io_out.wait_stream(cur)
        with torch.cuda.stream(self.io_in):   # host -> device, beside the front and the index
            self.q_all.copy_(h_q_all, non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(self.io_in)
        self.front()
        self.index()
        cur.wait_event(ready)
        lo = 0
        for li in range(len(LAYERS)):
            self.attention_layer(li)
            if li % 2 == 1 or li == len(LAYERS) - 1:
                done = torch.cuda.Event()
                done.record(cur)
                with torch.cuda.stream(self.io_out):   # device -> host, the other direction of the link
                    self.io_out.wait_event(done)
                    h_out_all[lo:li + 1].copy_(self.out_all[lo:li + 1], non_blocking=True)
                lo = li + 1
        cur.wait_stream(self.io_in)
        cur.wait_stream(self.io_out)

    LAUNCHES_PER_STEP = 2 + 1 + len(LAYERS)


def _graph(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm (first-call attributes) outside capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _oracle_baseline(seconds_target=12.0, max_reps=64):
    """The oracle (single-threaded C) on a bounded sample of the same workload:
    one batch row at the full 131,072-entry context, the whole step repeated."""
    import oracle
    seed = 9
    lat = synth.latent(synth.seed_of("bench-ctx", seed, 0), N_CTX, 0, "cpu")
    lb = synth.bf16_bits(lat)
    W = synth.proj_w(seed).numpy()
    t0 = time.perf_counter()
    olat, olsc = oracle.quant_nvfp4(lb)
    oik, oiks = oracle.index_k_proj(lb, W)
    setup_s = time.perf_counter() - t0
    olat, olsc = olat.reshape(1, N_CTX, 256), olsc.reshape(1, N_CTX, 32)
    oik, oiks = oik.reshape(1, N_CTX, 32), oiks.reshape(1, N_CTX, 4)
    new_lb = lb[-1:].copy()
    iq = synth.bf16_bits(synth.index_q(synth.seed_of("bench-iq", seed), 1, 1, "cpu")).reshape(-1, 64)
    w = synth.index_w(1, 1).numpy()
    q_pos = np.array([[N_CTX - 1]], np.int32)
    qs = [synth.bf16_bits(synth.attn_q(synth.seed_of("bench-q", seed, li), 1, 1)) for li in range(len(LAYERS))]
    swas = [synth.swa_kv(synth.seed_of("bench-swa", seed, li, 0), T_SWA, N_CTX - T_SWA) for li in range(len(LAYERS))]
    swas = [(c.numpy()[None], s.numpy()[None]) for c, s in swas]
    ne = np.array([N_CTX], np.int32)
    pos0 = np.array([N_CTX - T_SWA], np.int32)

    def step():
        a, b_ = oracle.quant_nvfp4(new_lb)
        olat[0, -1], olsc[0, -1] = a[0], b_[0]
        c_, d_ = oracle.index_k_proj(new_lb, W)
        oik[0, -1], oiks[0, -1] = c_[0], d_[0]
        qc, qsc = oracle.quant_nvfp4(iq)
        idx = oracle.index_topk(qc.reshape(1, 1, 128), qsc.reshape(1, 1, 16), w, oik, oiks, ne, 1, q_pos, TOPK)
        for li in range(len(LAYERS)):
            oracle.sparse_attn(qs[li], olat, olsc, ne, idx, swas[li][0], swas[li][1], pos0, T_SWA, None, q_pos)

    step()
    reps, t0 = 0, time.perf_counter()
    while reps < max_reps and (time.perf_counter() - t0) < seconds_target:
        step()
        reps += 1
    el = time.perf_counter() - t0
    return {"value": reps / el, "unit": "queries/s", "cores": 1, "kind": "oracle",
            "sample": f"1 of the 32 batch rows at the full 131,072-entry context; the whole step (append, "
                      f"indexer-q quantisation, index + Top-512, 4 attention layers) repeated {reps} times in "
                      f"{el:.1f} s (cache setup {setup_s:.1f} s untimed)"}


def run_reference(args, rank, world):
    """Reference arm: the oracle as it stands, on the host cores, rank 0 only."""
    if rank != 0:
        return
    cb = _oracle_baseline(seconds_target=max(3.0, min(20.0, 2.0 * args.steps)))
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "queries/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / cb["value"] * B,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e2m1+f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "l2": "n/a (CPU)"},
            "cpu_baseline": cb, "e2e": {"value": cb["value"], "unit": "queries/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import sparse_attention_fp4_quant_b200 as csa
    device = f"cuda:{local_rank}"
    torch.cuda.set_device(local_rank)
    csa.lib()
    grp = DecodeGroup(csa, seed=9 + rank, device=device, n_ctx=args.ctx)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    g_step = _graph(grp.step)
    g_front, g_index, g_attn = _graph(grp.front), _graph(grp.index), _graph(grp.attention)
    st = torch.cuda.current_stream()
    mk = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]  # noqa: E731

    for _ in range(args.warmup):
        flush.zero_()
        g_step.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.05)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    all_ev = []
    sampler.mark()
    t_wall = time.perf_counter()
    for _ in range(args.steps):
        flush.zero_()
        evs = mk(2)
        evs[0].record(st)
        g_step.replay()
        evs[1].record(st)
        all_ev.append(evs)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    wall_s = time.perf_counter() - t_wall
    clocks = sampler.stop()
    step_ms = [e[0].elapsed_time(e[1]) for e in all_ev]
    ms_max = max_over_ranks(float(np.mean(step_ms)), device, world)

    # breakdown (not the headline): the same step as three graphs with events between them
    seg_ev = []
    for it in range(args.warmup + args.steps):
        flush.zero_()
        evs = mk(4)
        evs[0].record(st)
        g_front.replay()
        evs[1].record(st)
        g_index.replay()
        evs[2].record(st)
        g_attn.replay()
        evs[3].record(st)
        if it >= args.warmup:
            seg_ev.append(evs)
    torch.cuda.synchronize()
    index_ms = [e[1].elapsed_time(e[2]) for e in seg_ev]
    attn_ms = [e[2].elapsed_time(e[3]) for e in seg_ev]
    front_ms = [e[0].elapsed_time(e[1]) for e in seg_ev]

    # end to end through the public API with host buffers: every step copies its inputs in
    # from pinned host memory and its four outputs back (one graph holding the copies, the
    # queries' and outputs' transfers overlapped with compute on a copy stream)
    h_small = grp.in_small.cpu().pin_memory()
    h_q_all = grp.q_all.cpu().pin_memory()
    h_out_all = torch.zeros(grp.out_all.shape, dtype=grp.out_all.dtype).pin_memory()
    h_out = [h_out_all[li] for li in range(len(LAYERS))]
    h2d = h_small.numel() * 2 + h_q_all.numel() * 2
    d2h = h_out_all.numel() * 2
    g_e2e = _graph(lambda: grp.step_with_host_io(h_small, h_q_all, h_out_all))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = []
    for it in range(args.warmup + args.steps):
        flush.zero_()
        for ho in h_out:
            ho.zero_()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        e0.record(st)
        g_e2e.replay()
        e1.record(st)
        e1.synchronize()
        if it >= args.warmup:
            e2e_ms.append(max(e0.elapsed_time(e1), (time.perf_counter() - t0) * 1000.0))
    for o, ho in zip(grp.out, h_out):   # the copies really delivered the step's outputs
        if not torch.equal(o.cpu(), ho):
            raise RuntimeError("end-to-end step: host outputs differ from the device outputs")
    e2e_max = max_over_ranks(float(np.mean(e2e_ms)), device, world)

    configs = None
    if world == 1 and not args.no_configs and args.ctx == N_CTX:
        del g_step, g_front, g_index, g_attn, g_e2e
        torch.cuda.empty_cache()
        configs = other_configs(csa, args, flush)
    if rank != 0:
        return
    peak, peak_kind = _peaks()
    idx_s = float(np.mean(index_ms)) / 1000.0
    achieved = index_launch_bytes(args.ctx) / idx_s / 1e9
    traffic = _ncu_traffic() if args.ctx == N_CTX else None
    cb = _oracle_baseline() if (world == 1 and not args.no_cpu_baseline and args.ctx == N_CTX) else None
    value = job_value(world, ms_max)
    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1+bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD if args.ctx == N_CTX else WORKLOAD.replace("131,072", f"{args.ctx:,}"),
                   "B_per_gpu": B, "ctx_entries": args.ctx, "topk": TOPK, "swa": T_SWA,
                   "l2": "flushed between timed steps (256 MiB write outside the step events)",
                   "graphs": "one CUDA graph per step (front with two branches, index, 4 attention layers)"},
        "index_attn_gbs": step_bytes(args.ctx) / (ms_max / 1000.0) / 1e9,
        "index_attn_frac_of_hbm": step_bytes(args.ctx) / (ms_max / 1000.0) / 1e9 / peak,
        "step_algorithmic_bytes": step_bytes(args.ctx),
        "segments_ms": {"front": float(np.mean(front_ms)), "index_topk": float(np.mean(index_ms)),
                        "attention_x4": float(np.mean(attn_ms)),
                        "how": "the step re-run as three graphs with events between them (diagnostic)"},
        "roofline": {"kernel": "csa2_index_topk (index_cluster_kernel)", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} copy bandwidth" + (" (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                                                                      else " (no MEASURED_PEAKS.json: 6.65 TB/s)"),
                     "bytes_per_launch": index_launch_bytes(args.ctx)},
        "cpu_baseline": cb,
        "e2e": {"value": job_value(world, e2e_max), "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_max},
        "gpu_launches": DecodeGroup.LAUNCHES_PER_STEP * args.steps,
        "clocks": clocks,
        "wall_s_timed_region": wall_s,
    }
    if configs is not None:
        line["configs"] = configs
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the other four workloads
DECODER_PATTERN = ["full", "reuse", "reuse", "reuse"] + ["reindex", "reuse", "reuse", "reuse"] * 4
N_POOL = 2048


def _timed_graph(g, steps, warmup, flush, st):
    """Per-step milliseconds of a graph (CUDA events on the launching stream, L2 flushed
    before every step outside the events)."""
    ms = []
    for it in range(warmup + steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        g.replay()
        e1.record(st)
        if it >= warmup:
            ms.append((e0, e1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ms]


class LayerStack:
    """One CSA2 layer group driven layer by layer through the public API (csa2_layer_step
    does the Full / Reindex / Reuse dispatch): B batch rows with Q queries each at token
    positions q_pos, n_cached entries in the cache.  With `append`, the Full layer first
    appends one new token per batch row (a decode step); with `replay`, attention uses the
    Bounded Replay mask from the first query's position (the decoder replay of the last
    Q tokens).  Every layer has its own attention query and FP8 window KV; Full and
    Reindex layers have their own indexer query, quantised in the step."""

    def __init__(self, csa, tag, device, B, cap, n_cached, q_pos, pattern, append, pool, replay=False):
        self.csa, self.B, self.cap, self.pattern, self.append = csa, B, cap, pattern, append
        self.Q = q_pos.shape[1]
        Q = self.Q
        self.kv = csa.KV(B, cap, 1, device)
        self.W = synth.proj_w(synth.seed_of(tag, "W")).to(device)
        for b in range(B):
            lat = synth.latent(synth.seed_of(tag, "ctx", b), n_cached, 0, device)
            csa.csa2_quant_nvfp4(lat, self.kv.lat[b].view(-1, 256), self.kv.lat_sc[b].view(-1, 32))
            csa.csa2_index_k_proj(lat, self.W, self.kv.ik[b].view(-1, 32), self.kv.ik_sc[b].view(-1, 4))
            del lat
        self.kv.n_entries.fill_(n_cached + (1 if append else 0))
        self.new_lat = torch.stack([synth.latent(synth.seed_of(tag, "new", b), 1, n_cached, device)[0]
                                    for b in range(B)])
        self.new_rows = torch.arange(B, device=device, dtype=torch.int64) * cap + n_cached
        self.q_pos = q_pos.to(device)
        first = int(q_pos[0, 0])
        last = int(q_pos[0, -1])
        self.swa_pos0 = torch.full((B,), (first if replay else last - T_SWA + 1), dtype=torch.int32, device=device)
        T = (last - first + 1) if replay else T_SWA
        self.replay_start = self.swa_pos0.clone() if replay else None
        self.q, self.swa, self.iq_bf, self.iq, self.iqs = [], [], {}, {}, {}
        for li, mode in enumerate(pattern):
            self.q.append(synth.attn_q(synth.seed_of(tag, "q", li), B, Q, device))
            cs = [synth.swa_kv(synth.seed_of(tag, "swa", li, b), T, int(self.swa_pos0[b]), device) for b in range(B)]
            self.swa.append((torch.stack([c[0] for c in cs]), torch.stack([c[1] for c in cs])))
            if mode != "reuse":
                self.iq_bf[li] = synth.index_q(synth.seed_of(tag, "iq", li), B, Q, device)
                self.iq[li] = torch.empty((B, Q, 128), dtype=torch.uint8, device=device)
                self.iqs[li] = torch.empty((B, Q, 16), dtype=torch.uint8, device=device)
        self.w = synth.index_w(B, Q, device)
        self.idx = torch.empty((B, Q, TOPK), dtype=torch.int32, device=device)
        self.pool = torch.empty((B, Q, N_POOL), dtype=torch.int32, device=device) if pool else None
        self.bm = torch.empty((B, Q, (cap + 7) // 8), dtype=torch.float32, device=device) if pool else None
        self.out = [torch.empty((B, Q, 16, 512), dtype=torch.bfloat16, device=device) for _ in pattern]
        self.ws = torch.zeros(csa.csa2_workspace_bytes(csa.OP_LAYER, B, Q, cap, TOPK, N_POOL), dtype=torch.uint8,
                              device=device)

    def layer(self, li):
        c, mode = self.csa, self.pattern[li]
        if mode != "reuse":
            c.csa2_quant_nvfp4(self.iq_bf[li].view(-1, 64), self.iq[li].view(-1, 32), self.iqs[li].view(-1, 4))
        app = self.append and li == 0
        swa, swa_sc = self.swa[li]
        c.csa2_layer_step(mode, self.kv, self.q_pos, self.q[li], swa, swa_sc, self.swa_pos0, self.idx, TOPK,
                          self.iq.get(li), self.iqs.get(li), self.w if mode != "reuse" else None,
                          pool=self.pool, blockmax=self.bm, new_latent=self.new_lat if app else None,
                          new_rows=self.new_rows if app else None, k_proj=self.W, replay_start=self.replay_start,
                          out=self.out[li], ws=self.ws)

    def step(self):
        for li in range(len(self.pattern)):
            self.layer(li)

    def index_only(self):
        """The Full layer's index call alone (for its roofline)."""
        self.csa.csa2_index_topk(self.iq[0], self.iqs[0], self.w, self.kv, self.q_pos, TOPK, self.idx,
                                 blockmax=self.bm if self.bm is not None else False, ws=self.ws)

    def launches(self):
        # the many-query index (more than 148 queries, at least 8 per batch row, at most 262,144
        # entries) is two kernels, scoring then selection; the other index paths are one
        mq = self.B * self.Q > 148 and self.Q >= 8 and self.cap <= 262144
        n = 1 if self.append else 0
        for mode in self.pattern:
            n += {"full": (4 if mq else 3) + (1 if self.pool is not None else 0), "reindex": 3, "reuse": 1}[mode]
        return n


def _attn_bytes(nq, k=TOPK, T=T_SWA):
    return nq * (k * ROW_BYTES + T * SWA_BYTES + Q_OUT_BYTES + k * 4)


def _oracle_stack(tag, b, n_cached, q_pos_row, pattern, append, pool, pos0, T, replay, cap, max_reps, seconds, sample):
    """The oracle on batch row b of a LayerStack workload (the same generator seeds; the
    queries are the row's first len(q_pos_row) draws): set-up (latents drawn on the GPU by
    the generator when one is present, the oracle's own indexer-K projection) untimed, then
    the step repeated.  Returns a cpu_baseline dict."""
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t0 = time.perf_counter()
    W = synth.proj_w(synth.seed_of(tag, "W")).numpy()
    lat = synth.bf16_bits(synth.latent(synth.seed_of(tag, "ctx", b), n_cached, 0, dev).cpu())
    ik = np.zeros((1, cap, 32), np.uint8)
    iks = np.zeros((1, cap, 4), np.uint8)
    ik[0, :n_cached], iks[0, :n_cached] = oracle.index_k_proj(lat, W)
    olat = np.zeros((1, cap, 256), np.uint8)   # filled lazily: only rows attention reads
    olsc = np.zeros((1, cap, 32), np.uint8)
    done = np.zeros(cap, bool)
    new = synth.bf16_bits(synth.latent(synth.seed_of(tag, "new", b), 1, n_cached, "cpu"))
    Q = len(q_pos_row)
    q_pos = np.array([q_pos_row], np.int32)
    rs = np.array([pos0], np.int32) if replay else None
    layers = []
    for li, mode in enumerate(pattern):
        qb = synth.bf16_bits(synth.attn_q(synth.seed_of(tag, "q", li), b + 1, Q))[b:b + 1]
        c, sc = synth.swa_kv(synth.seed_of(tag, "swa", li, b), T, pos0)
        iqb = None
        if mode != "reuse":
            iqb = synth.bf16_bits(synth.index_q(synth.seed_of(tag, "iq", li), b + 1, Q))[b:b + 1].reshape(-1, 64)
        layers.append((mode, qb, c.numpy()[None], sc.numpy()[None], iqb))
    setup = time.perf_counter() - t0
    ne = np.array([n_cached + (1 if append else 0)], np.int32)
    w = synth.index_w(1, Q).numpy()

    def step():
        if append:
            a, s_ = oracle.quant_nvfp4(new)
            olat[0, n_cached], olsc[0, n_cached] = a[0], s_[0]
            c_, d_ = oracle.index_k_proj(new, W)
            ik[0, n_cached], iks[0, n_cached] = c_[0], d_[0]
            done[n_cached] = True
        idx = pl = None
        for mode, qb, swa, swa_sc, iqb in layers:
            if mode != "reuse":
                qc, qsc = oracle.quant_nvfp4(iqb)
                qc, qsc = qc.reshape(1, Q, 128), qsc.reshape(1, Q, 16)
            if mode == "full":
                idx, bm = oracle.index_topk(qc, qsc, w, ik, iks, ne, 1, q_pos, TOPK, blockmax=True)
                if pool:
                    pl = oracle.pool_build(bm, ne, 1, q_pos, N_POOL)
            elif mode == "reindex":
                idx = oracle.pool_topk(qc, qsc, w, ik, iks, ne, 1, pl, q_pos, TOPK)
            need = np.unique(idx[idx >= 0])
            need = need[~done[need]]
            if need.size:   # the oracle quantises the main rows attention reads
                a, s_ = oracle.quant_nvfp4(lat[need])
                olat[0, need], olsc[0, need] = a, s_
                done[need] = True
            oracle.sparse_attn(qb, olat, olsc, ne, idx, swa, swa_sc, np.array([pos0], np.int32), T_SWA, rs, q_pos)

    reps, t0 = 0, time.perf_counter()
    while reps < max_reps and (reps == 0 or (time.perf_counter() - t0) < seconds):
        step()
        reps += 1
    el = time.perf_counter() - t0
    return {"value": reps * Q / el, "unit": "queries/s", "cores": 1, "kind": "oracle",
            "sample": f"{sample}; repeated {reps} times in {el:.1f} s (set-up {setup:.1f} s untimed)"}


def _stack_config(csa, name, workload, tag, B, cap, n_cached, q_pos, pattern, append, pool, replay, steps, warmup,
                  flush, bytes_alg, roof_bytes=None, roof_flop=None, cpu=None):
    """Time one LayerStack workload: the whole step as one CUDA graph, and its Full-layer
    index call alone (the roofline kernel)."""
    st = torch.cuda.current_stream()
    stk = LayerStack(csa, tag, "cuda", B, cap, n_cached, q_pos, pattern, append, pool, replay)
    g = _graph(stk.step)
    ms = _timed_graph(g, steps, warmup, flush, st)
    gi = _graph(stk.index_only)
    ims = _timed_graph(gi, steps, warmup, flush, st)
    step_ms, idx_ms = float(np.mean(ms)), float(np.mean(ims))
    nq = B * q_pos.shape[1]
    rec = {"workload": workload, "ms_per_step": step_ms, "value": nq / (step_ms * 1e-3), "unit": "queries/s",
           "algorithmic_bytes": bytes_alg, "achieved_gbs": bytes_alg / (step_ms * 1e-3) / 1e9,
           "index_ms": idx_ms, "gpu_launches_per_step": stk.launches()}
    if roof_bytes is not None:
        peak, kind = _peaks()
        ach = roof_bytes / (idx_ms * 1e-3) / 1e9
        rec["roofline"] = {"kernel": "csa2_index_topk (Full layer)", "bound": "hbm", "achieved": ach, "peak": peak,
                           "unit": "GB/s", "frac": ach / peak, "peak_source": f"{kind} copy bandwidth",
                           "bytes_per_launch": roof_bytes}
        rec["frac_of_hbm_whole_step"] = rec["achieved_gbs"] / peak
    if roof_flop is not None:
        bf16, kind = _bf16_peak()
        ach = roof_flop / (idx_ms * 1e-3) / 1e12
        rec["roofline"] = {"kernel": "csa2_index_topk (Full layer)", "bound": "tensor", "achieved": ach,
                           "peak": 4 * bf16, "unit": "TFLOP/s", "frac": ach / (4 * bf16),
                           "peak_source": f"{kind} bf16 GEMM burst x 4 (nominal FP4/BF16 ratio)",
                           "flop_per_launch": roof_flop}
    del stk, g, gi
    torch.cuda.empty_cache()
    if cpu is not None:
        rec["cpu_baseline"] = cpu()
    return rec


def measure_c0(csa, steps, warmup, flush, with_cpu):
    n = 4096
    q_pos = torch.full((1, 1), n - 1, dtype=torch.int32)
    cpu = (lambda: _oracle_stack("c0", 0, n - 1, [n - 1], ["full"], True, False, n - T_SWA, T_SWA, False, n, 200, 4.0,
                                 "the whole step (append, index over 4,096 entries, one attention layer)")) \
        if with_cpu else None
    rec = _stack_config(csa, "c0", "c0: decode, B=1, 4,096 entries, m=1, one Full layer", "c0", 1, n, n - 1, q_pos,
                        ["full"], True, False, False, steps, warmup, flush,
                        n * IDX_BYTES_PER_ENTRY + _attn_bytes(1), cpu=cpu)
    rec["bound"] = "latency: about 0.4 MB of algorithmic bytes per step"
    return rec


def measure_c2(csa, steps, warmup, flush, with_cpu):
    Bc, n = 8, 1 << 20
    q_pos = torch.full((Bc, 1), n - 1, dtype=torch.int32)
    idx_bytes = Bc * n * IDX_BYTES_PER_ENTRY
    bytes_alg = idx_bytes + Bc * N_POOL * 8 * IDX_BYTES_PER_ENTRY + 2 * _attn_bytes(Bc)
    cpu = (lambda: _oracle_stack("c2", 0, n - 1, [n - 1], ["full", "reindex"], True, True, n - T_SWA, T_SWA, False, n,
                                 1, 0.0,
                                 "1 of the 8 batch rows, one step: append, index over 1,048,576 entries with "
                                 "block maxima, pool build, Reindex in the pool, two attention layers")) \
        if with_cpu else None
    return _stack_config(csa, "c2", "c2: hierarchical indexer, decode, B=8, 1,048,576 entries, m=1, Full (index, "
                         "Top-512, pool of 2,048 x 8) + Reindex (Top-512 in the pool), each with attention + SWA-128",
                         "c2", Bc, n, n - 1, q_pos, ["full", "reindex"], True, True, False, steps, warmup, flush,
                         bytes_alg, roof_bytes=idx_bytes, cpu=cpu)


def measure_c4(csa, steps, warmup, flush, with_cpu):
    Bc, n = 4, 1 << 18
    n_cached = n - 1
    # replay: the last 128 cached tokens through the 20 layers, mask start s = their first position
    s0 = n_cached - 128
    rq = torch.arange(s0, n_cached, dtype=torch.int32).view(1, -1).repeat(Bc, 1)
    nv = np.arange(s0, n_cached, dtype=np.int64) + 1
    replay_flop = float(Bc * nv.sum()) * 4 * 64 * 2
    cpu_r = (lambda: _oracle_stack("c4r", 0, n_cached, [s0, s0 + 64], DECODER_PATTERN, False, True, s0, 128, True, n,
                                   1, 0.0,
                                   "2 of the 512 replay queries (positions s and s + 64 of batch row 0) through the "
                                   "20 layers")) if with_cpu else None
    rep = _stack_config(csa, "c4_replay", "c4 replay: B=4, 262,143 cached entries, the last 128 tokens replayed "
                        "(mask start s = ctx - 128) through the 20-layer decoder pattern, fresh FP8 SWA per layer",
                        "c4r", Bc, n, n_cached, rq, DECODER_PATTERN, False, True, True, max(2, steps // 4), warmup,
                        flush, Bc * n_cached * IDX_BYTES_PER_ENTRY, roof_flop=replay_flop, cpu=cpu_r)
    dq = torch.full((Bc, 1), n_cached, dtype=torch.int32)
    dec_bytes = Bc * n * IDX_BYTES_PER_ENTRY + 4 * Bc * N_POOL * 8 * IDX_BYTES_PER_ENTRY + 20 * _attn_bytes(Bc)
    cpu_d = (lambda: _oracle_stack("c4d", 0, n_cached, [n_cached], DECODER_PATTERN, True, True, n - T_SWA, T_SWA, False,
                                   n, 2, 3.0,
                                   "1 of the 4 batch rows, the whole decode step (append, 20 layers)")) \
        if with_cpu else None
    dec = _stack_config(csa, "c4_decode", "c4 decode step: B=4, 262,144 entries, append + 20 layers "
                        "(1 Full + 3 Reuse, then 4 x (1 Reindex + 3 Reuse))", "c4d", Bc, n, n_cached, dq,
                        DECODER_PATTERN, True, True, False, steps, warmup, flush, dec_bytes,
                        roof_bytes=Bc * n * IDX_BYTES_PER_ENTRY, cpu=cpu_d)
    return {"replay": rep, "decode_step": dec}


def _rope_tables(pos):
    k = np.arange(32, dtype=np.float64)
    ang = np.asarray(pos, np.float64).reshape(-1, 1) * 10000.0 ** (-2.0 * k / 64.0)
    return (torch.from_numpy(np.cos(ang).astype(np.float32)), torch.from_numpy(np.sin(ang).astype(np.float32)))


def measure_front_end(csa, steps, warmup, flush, with_cpu):
    """The fused front end (RMSNorm + RoPE + bf16 + NVFP4 + indexer-K projection) for the 32 new
    tokens of a decode step and for the 32,768 entries of a prefill chunk's cache.  Bound: the
    fp32 fused multiply-add chains (about 33,300 per row) on the CUDA cores."""
    out = {}
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    peak_fma = sms * 128 * 1.965e9   # fp32 FMA lanes x the B200's maximum SM clock
    for name, rows in (("decode_32_rows", 32), ("prefill_32768_rows", 32768)):
        x = (synth.normal(synth.seed_of("bench-front", rows), (rows, 512), "cuda") * 1.7).to(torch.bfloat16)
        cos, sin = _rope_tables(np.arange(rows) * 3 + 5)
        cos, sin = cos.cuda(), sin.cuda()
        W = synth.proj_w(3).cuda()
        cap = (rows + 127) // 128 * 128
        outs = tuple(torch.zeros((cap, n), dtype=torch.uint8, device="cuda") for n in (256, 32, 32, 4))
        g = _graph(lambda: csa.csa2_front_end(x, cos, sin, W, outs))
        ms = float(np.mean(_timed_graph(g, steps, warmup, flush, torch.cuda.current_stream())))
        fma = rows * (512 + 512 * 64)
        bytes_ = rows * (1024 + 256 + 288 + 36)
        out[name] = {"rows": rows, "ms": ms, "rows_per_s": rows / (ms * 1e-3),
                     "achieved_gbs": bytes_ / (ms * 1e-3) / 1e9,
                     "roofline": {"bound": "alu", "achieved": fma / (ms * 1e-3) / 1e12, "peak": peak_fma / 1e12,
                                  "unit": "T FMA/s", "frac": fma / (ms * 1e-3) / peak_fma,
                                  "peak_source": f"{sms} SMs x 128 fp32 FMA lanes x 1.965 GHz (max SM clock)"}}
        del g, outs, x
    if with_cpu:
        import oracle
        rows = 256
        x = synth.bf16_bits((synth.normal(synth.seed_of("bench-front", rows), (rows, 512)) * 1.7).to(torch.bfloat16))
        cos, sin = _rope_tables(np.arange(rows) * 3 + 5)
        W = synth.proj_w(3).numpy()
        t0 = time.perf_counter()
        y = oracle.front_end(x, cos.numpy(), sin.numpy())
        oracle.quant_nvfp4(y)
        oracle.index_k_proj(y, W)
        el = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": rows / el, "unit": "rows/s", "cores": 1, "kind": "oracle",
                               "sample": f"{rows} rows through the oracle's front end, quantiser and projection "
                                         f"in {el:.2f} s"}
    torch.cuda.empty_cache()
    return out


def measure_encoder_prefill(csa, steps, warmup, flush, with_cpu):
    """The encoder side at m = 2: a 65,536-token prompt as 16 chunks of 4,096 queries through
    3 groups of (1 Full + 5 Reuse) via csa2_layer_step; each Full layer appends the chunk's
    2,048 compressed entries to its group's cache first.  Per-layer queries and windows are
    drawn once and reused by every chunk (timing only)."""
    tokens, chunk, groups = 65536, 4096, 3
    n = tokens // 2
    dev = "cuda"
    kvs = [csa.KV(1, n, 2, dev) for _ in range(groups)]
    Ws = [synth.proj_w(synth.seed_of("bench-enc-W", g)).to(dev) for g in range(groups)]
    lats = [synth.latent(synth.seed_of("bench-enc", g), n, 0, dev) for g in range(groups)]
    pattern = (["full"] + ["reuse"] * 5) * groups
    qs = [synth.attn_q(synth.seed_of("bench-enc-q", li), 1, chunk, dev) for li in range(len(pattern))]
    T = chunk + 127
    swas = []
    for li in range(len(pattern)):
        c, sc = synth.swa_kv(synth.seed_of("bench-enc-swa", li), T, 0, dev)
        swas.append((c.unsqueeze(0), sc.unsqueeze(0)))
    iqs = []
    for g in range(groups):
        iq, iqsc = csa.csa2_quant_nvfp4(synth.index_q(synth.seed_of("bench-enc-iq", g), 1, chunk, dev).view(-1, 64))
        iqs.append((iq.view(1, chunk, 128), iqsc.view(1, chunk, 16)))
    w = synth.index_w(1, chunk, dev)
    idx = torch.empty((1, chunk, TOPK), dtype=torch.int32, device=dev)
    outb = torch.empty((1, chunk, 16, 512), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(csa.csa2_workspace_bytes(csa.OP_LAYER, 1, chunk, n, TOPK, N_POOL), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    pos = [torch.from_numpy((c * chunk + np.arange(chunk)).astype(np.int32).reshape(1, -1)).to(dev)
           for c in range(tokens // chunk)]
    rows = [torch.arange(c * chunk // 2, (c + 1) * chunk // 2, dtype=torch.int64, device=dev)
            for c in range(tokens // chunk)]

    def prefill(events=None):
        for c in range(tokens // chunk):
            p0 = torch.full((1,), max(0, c * chunk - 127), dtype=torch.int32, device=dev)
            if events is not None:
                events[c][0].record(st)
            for li, mode in enumerate(pattern):
                g = li // 6
                swa, swa_sc = swas[li]
                if mode == "full":
                    kvs[g].n_entries.fill_((c + 1) * chunk // 2)
                    csa.csa2_layer_step("full", kvs[g], pos[c], qs[li], swa, swa_sc, p0, idx, TOPK, iqs[g][0],
                                        iqs[g][1], w, new_latent=lats[g][c * chunk // 2:(c + 1) * chunk // 2],
                                        new_rows=rows[c], k_proj=Ws[g], out=outb, ws=ws)
                else:
                    csa.csa2_layer_step("reuse", kvs[g], pos[c], qs[li], swa, swa_sc, p0, idx, TOPK, out=outb, ws=ws)
            if events is not None:
                events[c][1].record(st)

    for _ in range(max(1, warmup // 3)):
        prefill()
    reps = max(1, steps // 5)
    per_chunk = np.zeros(tokens // chunk)
    total = []
    for _ in range(reps):
        flush.zero_()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(tokens // chunk)]
        prefill(evs)
        torch.cuda.synchronize()
        ms = np.array([a.elapsed_time(b) for a, b in evs])
        per_chunk += ms / reps
        total.append(evs[0][0].elapsed_time(evs[-1][1]))
    del kvs, lats, qs, swas, ws
    torch.cuda.empty_cache()
    return {"workload": "f1: encoder prefill, 65,536 tokens at m=2 in 16 chunks of 4,096 queries, 3 groups of "
                        "(1 Full + 5 Reuse), Top-512, SWA-128",
            "ms_per_prompt": float(np.mean(total)), "tokens_per_s": tokens / (float(np.mean(total)) * 1e-3),
            "ms_per_chunk": [round(float(v), 3) for v in per_chunk],
            "gpu_launches_per_chunk": groups * (4 + 5),
            "note": "launched call by call from Python (no graph); per-chunk times from CUDA events"}


def _prefill_cpu_sample(n, Q, tokens, T, pos0, n_sample=12):
    """The oracle on n_sample of the chunk's 4,096 queries (spread over the chunk): index +
    Top-512 over their causally visible entries (m = 2) and one attention layer."""
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t0 = time.perf_counter()
    lat = synth.bf16_bits(synth.latent(synth.seed_of("prefill-ctx", 0), n, 0, dev).cpu())
    W = synth.proj_w(130).numpy()
    ik, iks = oracle.index_k_proj(lat, W)
    ik, iks = ik.reshape(1, n, 32), iks.reshape(1, n, 4)
    olat, olsc = oracle.quant_nvfp4(lat)
    olat, olsc = olat.reshape(1, n, 256), olsc.reshape(1, n, 32)
    sel = np.linspace(0, Q - 1, n_sample).astype(np.int64)
    iqb = synth.bf16_bits(synth.index_q(synth.seed_of("prefill-iq"), 1, Q, dev).cpu())[0, sel].reshape(-1, 64)
    qb = synth.bf16_bits(synth.attn_q(synth.seed_of("prefill-q"), 1, Q, dev).cpu())[:, sel]
    c, sc = synth.swa_kv(synth.seed_of("prefill-swa"), T, pos0, dev)
    swa, swa_sc = c.cpu().numpy()[None], sc.cpu().numpy()[None]
    q_pos = (sel + (tokens - Q)).astype(np.int32).reshape(1, -1)
    w = synth.index_w(1, n_sample).numpy()
    setup = time.perf_counter() - t0
    ne = np.array([n], np.int32)
    t0 = time.perf_counter()
    qc, qsc = oracle.quant_nvfp4(iqb)
    idx = oracle.index_topk(qc.reshape(1, -1, 128), qsc.reshape(1, -1, 16), w, ik, iks, ne, 2, q_pos, TOPK)
    oracle.sparse_attn(qb, olat, olsc, ne, idx, swa, swa_sc, np.array([pos0], np.int32), T_SWA, None, q_pos)
    el = time.perf_counter() - t0
    return {"value": n_sample / el, "unit": "queries/s", "cores": 1, "kind": "oracle",
            "sample": f"{n_sample} of the 4,096 queries spread over the chunk: index + Top-512 over their visible "
                      f"entries and one attention layer, in {el:.1f} s (set-up {setup:.1f} s untimed)"}


def measure_c3(csa, steps, warmup, flush, with_cpu):
    """The prefill chunk (one GPU): 65,536-token prompt compressed 2:1 into 32,768 entries,
    4,096 queries at its end; index + Top-512 and one attention layer (main + SWA-128),
    each timed with CUDA events over K steps, L2 flushed between steps."""
    device = "cuda"
    Bp, n, Q, tokens, T = 1, 32768, 4096, 65536, 4096 + T_SWA - 1
    kv = csa.KV(Bp, n, 2, device)
    W = synth.proj_w(130).to(device)
    lat = synth.latent(synth.seed_of("prefill-ctx", 0), n, 0, device)
    csa.csa2_quant_nvfp4(lat, kv.lat.view(-1, 256), kv.lat_sc.view(-1, 32))
    csa.csa2_index_k_proj(lat, W, kv.ik.view(-1, 32), kv.ik_sc.view(-1, 4))
    del lat
    kv.n_entries.fill_(n)
    iq, iqs = csa.csa2_quant_nvfp4(synth.index_q(synth.seed_of("prefill-iq"), Bp, Q, device).view(-1, 64))
    iq, iqs = iq.view(Bp, Q, 128), iqs.view(Bp, Q, 16)
    w = synth.index_w(Bp, Q, device)
    q_pos = (torch.arange(Q, device=device, dtype=torch.int32) + (tokens - Q)).view(Bp, Q)
    q = synth.attn_q(synth.seed_of("prefill-q"), Bp, Q, device)
    pos0 = tokens - T
    swa, swa_sc = synth.swa_kv(synth.seed_of("prefill-swa"), T, pos0, device)
    swa, swa_sc = swa.unsqueeze(0), swa_sc.unsqueeze(0)
    pos0_t = torch.tensor([pos0], dtype=torch.int32, device=device)
    idx = torch.empty((Bp, Q, TOPK), dtype=torch.int32, device=device)
    out = torch.empty((Bp, Q, 16, 512), dtype=torch.bfloat16, device=device)
    ws = torch.zeros(max(csa.csa2_workspace_bytes(csa.OP_INDEX_TOPK, Bp, Q, n, TOPK),
                         csa.csa2_workspace_bytes(csa.OP_SPARSE_ATTN, Bp, Q, n, TOPK)), dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream()
    t_idx, t_att = [], []
    for it in range(warmup + steps):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(st)
        csa.csa2_index_topk(iq, iqs, w, kv, q_pos, TOPK, idx, ws=ws)
        ev[1].record(st)
        csa.csa2_sparse_attn(q, kv, idx, swa, swa_sc, pos0_t, q_pos, out=out, ws=ws)
        ev[2].record(st)
        torch.cuda.synchronize()
        if it >= warmup:
            t_idx.append(ev[0].elapsed_time(ev[1]))
            t_att.append(ev[1].elapsed_time(ev[2]))
    idx_ms, att_ms = float(np.mean(t_idx)), float(np.mean(t_att))
    nvis = np.minimum((q_pos.cpu().numpy().astype(np.int64) + 1) // 2, n)
    idx_flop = float(nvis.sum()) * 4 * 64 * 2           # dense-equivalent indexer Q.K^T
    att_flop = float(Q) * 16 * (TOPK + T_SWA) * 512 * 4  # S and P V over every slot
    bf16, bf16_kind = _bf16_peak()
    fp4_peak = bf16 * 4.0   # nominal dense FP4 / BF16 ratio (9 / 2.25 PFLOP/s)
    achieved = idx_flop / (idx_ms * 1e-3) / 1e12
    del kv, ws, out, idx
    torch.cuda.empty_cache()
    rec = {
        "workload": "c3: prefill chunk, 65,536-token prompt, m=2 (32,768 entries), 4,096 queries, Top-512, SWA-128",
        "ms_per_step": idx_ms + att_ms, "value": Q / ((idx_ms + att_ms) * 1e-3), "unit": "queries/s",
        "index_ms": idx_ms, "attention_ms": att_ms, "gpu_launches_per_step": 3,
        "roofline": {"kernel": "csa2_index_topk (mq_score_kernel + mq_select_kernel)", "bound": "tensor",
                     "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                     "peak_source": f"{bf16_kind} bf16 GEMM burst x 4, the nominal FP4/BF16 ratio",
                     "flop_per_launch": idx_flop},
        "attention_tflops": att_flop / (att_ms * 1e-3) / 1e12,
        "attention_frac_of_bf16_peak": att_flop / (att_ms * 1e-3) / 1e12 / bf16,
    }
    if with_cpu:
        rec["cpu_baseline"] = _prefill_cpu_sample(n, Q, tokens, T, pos0)
    return rec


def run_prefill(args):
    import sparse_attention_fp4_quant_b200 as csa
    torch.cuda.set_device(0)
    csa.lib()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    rec = measure_c3(csa, args.steps, args.warmup, flush, not args.no_cpu_baseline)
    print(json.dumps({"metric": "CSA2 prefill chunk queries/s (index + Top-512 + one attention layer)",
                      "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                      "dtype": "e2m1+bf16", "data": "synthetic", "config": {"workload": rec["workload"],
                                                                              "l2": "flushed between timed steps"},
                      **{k: v for k, v in rec.items() if k != "workload"}}))


def run_config(args, name):
    """One of the other workloads alone (one GPU), printed as its own JSON line."""
    import sparse_attention_fp4_quant_b200 as csa
    torch.cuda.set_device(0)
    csa.lib()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    fn = {"c0": measure_c0, "c2": measure_c2, "c4": measure_c4, "encoder": measure_encoder_prefill,
          "front": measure_front_end}[name]
    rec = fn(csa, args.steps, args.warmup, flush, not args.no_cpu_baseline)
    print(json.dumps({"config": name, **rec}))


def other_configs(csa, args, flush):
    """Configurations 0, 2, 3 and 4 for the headline line (fewer steps than the headline)."""
    steps, warmup = max(3, min(args.steps, 10)), 3
    with_cpu = not args.no_cpu_baseline
    out = {}
    for name, fn in (("c0", measure_c0), ("c2", measure_c2), ("c3", measure_c3), ("c4", measure_c4),
                     ("f1_encoder_prefill", measure_encoder_prefill), ("f3_front_end", measure_front_end)):
        t0 = time.perf_counter()
        out[name] = fn(csa, steps, warmup, flush, with_cpu)
        out[name]["wall_s"] = time.perf_counter() - t0
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ctx", type=int, default=N_CTX,
                    help="decode context in entries (default the headline 131,072; smaller sizes serve profiling)")
    ap.add_argument("--workload", choices=["decode", "prefill", "c0", "c2", "c4", "encoder", "front"], default="decode",
                    help="decode: the headline B=32 step, with the other four workloads in its line (default); "
                         "prefill (c3), c0, c2, c4: that workload alone on one GPU")
    ap.add_argument("--no-configs", action="store_true", help="leave the other four workloads out of the headline line")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.workload == "prefill":
        run_prefill(args)
        return
    if args.workload in ("c0", "c2", "c4", "encoder", "front"):
        run_config(args, args.workload)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
