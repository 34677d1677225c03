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
INDEX_LAUNCH_BYTES = B * N_CTX * IDX_BYTES_PER_ENTRY + B * (128 + 16 + 16) + B * TOPK * 4
ATTN_LAYER_BYTES = B * (TOPK * ROW_BYTES + T_SWA * SWA_BYTES + Q_OUT_BYTES + IDX_LIST_BYTES)
STEP_BYTES = B * N_CTX * IDX_BYTES_PER_ENTRY + len(LAYERS) * ATTN_LAYER_BYTES


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


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
    h = hashlib.sha256()
    for f in ("index_cluster.cu", "index_pipe.cuh", "index_tc.cu", "tc.cuh", "common.cuh", "cluster.cuh", "kernels.h"):
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

    def __init__(self, csa, seed, device):
        self.csa = csa
        self.device = device
        self.kv = csa.KV(B, N_CTX, 1, device)
        self.W = synth.proj_w(seed).to(device)
        # context: N_CTX - 1 cached entries; the step appends the new token at N_CTX - 1
        for b in range(B):
            lat = synth.latent(synth.seed_of("bench-ctx", seed, b), N_CTX - 1, 0, device)
            csa.csa2_quant_nvfp4(lat, self.kv.lat[b].view(-1, 256), self.kv.lat_sc[b].view(-1, 32))
            csa.csa2_index_k_proj(lat, self.W, self.kv.ik[b].view(-1, 32), self.kv.ik_sc[b].view(-1, 4))
            del lat
        self.kv.n_entries.fill_(N_CTX)
        self.new_lat = torch.stack([synth.latent(synth.seed_of("bench-new", seed, b), 1, N_CTX - 1, device)[0]
                                    for b in range(B)])
        self.new_rows = (torch.arange(B, device=device, dtype=torch.int64) * N_CTX + (N_CTX - 1))
        self.iq_bf = synth.index_q(synth.seed_of("bench-iq", seed), B, 1, device)
        self.w = synth.index_w(B, 1, device)
        self.q_pos = torch.full((B, 1), N_CTX - 1, dtype=torch.int32, device=device)
        self.q = [synth.attn_q(synth.seed_of("bench-q", seed, li), B, 1, device) for li in range(len(LAYERS))]
        self.swa = []
        for li in range(len(LAYERS)):
            cs = [synth.swa_kv(synth.seed_of("bench-swa", seed, li, b), T_SWA, N_CTX - T_SWA, device) for b in range(B)]
            self.swa.append((torch.stack([c[0] for c in cs]), torch.stack([c[1] for c in cs])))
        self.swa_pos0 = torch.full((B,), N_CTX - T_SWA, dtype=torch.int32, device=device)
        self.iq = torch.empty((B, 1, 128), dtype=torch.uint8, device=device)
        self.iqs = torch.empty((B, 1, 16), dtype=torch.uint8, device=device)
        self.idx = torch.empty((B, 1, TOPK), dtype=torch.int32, device=device)
        self.out = [torch.empty((B, 1, 16, 512), dtype=torch.bfloat16, device=device) for _ in LAYERS]
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

    def step_with_host_io(self, h_new, h_iq, h_q, h_out):
        """One step fed from pinned host buffers and read back to them: the append and
        indexer inputs are copied in first; the attention queries travel on a copy stream
        while the front and the index run; each layer's output is copied back as soon as
        the layer is done."""
        cur = torch.cuda.current_stream()
        self.new_lat.copy_(h_new, non_blocking=True)
        self.iq_bf.copy_(h_iq, non_blocking=True)
        self.io_in.wait_stream(cur)
        self.io_out.wait_stream(cur)
        ready = []
        with torch.cuda.stream(self.io_in):   # host -> device, beside the front and the index
            for q, hq in zip(self.q, h_q):
                q.copy_(hq, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.io_in)
                ready.append(ev)
        self.front()
        self.index()
        for li in range(len(LAYERS)):
            cur.wait_event(ready[li])
            self.attention_layer(li)
            done = torch.cuda.Event()
            done.record(cur)
            with torch.cuda.stream(self.io_out):   # device -> host, the other direction of the link
                self.io_out.wait_event(done)
                h_out[li].copy_(self.out[li], non_blocking=True)
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
    grp = DecodeGroup(csa, seed=9 + rank, device=device)
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
    h_new = grp.new_lat.cpu().pin_memory()
    h_iq = grp.iq_bf.cpu().pin_memory()
    h_q = [q.cpu().pin_memory() for q in grp.q]
    h_out = [torch.zeros(o.shape, dtype=o.dtype).pin_memory() for o in grp.out]
    h2d = h_new.numel() * 2 + h_iq.numel() * 2 + sum(q.numel() * 2 for q in h_q)
    d2h = sum(o.numel() * 2 for o in h_out)
    g_e2e = _graph(lambda: grp.step_with_host_io(h_new, h_iq, h_q, h_out))
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

    if rank != 0:
        return
    peak, peak_kind = _peaks()
    idx_s = float(np.mean(index_ms)) / 1000.0
    achieved = INDEX_LAUNCH_BYTES / idx_s / 1e9
    traffic = _ncu_traffic()
    cb = _oracle_baseline() if (world == 1 and not args.no_cpu_baseline) else None
    value = job_value(world, ms_max)
    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1+bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B_per_gpu": B, "ctx_entries": N_CTX, "topk": TOPK, "swa": T_SWA,
                   "l2": "flushed between timed steps (256 MiB write outside the step events)",
                   "graphs": "one CUDA graph per step (front with two branches, index, 4 attention layers)"},
        "index_attn_gbs": STEP_BYTES / (ms_max / 1000.0) / 1e9,
        "index_attn_frac_of_hbm": STEP_BYTES / (ms_max / 1000.0) / 1e9 / peak,
        "step_algorithmic_bytes": STEP_BYTES,
        "segments_ms": {"front": float(np.mean(front_ms)), "index_topk": float(np.mean(index_ms)),
                        "attention_x4": float(np.mean(attn_ms)),
                        "how": "the step re-run as three graphs with events between them (diagnostic)"},
        "roofline": {"kernel": "csa2_index_topk (index_cluster_kernel)", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                     "bytes_per_launch": INDEX_LAUNCH_BYTES},
        "cpu_baseline": cb,
        "e2e": {"value": job_value(world, e2e_max), "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_max},
        "gpu_launches": DecodeGroup.LAUNCHES_PER_STEP * args.steps,
        "clocks": clocks,
        "wall_s_timed_region": wall_s,
    }
    print(json.dumps(line), flush=True)


def run_prefill(args):
    """The prefill chunk (one GPU): 65,536-token prompt compressed 2:1 into 32,768 entries,
    4,096 queries at its end; index + Top-512 and one attention layer (main + SWA-128),
    each timed with CUDA events over K steps, L2 flushed between steps."""
    import sparse_attention_fp4_quant_b200 as csa
    torch.cuda.set_device(0)
    csa.lib()
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
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream()
    t_idx, t_att = [], []
    for it in range(args.warmup + args.steps):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(st)
        csa.csa2_index_topk(iq, iqs, w, kv, q_pos, TOPK, idx, ws=ws)
        ev[1].record(st)
        csa.csa2_sparse_attn(q, kv, idx, swa, swa_sc, pos0_t, q_pos, out=out, ws=ws)
        ev[2].record(st)
        torch.cuda.synchronize()
        if it >= args.warmup:
            t_idx.append(ev[0].elapsed_time(ev[1]))
            t_att.append(ev[1].elapsed_time(ev[2]))
    idx_ms, att_ms = float(np.mean(t_idx)), float(np.mean(t_att))
    nvis = np.minimum((q_pos.cpu().numpy().astype(np.int64) + 1) // 2, n)
    idx_flop = float(nvis.sum()) * 4 * 64 * 2           # dense-equivalent indexer Q.K^T
    att_flop = float(Q) * 16 * (TOPK + T_SWA) * 512 * 4  # S and P V over every slot
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
        bf16 = float(json.load(f)["bf16_tflops"])
    fp4_peak = bf16 * 4.0   # nominal dense FP4 / BF16 ratio (9 / 2.25 PFLOP/s)
    achieved = idx_flop / (idx_ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": "CSA2 prefill chunk queries/s (index + Top-512 + one attention layer)",
        "value": Q / ((idx_ms + att_ms) * 1e-3), "unit": "queries/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": idx_ms + att_ms, "higher_is_better": True, "dtype": "e2m1+bf16",
        "data": "synthetic",
        "config": {"workload": "c3: prefill chunk, 65,536-token prompt, m=2 (32,768 entries), 4,096 queries, "
                               "Top-512, SWA-128", "l2": "flushed between timed steps"},
        "index_ms": idx_ms, "attention_ms": att_ms,
        "roofline": {"kernel": "csa2_index_topk (mq_score_kernel + mq_select_kernel)", "bound": "tensor",
                     "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                     "peak_source": "measured bf16 GEMM burst (MEASURED_PEAKS.json) x 4, the nominal FP4/BF16 ratio",
                     "flop_per_launch": idx_flop},
        "attention_tflops": att_flop / (att_ms * 1e-3) / 1e12,
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["decode", "prefill"], default="decode",
                    help="decode: the headline B=32 step (default); prefill: the 4,096-query chunk, one GPU")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.workload == "prefill":
        run_prefill(args)
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
