#!/usr/bin/env python
"""Decode-step benchmark of the paged INT4/INT8-protected KV cache on B200.

One step = the whole hot path for one batch, through one library call
(kv4_decode_step): fused rotate+quantize+append of one new token per sequence
and the query operands in one kernel, then decode attention (one persistent
stream-K kernel over the INT4 pages and the INT8 sink/recent store that plans
its own split and stores the groups it covers whole; a merge kernel for the
groups split over several CTAs).  --two-calls times the same step as
kv4_rotate_quantize_append + kv4_decode_attention.  The metric is the algorithmic KV bytes the attention reads
per step divided by the step time (GB/s), with decode tokens/s and the fraction
of the measured HBM bandwidth beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl kv4|reference]

Under torchrun each rank runs its own replica of the workload (independent
sequences, weak scaling, no collective on the data path); the step time is the
device time (CUDA events) summed over the K steps, maximum over ranks.
`--impl reference` times the CPU oracle (tests-only restatement of the method)
on a bounded sample of the same workload.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "decode-attention KV GB/s and tokens/s (INT4+INT8-protect), % of B200 HBM peak"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="qwen3_8b_layer")
    ap.add_argument("--impl", default="kv4", choices=["kv4", "reference"])
    ap.add_argument("--no-compare", action="store_true", help="skip the BF16-KV and INT4-only legs")
    ap.add_argument("--two-calls", action="store_true",
                    help="run each step as kv4_rotate_quantize_append + kv4_decode_attention instead of kv4_decode_step")
    ap.add_argument("--rope", action="store_true",
                    help="fuse RoPE (neox, rotary dim = head dim, base 1e6) into the append and query kernels")
    ap.add_argument("--cpu-seqs", type=int, default=4, help="sequences in the CPU oracle sample")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the device steps only (no e2e leg, comparison legs or CPU baseline): for profilers")
    return ap.parse_args()


# --------------------------------------------------------------------------- helpers

def kv_bytes(lengths, Hkv, D, S, W, int4_only=False):
    """Algorithmic KV bytes one attention call reads: INT4 136 B and INT8 264 B per token and KV head at D=128."""
    L = np.asarray(lengths, np.int64)
    prot = np.zeros_like(L) if int4_only else np.minimum(L, S + W)
    return int(np.sum(Hkv * ((L - prot) * 2 * (D // 2 + 4) + prot * 2 * (D + 4))))


def bf16_bytes(lengths, Hkv, D):
    return int(np.sum(np.asarray(lengths, np.int64) * Hkv * 2 * D * 2))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


KERNEL_SOURCES = ("kv4_attention_grouped.cu", "kv4_attn_tiles.cuh", "kv4_common.cuh")


def kernel_source_hash():
    """Digest of the sources of the timed attention kernel (a profile summary is valid for this digest only)."""
    h = hashlib.sha1()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "int4_kv_cache_paged_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def profiled_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", "gattn_kernel_%s.md" % workload)
    try:
        text = open(path).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        item = line.strip().lstrip("-* ").strip()
        if ":" in item and item.startswith(("traffic_bytes_per_launch", "source_sha1")):
            k, v = item.split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha1") != kernel_source_hash():
        return None
    try:
        return int(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """SM clock and clock-event reasons read through NVML every 2 ms by a background thread.

    `window()` brackets a timed region (host time after a device synchronize on
    both sides); `summary()` reports the samples that fall inside the windows.
    Only reads the GPU's state.
    """

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.windows = []
        self.error = None
        self.nvml = None   # (pynvml, handle, max SM clock, reasons getter) once the thread has them

    def _handle(self, pynvml):
        """NVML handle of the torch device, matched by its PCI address (torch reports the parts as integers)."""
        import torch
        props = torch.cuda.get_device_properties(self.dev)
        dom = getattr(props, "pci_domain_id", None)
        bus = getattr(props, "pci_bus_id", None)
        dev = getattr(props, "pci_device_id", None)
        if all(isinstance(x, int) for x in (dom, bus, dev)):
            addr = "%08x:%02x:%02x.0" % (dom, bus, dev)
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                info = pynvml.nvmlDeviceGetPciInfo(h)
                got = info.busId.decode() if isinstance(info.busId, bytes) else str(info.busId)
                if got.lower().endswith(addr[-12:]):
                    return h
        return pynvml.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def _run(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._handle(pynvml)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.nvml = (pynvml, h, smax, get_reasons)
            self.ready.set()
            while not self.stop.is_set():
                self.sample_now()
                time.sleep(0.002)
            self.nvml = None
            pynvml.nvmlShutdown()
        except Exception as e:   # no NVML: reported as unavailable
            self.error = "%s: %s" % (type(e).__name__, e)
        self.ready.set()

    def __enter__(self):
        import threading
        self.stop = threading.Event()
        self.ready = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        self.ready.wait(10.0)   # NVML is up (or known to be missing) before the timed region starts
        return self

    def __exit__(self, *a):
        self.stop.set()
        self.thread.join(timeout=5)

    def sample_now(self, n=1, gap=0.0):
        """Take n samples from the calling thread (the timed loop calls it while its steps run on the GPU, so
        that a short timed region has samples even when the sampling thread does not get to run)."""
        for i in range(n):
            nv = self.nvml
            if nv is None:
                return
            pynvml, h, smax, get_reasons = nv
            t = time.perf_counter()
            self.samples.append((t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), smax, int(get_reasons(h))))
            if gap:
                time.sleep(gap)

    def window(self, t0, t1):
        self.windows.append((t0, t1))

    def summary(self):
        inside = [x for x in self.samples if any(t0 <= x[0] <= t1 for t0, t1 in self.windows)]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0,
                    "note": self.error or "no sample inside the timed region"}
        reasons = sorted({name for x in inside for name, bit in self.REASONS if x[3] & bit})
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": max(x[2] for x in inside),
                "reasons": reasons, "samples": len(inside),
                "source": "NVML: every 2 ms from a thread, plus samples taken while the timed steps run"}


# --------------------------------------------------------------------------- GPU workload

class Workload:
    """One replica: INT4 cache populated to L_b - 1 tokens, per-step new tokens and queries on the device."""

    def __init__(self, w, device, extra_tokens, torch, rope=False):
        import int4_kv_cache_paged_b200 as kv4
        self.w = w
        self.device = device
        self.L = workloads.context_lengths(w)
        self.B = len(self.L)
        table, num_pages, mpps = workloads.block_table(w, self.L, extra_tokens=extra_tokens)
        self.table = table
        self.cfg = workloads.cache_config(w, num_pages, mpps)
        self.cache = kv4.KV4Cache(self.cfg, torch.from_numpy(table), device)
        self.seq_ids = torch.arange(self.B, dtype=torch.int32, device=device)
        self.cu_one = torch.arange(self.B + 1, dtype=torch.int32, device=device)
        self.steps_k = []  # per step: k [B, Hkv, D] bf16
        self.steps_v = []
        self.rope = rope
        if rope:   # the model's angle table (an input), registered once
            max_pos = int(np.max(self.L)) + extra_tokens + 1
            self.cache.set_rope(torch.from_numpy(workloads.rope_cos_sin(max_pos, w["D"])), w["D"], kv4.KV4_ROPE_NEOX)
        self.populate(torch, lambda *a, **k: self.cache.append(*a, rope=rope, **k), extra_tokens)

    def populate(self, torch, append_fn, extra_tokens, layer=0, keep_steps=True):
        w, dev = self.w, self.device
        batch_k, batch_v, counts, ids = [], [], [], []
        step_k = [[None] * self.B for _ in range(extra_tokens)]
        step_v = [[None] * self.B for _ in range(extra_tokens)]
        budget = 0
        for s in range(self.B):
            L = int(self.L[s])
            k, v = workloads.kv_sequence(w, layer, s, L - 1 + extra_tokens, device=dev)
            batch_k.append(k[:L - 1])
            batch_v.append(v[:L - 1])
            counts.append(L - 1)
            ids.append(s)
            for j in range(extra_tokens):
                step_k[j][s] = k[L - 1 + j]
                step_v[j][s] = v[L - 1 + j]
            budget += L
            if budget > 2_000_000 or s == self.B - 1:
                cu = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32, device=dev)
                append_fn(layer, torch.tensor(ids, dtype=torch.int32, device=dev), cu,
                          torch.cat(batch_k).contiguous(), torch.cat(batch_v).contiguous(), total_new=int(sum(counts)))
                batch_k, batch_v, counts, ids, budget = [], [], [], [], 0
        if keep_steps:
            self.steps_k = [torch.stack(x).contiguous() for x in step_k]
            self.steps_v = [torch.stack(x).contiguous() for x in step_v]
        torch.cuda.synchronize()


def reduce_over_ranks(times, counts, device, world):
    """Whole-job figures: the maximum of each timing and the sum of each count over all ranks.

    Every rank calls this once with the same list lengths (one all-reduce each for
    the max and the sum, in the same order on every rank); with one process it
    returns the inputs."""
    if world <= 1:
        return list(times), list(counts)
    import torch
    import torch.distributed as dist
    t = torch.tensor(times, dtype=torch.float64, device=device)
    c = torch.tensor(counts, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(c, op=dist.ReduceOp.SUM)
    return t.tolist(), c.tolist()


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import int4_kv_cache_paged_b200 as kv4

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=device)

    W_, K = args.warmup, args.steps
    w = workloads.workload(args.workload)
    if rank > 0:
        w = workloads.workload(args.workload, seed=w["seed"] + 7919 * rank)   # independent sequences per rank
    if w["layers"] > 1:
        raise SystemExit("the benchmark times single-layer workloads; use the stack test for %s" % args.workload)
    extra = W_ + 5 * K + 1   # warm-up + timed steps, the kernel-event pass, e2e, two comparison legs
    t0 = time.time()
    wl = Workload(w, device, extra, torch, rope=args.rope)
    amode = kv4.KV4_MODE_ROPE_Q if args.rope else 0
    setup_s = time.time() - t0
    B, Hkv, D, S, Wn = wl.B, w["Hkv"], w["D"], w["S"], w["W"]
    ws = wl.cache.workspace(B)
    out = torch.empty((B, w["Hq"], D), dtype=torch.bfloat16, device=device)
    qs = [workloads.queries(w, 0, i, device=device) for i in range(W_ + K)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    n = W_ + K
    e_step = [(ev(), ev()) for _ in range(n)]
    e_kern = [(ev(), ev()) for _ in range(K)]
    step_bytes, kern_bytes = [], []

    def one_step(i, q):
        """The decode step on token i of every sequence: one library call (or the two calls)."""
        if args.two_calls:
            wl.cache.append(0, wl.seq_ids, wl.cu_one, wl.steps_k[i], wl.steps_v[i], total_new=B, rope=args.rope)
            wl.cache.attention(0, wl.seq_ids, q, out=out, workspace=ws, mode=amode)
        else:   # append + query operands, then the attention and merge kernels
            wl.cache.decode_step(0, wl.seq_ids, wl.steps_k[i], wl.steps_v[i], q, out=out, workspace=ws, mode=amode)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    barrier()
    with ClockSampler(device) as clocks:
        for i in range(n):
            if i == W_:
                barrier()
                t_window = time.perf_counter()
            flush.fill_(i & 0xFF)                  # evict the KV of the previous step from L2 (not timed)
            e_step[i][0].record(stream)
            one_step(i, qs[i])
            e_step[i][1].record(stream)
            step_bytes.append(kv_bytes(wl.L + i, Hkv, D, S, Wn))
        clocks.sample_now(4, 0.0003)                # while the queued steps run
        barrier()
        clocks.window(t_window, time.perf_counter())
        # the same steps again on the next K tokens, now with the library's events around the attention
        # kernel and its merge kernel (with --two-calls also the query-operand kernel): they give the
        # roofline's kernel time.  They are kept out of the loop above because each event marker between
        # two launches adds about 2 us to the step.
        t_window = time.perf_counter()
        for j in range(K):
            flush.fill_(j & 0xFF)
            kv4.kv4_set_attention_events(wl.cache.handle, *e_kern[j])
            one_step(n + j, qs[W_ + j])
            kern_bytes.append(kv_bytes(wl.L + n + j, Hkv, D, S, Wn))
        clocks.sample_now(4, 0.0003)
        barrier()
        clocks.window(t_window, time.perf_counter())
    kv4.kv4_set_attention_events(wl.cache.handle, None, None)
    status = wl.cache.status()

    timed = range(W_, n)
    t_step = sum(e_step[i][0].elapsed_time(e_step[i][1]) for i in timed) / 1e3
    t_kern = sum(a.elapsed_time(b) for a, b in e_kern) / 1e3
    t_attn = t_kern
    bytes_timed = sum(step_bytes[i] for i in timed)
    bytes_kern = sum(kern_bytes)
    n += K                                          # tokens used so far

    # ---- e2e through the public API with host buffers (pinned), copies inside the timed region
    if args.kernel_only:
        K_e2e = 0
    else:
        K_e2e = K
    # each step's inputs (new K, new V, q) packed in one pinned host buffer: one host->device copy per step
    kv_elems, q_elems = wl.steps_k[0].numel(), qs[0].numel()
    hin = []
    for j in range(K_e2e):
        h = torch.empty(2 * kv_elems + q_elems, dtype=torch.bfloat16).pin_memory()
        h[:kv_elems].copy_(wl.steps_k[n + j].reshape(-1).cpu())
        h[kv_elems:2 * kv_elems].copy_(wl.steps_v[n + j].reshape(-1).cpu())
        h[2 * kv_elems:].copy_(workloads.queries(w, 0, n + j, device="cpu").reshape(-1))
        hin.append(h)
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    din = torch.empty(2 * kv_elems + q_elems, dtype=torch.bfloat16, device=device)
    dk = din[:kv_elems].view(wl.steps_k[0].shape)
    dv = din[kv_elems:2 * kv_elems].view(wl.steps_v[0].shape)
    dq = din[2 * kv_elems:].view(qs[0].shape)
    e_e2e = [(ev(), ev()) for _ in range(K_e2e)]
    e2e_bytes = 0
    barrier()
    for j in range(K_e2e):
        flush.fill_(j & 0xFF)
        e_e2e[j][0].record(stream)
        din.copy_(hin[j], non_blocking=True)
        if args.two_calls:
            wl.cache.append(0, wl.seq_ids, wl.cu_one, dk, dv, total_new=B, rope=args.rope)
            wl.cache.attention(0, wl.seq_ids, dq, out=out, workspace=ws, mode=amode)
        else:
            wl.cache.decode_step(0, wl.seq_ids, dk, dv, dq, out=out, workspace=ws, mode=amode)
        hout.copy_(out, non_blocking=True)
        e_e2e[j][1].record(stream)
        e2e_bytes += kv_bytes(wl.L + n + j, Hkv, D, S, Wn)
    barrier()
    t_e2e = sum(a.elapsed_time(b) for a, b in e_e2e) / 1e3 if K_e2e else float("nan")
    h2d = dk.numel() * 2 + dv.numel() * 2 + dq.numel() * 2
    d2h = hout.numel() * 2

    # ---- comparison legs on identical inputs (rank-local, untimed by the contract)
    compare = None
    if not args.no_compare and not args.kernel_only and not args.rope and world == 1:
        compare = compare_legs(torch, kv4, w, wl, K, device, flush, n + K_e2e)

    (t_step_all, t_e2e_all), (bytes_all, e2e_bytes_all) = reduce_over_ranks(
        [t_step, t_e2e], [float(bytes_timed), float(e2e_bytes)], device, world)

    result = None
    if rank == 0:
        peaks, peak_kind = measured_peaks()
        hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        achieved = bytes_kern / t_kern / 1e9
        value = bytes_all / t_step_all / 1e9
        traffic = profiled_traffic(args.workload)
        clk = clocks.summary()
        result = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": W_,
            "ms_per_step": round(t_step_all / K * 1e3, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "int4/int8 codes, fp16 scales, bf16 q/out, fp16 tensor-core operands, fp32 accumulate",
            "data": "synthetic (seeded N(0,1) K/V with outlier K channels and a large-norm sink, bf16)",
            "config": {"workload": args.workload, "batch": B, "q_heads": w["Hq"], "kv_heads": Hkv, "head_dim": D,
                       "page": w["P"], "hadamard_block": w["Bh"], "sinks": S, "recent_window": Wn,
                       "context": "%s, mean %.0f at the first timed step" % (w["ctx"][0], float(np.mean(wl.L + W_))),
                       "kv_bytes_per_step_mb": round(bytes_timed / K / 1e6, 1),
                       "l2": "flushed before every step by a 256 MB write outside the timed events; "
                             "per-step KV also exceeds the 126 MB L2",
                       "parallelism": "replica per GPU" if world > 1 else "single GPU",
                       "rope": ("neox, rotary dim %d, base 1e6, fused into the append and query kernels" % D
                                if args.rope else "none (keys arrive post-RoPE)")},
            "tokens_per_s": round(B * world * K / t_step_all, 1),
            "hbm_frac_of_%s" % peak_kind: round(value / hbm, 4),
            "attention_kv_gbs": round(bytes_kern / t_attn / 1e9, 2),
            "api": "two calls: kv4_rotate_quantize_append + kv4_decode_attention" if args.two_calls else
                   "one call: kv4_decode_step",
            ("append_us_per_step" if args.two_calls else "append_and_query_us_per_step"):
                round((t_step - t_attn) / K * 1e6, 2),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": hbm, "unit": "GB/s",
                         "frac": round(achieved / hbm, 4), "traffic": traffic,
                         "kernel": "gattn_kernel: persistent stream-K attention over the INT4 pages and the "
                                   "INT8 store (the events span it and the merge kernel, its programmatic "
                                   "dependent; with --two-calls also the query-operand kernel before it)",
                         "peak_source": peak_kind, "bytes_per_launch": int(bytes_kern / K),
                         "timing": "CUDA events recorded by the library around the kernels, over K steps that "
                                   "follow the timed loop on the same workload"},
            "e2e": ({"value": round(e2e_bytes_all / t_e2e_all / 1e9, 2), "unit": "GB/s",
                     "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                     "tokens_per_s": round(B * world * K / t_e2e_all, 1)} if K_e2e else None),
            # per step: gstep_kernel, gattn_kernel, gmerge_kernel (two calls: append_kernel, gq_kernel, gattn, gmerge)
            "gpu_launches": (4 if args.two_calls else 3) * K,
            "clocks": clk,
            "device_status": status,
            "setup_s": round(setup_s, 1),
        }
        if compare:
            result["compare"] = compare
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def compare_legs(torch, kv4, w, wl, K, device, flush, first_token):
    """Attention-only time of the INT4 path, the INT4-only mode, the multi-token query path and the BF16-KV
    kernel on identical inputs."""
    B, Hkv, D, S, Wn = wl.B, w["Hkv"], w["D"], w["S"], w["W"]
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    qs = [workloads.queries(w, 0, 1000 + i, device=device) for i in range(K)]
    out = torch.empty((B, w["Hq"], D), dtype=torch.bfloat16, device=device)

    def time_attn(fn):
        es = [(ev(), ev()) for _ in range(K)]
        for i in range(3):
            fn(qs[i])
        torch.cuda.synchronize()
        for i in range(K):
            flush.fill_(i & 0xFF)
            es[i][0].record()
            fn(qs[i])
            es[i][1].record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in es) / 1e3 / K

    ws = wl.cache.workspace(B)
    # the decode step as two calls (append, then attention), then as one call, on the next 2K tokens
    def time_steps(fn, t0):
        es = [(ev(), ev()) for _ in range(K)]
        for i in range(K):
            flush.fill_(i & 0xFF)
            es[i][0].record()
            fn(t0 + i, qs[i])
            es[i][1].record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in es) / 1e3 / K

    def two_calls(i, q):
        wl.cache.append(0, wl.seq_ids, wl.cu_one, wl.steps_k[i], wl.steps_v[i], total_new=B)
        wl.cache.attention(0, wl.seq_ids, q, out=out, workspace=ws)

    t_two = time_steps(two_calls, first_token)
    t_one = time_steps(lambda i, q: wl.cache.decode_step(0, wl.seq_ids, wl.steps_k[i], wl.steps_v[i], q, out=out,
                                                          workspace=ws), first_token + K)
    L_now = wl.L + int(wl.cache.seq_lens()[0, 0].item()) - int(wl.L[0])
    t_int4 = time_attn(lambda q: wl.cache.attention(0, wl.seq_ids, q, out=out, workspace=ws))
    t_only = time_attn(lambda q: wl.cache.attention(0, wl.seq_ids, q, out=out, workspace=ws,
                                                    mode=kv4.KV4_MODE_INT4_ONLY))
    res = {"step_as_two_calls": {"ms_per_step": round(t_two * 1e3, 4)},
           "step_as_one_call": {"ms_per_step": round(t_one * 1e3, 4)},
           "int4_protected": {"attention_ms": round(t_int4 * 1e3, 4),
                              "kv_gbs": round(kv_bytes(L_now, Hkv, D, S, Wn) / t_int4 / 1e9, 1)},
           "int4_only": {"attention_ms": round(t_only * 1e3, 4),
                         "kv_gbs": round(kv_bytes(L_now, Hkv, D, S, Wn, int4_only=True) / t_only / 1e9, 1)}}
    # multi-token query (speculative verification): the most query tokens whose
    # heads fit one 8-column operand, causal over the same cache
    T = 8 // (w["Hq"] // Hkv)
    if T >= 2:
        gen = torch.Generator(device=device).manual_seed(4242)
        qx = [torch.randn((B, T, w["Hq"], D), generator=gen, device=device).to(torch.bfloat16) for _ in range(3)]
        outx = torch.empty((B, T, w["Hq"], D), dtype=torch.bfloat16, device=device)
        wsx = wl.cache.extend_workspace(B, T)
        ix = iter(range(1 << 30))
        t_ext = time_attn(lambda q: wl.cache.extend_attention(0, wl.seq_ids, qx[next(ix) % 3], out=outx,
                                                                workspace=wsx))
        res["extend"] = {"q_len": T, "attention_ms": round(t_ext * 1e3, 4),
                         "kv_gbs": round(kv_bytes(L_now, Hkv, D, S, Wn) / t_ext / 1e9, 1),
                         "query_tokens_per_s": round(B * T / t_ext, 1)}
    need = bf16_bytes(L_now, Hkv, D)
    free = torch.cuda.mem_get_info()[0]
    if need * 1.3 < free:
        cache16 = kv4.BF16Cache(wl.cfg, torch.from_numpy(wl.table), device)
        lens = L_now
        extra_w = dict(w)
        # identical K/V values: regenerate the same per-sequence tokens up to the current length
        tmp = Workload.__new__(Workload)
        tmp.w, tmp.device, tmp.B = w, device, B
        tmp.L = lens + 1
        tmp.populate(torch, cache16.append, 0, keep_steps=False)
        ws16 = cache16.workspace(B)
        t_bf16 = time_attn(lambda q: cache16.attention(0, wl.seq_ids, q, out=out, workspace=ws16))
        res["bf16_kv"] = {"attention_ms": round(t_bf16 * 1e3, 4), "kv_gbs": round(need / t_bf16 / 1e9, 1),
                          "speedup_int4_protected_vs_bf16": round(t_bf16 / t_int4, 3)}
        del cache16, extra_w
    else:
        res["bf16_kv"] = {"skipped": "BF16 cache of %.1f GB does not fit" % (need / 1e9)}
    return res


# --------------------------------------------------------------------------- CPU oracle

def run_oracle_sample(w, n_seqs, steps, warm=1, rope=False):
    """The oracle on `n_seqs` sequences of the workload: populate (untimed), then `steps` decode steps."""
    import torch
    from threadpoolctl import threadpool_limits
    from oracle import OracleKV4Cache, decode_attention, ROPE_NEOX

    L = workloads.context_lengths(w)[:n_seqs]
    table, num_pages, mpps = workloads.block_table(dict(w, batch=n_seqs), L, extra_tokens=steps + warm + 1)
    cfg = workloads.cache_config(w, num_pages, mpps, max_seqs=n_seqs)
    orc = OracleKV4Cache(cfg, table)
    rp = (workloads.rope_cos_sin(int(np.max(L)) + steps + warm + 1, w["D"]), w["D"], ROPE_NEOX) if rope else None
    toks = []
    with threadpool_limits(1):
        for s in range(n_seqs):
            k, v = workloads.kv_sequence(w, 0, s, int(L[s]) + steps + warm, device="cpu")
            k, v = k.float().numpy(), v.float().numpy()
            orc.append(0, [s], [0, int(L[s]) - 1], k[:L[s] - 1], v[:L[s] - 1], rope=rp)
            toks.append((k, v))
        times, nbytes = [], []
        for i in range(steps + warm):
            kn = np.stack([toks[s][0][L[s] - 1 + i] for s in range(n_seqs)])
            vn = np.stack([toks[s][1][L[s] - 1 + i] for s in range(n_seqs)])
            q = workloads.queries(w, 0, i, n=n_seqs, device="cpu").float().numpy()
            t0 = time.perf_counter()
            orc.append(0, list(range(n_seqs)), np.arange(n_seqs + 1), kn, vn, rope=rp)
            decode_attention(orc, 0, list(range(n_seqs)), q, rope=rp)
            dt = time.perf_counter() - t0
            if i >= warm:
                times.append(dt)
                nbytes.append(kv_bytes(L + i, w["Hkv"], w["D"], w["S"], w["W"]))
    return sum(nbytes) / sum(times) / 1e9, times, int(np.mean(L))


def cpu_baseline(w, n_seqs, rope=False):
    gbs, times, mean_l = run_oracle_sample(w, n_seqs, steps=2, rope=rope)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d of %d sequences (mean context %d), 2 decode steps (append + attention), numpy, "
                      "BLAS limited to 1 thread; %.1f s per step" % (n_seqs, w["batch"], mean_l, np.mean(times))}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    w = workloads.workload(args.workload)
    n_seqs = max(1, min(args.cpu_seqs, 2))
    gbs, times, mean_l = run_oracle_sample(w, n_seqs, steps=args.steps, warm=args.warmup, rope=args.rope)
    t = sum(times)
    base = {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d of %d sequences (mean context %d) per step, numpy, BLAS limited to 1 thread"
                      % (n_seqs, w["batch"], mean_l)}
    return {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 attention, f32 codes",
            "data": "synthetic", "config": {"workload": args.workload, "batch_sample": n_seqs,
                                            "rope": "neox, fused" if args.rope else "none"},
            "cpu_baseline": base, "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                                          "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.impl == "reference":
        res = run_reference(args)
        if res is not None:
            print(json.dumps(res))
        return
    res = run_gpu(args)
    if res is not None:
        if res["n_gpus"] == 1 and not args.kernel_only:
            res["cpu_baseline"] = cpu_baseline(workloads.workload(args.workload), args.cpu_seqs, rope=args.rope)
        print(json.dumps(res))


if __name__ == "__main__":
    main()
