#!/usr/bin/env python
"""Decode-step benchmark of the paged INT4/INT8-protected KV cache on B200.

The headline workload is the 36-layer decode stack of a Qwen3-8B-shaped model
(36 independent layer caches, 256 sequences of 4096-16384 tokens, 32/8 heads,
head dim 128).  One step is the whole hot path for one decode token of every
sequence through all 36 layers: per layer one library call, kv4_decode_step
(fused rotate+quantize+append of the new token and the query operands in one
kernel, then the persistent stream-K attention kernel over the INT4 pages and
the INT8 sink/recent store, and a merge kernel for the head groups split over
several CTAs).  --two-calls times each layer as kv4_rotate_quantize_append +
kv4_decode_attention.  The metric is the algorithmic KV bytes the attention
reads per step divided by the step time (GB/s), with decode tokens/s and the
fraction of the measured HBM bandwidth beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl kv4|reference]

Beside the headline line it reports, on the same seeded inputs: the INT4-only
(no protection) mode and the BF16-KV kernel (on as many layer caches as fit),
and a `workloads` object with the single-layer workloads (64-sequence layer,
512-sequence async-RL batch, 8 x 131072 long context), each with its own step
throughput, roofline fraction and speedup over the BF16-KV kernel.

Under torchrun each rank runs its own replica of the workload (independent
sequences, weak scaling, no collective on the data path); the step time is the
device time (CUDA events) summed over the K steps, maximum over ranks.
`--impl reference` times the CPU oracle (the tests-only restatement of the
method) on a bounded sample of the same workload, one sequence per host core.
"""

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "decode-attention KV GB/s and tokens/s (INT4+INT8-protect), % of B200 HBM peak"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
SUBLINES = ("qwen3_8b_layer", "async_rl", "long_context", "tiny")   # tiny: the parity fixture, a latency
BF16_MAX_LAYERS = 12          # distinct BF16 layer caches of the comparison leg on the stack (at most)


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="stack36")
    ap.add_argument("--layers", type=int, default=0,
                    help="use only the first N layer caches of the workload (profiling a smaller case)")
    ap.add_argument("--impl", default="kv4", choices=["kv4", "reference"])
    ap.add_argument("--no-compare", action="store_true", help="skip the BF16-KV, INT4-only and multi-token legs")
    ap.add_argument("--no-sublines", action="store_true", help="skip the single-layer workloads object")
    ap.add_argument("--sub-steps", type=int, default=10, help="timed steps of each single-layer sub-line")
    ap.add_argument("--two-calls", action="store_true",
                    help="run each layer as kv4_rotate_quantize_append + kv4_decode_attention instead of "
                         "kv4_decode_step")
    ap.add_argument("--rope", action="store_true",
                    help="fuse RoPE (neox, rotary dim = head dim, base 1e6) into the append and query kernels")
    ap.add_argument("--cpu-procs", type=int, default=0,
                    help="processes of the CPU oracle sample (0: one per host core)")
    ap.add_argument("--cpu-steps", type=int, default=2, help="timed decode steps of the CPU oracle sample")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the device steps only (no e2e leg, comparison legs, sub-lines or CPU baseline): "
                         "for profilers")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------- helpers

def kv_bytes(lengths, Hkv, D, S, W, int4_only=False, fmt=0):
    """Algorithmic KV bytes one attention call reads: INT4 136 B (NVFP4 pages 144 B, INT2 pages 72 B) and INT8
    264 B per token and KV head at D=128."""
    L = np.asarray(lengths, np.int64)
    prot = np.zeros_like(L) if int4_only else np.minimum(L, S + W)
    page = {0: 2 * (D // 2 + 4), 1: 2 * (D // 2 + D // 16), 2: 2 * (D // 4 + 4)}[fmt]
    return int(np.sum(Hkv * ((L - prot) * page + prot * 2 * (D + 4))))


def bf16_bytes(lengths, Hkv, D):
    return int(np.sum(np.asarray(lengths, np.int64) * Hkv * 2 * D * 2))


def side_bytes(lengths, w, layers):
    """Bytes a decode step moves outside the KV stream (not in `value`), summed over `layers`: the bf16 queries
    read and outputs written, the new token's bf16 K and V read and its codes written (INT4 pages and the INT8
    store: the newest position is always protected), and the block-table entries the attention kernel reads
    (one int32 per page and group of 4, 2 or 1 KV heads).  `lengths` are the cache lengths the step attends."""
    L = np.asarray(lengths, np.int64)
    B, Hq, Hkv, D, P = len(L), w["Hq"], w["Hkv"], w["D"], w["P"]
    gwr = 4 if Hkv % 4 == 0 else (2 if Hkv % 2 == 0 else 1)
    q = B * Hq * D * 2
    new_read = B * Hkv * 2 * D * 2
    new_written = B * Hkv * (2 * (D // 2 + 4) + 2 * (D + 4))
    table = int(np.sum(-(-L // P))) * (Hkv // gwr) * 4
    per_layer = {"q_read": q, "out_written": q, "new_kv_read": new_read, "new_kv_written": new_written,
                 "block_table_read": table}
    res = {k: v * layers for k, v in per_layer.items()}
    res["total"] = sum(res.values())
    res["kv_stream"] = kv_bytes(L, Hkv, D, w["S"], w["W"]) * layers
    return res


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


KERNEL_SOURCES = ("kv4_attention_grouped.cu", "kv4_attn_tiles.cuh", "kv4_common.cuh", "kv4_append_ops.cuh")


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

class Replica:
    """One replica of a workload on one GPU: a cache of `layers` layer caches, each populated to L_b - 1
    tokens of every sequence, the new K/V of `extra` decode steps per layer and the queries of `n_q` steps
    per layer (all on the device)."""

    def __init__(self, w, layers, device, extra, n_q, torch, rope=False):
        import int4_kv_cache_paged_b200 as kv4
        self.w = w
        self.layers = layers
        self.device = device
        self.L = workloads.context_lengths(w)
        self.B = len(self.L)
        table, num_pages, mpps = workloads.block_table(w, self.L, extra_tokens=extra)
        self.table = table
        self.cfg = workloads.cache_config(w, num_pages, mpps, layers=layers)
        self.cache = kv4.KV4Cache(self.cfg, torch.from_numpy(table), device)
        self.seq_ids = torch.arange(self.B, dtype=torch.int32, device=device)
        self.cu_one = torch.arange(self.B + 1, dtype=torch.int32, device=device)
        self.rope = rope
        if rope:   # the model's angle table (an input), registered once
            max_pos = int(np.max(self.L)) + extra + 1
            self.cache.set_rope(torch.from_numpy(workloads.rope_cos_sin(max_pos, w["D"])), w["D"], kv4.KV4_ROPE_NEOX)
        self.steps_k, self.steps_v = [], []   # per layer: [extra, B, Hkv, D] bf16
        for layer in range(layers):
            k, v = populate(torch, w, self.L, lambda *a, **kw: self.cache.append(*a, rope=rope, **kw), layer,
                            extra, device)
            self.steps_k.append(k)
            self.steps_v.append(v)
        # queries per (layer, step), drawn once (outside every timed region)
        self.qs = [torch.stack([workloads.queries(w, layer, i, device=device) for i in range(n_q)])
                   for layer in range(layers)]
        torch.cuda.synchronize()

    def bytes_at(self, tokens_appended, int4_only=False):
        """Algorithmic KV bytes of one attention call of one layer after `tokens_appended` decode appends."""
        w = self.w
        return kv_bytes(self.L - 1 + tokens_appended, w["Hkv"], w["D"], w["S"], w["W"], int4_only)


def populate(torch, w, L, append_fn, layer, extra, device, upto=0, budget_tokens=1_000_000):
    """Append the seeded tokens 0 .. L_b - 2 + upto of every sequence to `layer` (batched calls); return the
    tokens L_b - 1 + upto .. L_b - 2 + extra of every sequence as [extra - upto, B, Hkv, D] K and V tensors.
    Each sequence is drawn with length L_b - 1 + extra whatever `upto` is, so the same (L, extra) gives the
    same token values (the generator draws V after all of K)."""
    B = len(L)
    batch_k, batch_v, counts, ids = [], [], [], []
    step_k = torch.empty((extra - upto, B, w["Hkv"], w["D"]), dtype=torch.bfloat16, device=device)
    step_v = torch.empty_like(step_k)
    budget = 0
    for s in range(B):
        n = int(L[s]) - 1 + upto
        k, v = workloads.kv_sequence(w, layer, s, int(L[s]) - 1 + extra, device=device)
        batch_k.append(k[:n])
        batch_v.append(v[:n])
        counts.append(n)
        ids.append(s)
        step_k[:, s] = k[n:]
        step_v[:, s] = v[n:]
        budget += n
        if budget > budget_tokens or s == B - 1:
            cu = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32, device=device)
            append_fn(layer, torch.tensor(ids, dtype=torch.int32, device=device), cu,
                      torch.cat(batch_k).contiguous(), torch.cat(batch_v).contiguous(), total_new=int(sum(counts)))
            batch_k, batch_v, counts, ids, budget = [], [], [], [], 0
    return step_k, step_v


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


class Nvtx:
    """NVTX ranges through torch, or nothing where its build has none."""

    def __init__(self, torch):
        self.m = getattr(torch.cuda, "nvtx", None)
        try:
            self.m.range_push("kv4")
            self.m.range_pop()
        except Exception:   # noqa: BLE001 -- any failure: no ranges
            self.m = None

    def push(self, name):
        if self.m is not None:
            self.m.range_push(name)

    def pop(self):
        if self.m is not None:
            self.m.range_pop()


def measure(torch, kv4, w, layers, args, K, W_, device, clocks, world=1, compare=True):
    """Build a replica of workload `w` (its first `layers` layer caches) and time it.

    Returns the per-rank raw figures (step time, bytes, kernel time, e2e) and the rank-local comparison
    legs.  The collective steps (barriers) are the same on every rank."""
    import torch.distributed as dist
    B, Hkv, D, S, Wn, Hq = w["batch"], w["Hkv"], w["D"], w["S"], w["W"], w["Hq"]
    two, rope = args.two_calls, args.rope
    amode = kv4.KV4_MODE_ROPE_Q if rope else 0
    K_e2e = 0 if args.kernel_only else K
    do_cmp = compare and not args.kernel_only and not rope and world == 1
    n_cmp = 2 * K if do_cmp else 0              # the step as two calls and as one call
    n_diag = min(K_e2e, 5)                       # the e2e breakdown
    extra = W_ + 2 * K + K_e2e + n_diag + n_cmp + 1   # timed loop, kernel-event pass, e2e, comparison steps
    t0 = time.time()
    rep = Replica(w, layers, device, extra, W_ + K, torch, rope=rope)
    rep.extra = extra
    setup_s = time.time() - t0
    cache = rep.cache
    ws = cache.workspace(B)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def layer_step(layer, i, qi, o=out):
        """Decode step of layer `layer` on the i-th new token of every sequence (one call, or the two)."""
        if two:
            cache.append(layer, rep.seq_ids, rep.cu_one, rep.steps_k[layer][i], rep.steps_v[layer][i], total_new=B,
                         rope=rope)
            cache.attention(layer, rep.seq_ids, rep.qs[layer][qi], out=o, workspace=ws, mode=amode)
        else:
            cache.decode_step(layer, rep.seq_ids, rep.steps_k[layer][i], rep.steps_v[layer][i], rep.qs[layer][qi],
                              out=o, workspace=ws, mode=amode)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    nvtx = Nvtx(torch)       # phase ranges for profilers (no per-layer markers in the timed loops)

    # ---- the timed loop: W_ warm-up steps, then K steps, each through every layer
    n = W_ + K
    e_step = [(ev(), ev()) for _ in range(n)]
    barrier()
    nvtx.push("kv4 timed steps")
    for i in range(n):
        if i == W_:
            barrier()
            t_window = time.perf_counter()
        flush.fill_(i & 0xFF)                   # evict the previous step's KV from L2 (outside the events)
        e_step[i][0].record(stream)
        for layer in range(layers):
            layer_step(layer, i, i)
        e_step[i][1].record(stream)
    clocks.sample_now(4, 0.0003)                # while the queued steps run
    barrier()
    nvtx.pop()
    clocks.window(t_window, time.perf_counter())
    t_step = sum(e_step[i][0].elapsed_time(e_step[i][1]) for i in range(W_, n)) / 1e3
    bytes_timed = sum(rep.bytes_at(i + 1) * layers for i in range(W_, n))

    # ---- the same steps on the next K tokens with the library's events around every layer's attention and
    # merge kernels (the roofline's kernel time); kept out of the loop above because an event marker between
    # two launches adds about 2 us to a layer
    e_kern = [[(ev(), ev()) for _ in range(layers)] for _ in range(K)]
    e_kstep = [(ev(), ev()) for _ in range(K)]   # the steps of this pass, for the time outside the kernels
    nvtx.push("kv4 steps with kernel events")
    t_window = time.perf_counter()
    for j in range(K):
        flush.fill_(j & 0xFF)
        e_kstep[j][0].record(stream)
        for layer in range(layers):
            kv4.kv4_set_attention_events(cache.handle, *e_kern[j][layer])
            layer_step(layer, n + j, W_ + j)
        e_kstep[j][1].record(stream)
    clocks.sample_now(4, 0.0003)
    barrier()
    nvtx.pop()
    clocks.window(t_window, time.perf_counter())
    kv4.kv4_set_attention_events(cache.handle, None, None)
    t_kern = sum(a.elapsed_time(b) for row in e_kern for a, b in row) / 1e3
    t_kstep = sum(a.elapsed_time(b) for a, b in e_kstep) / 1e3
    bytes_kern = sum(rep.bytes_at(n + j + 1) * layers for j in range(K))
    used = n + K                                 # new tokens used so far

    # ---- e2e through the public API with host buffers: each step copies every layer's new K, V and q from
    # pinned host memory (one transfer per layer, on a copy stream, ahead of the layer that reads it) and every
    # layer's output back to pinned host memory (on a second copy stream, behind the layer that writes it).
    # The device staging buffers are doubled (step parity), so the copies of step j+1 overlap step j.
    e2e = None
    if K_e2e:
        kv_el, q_el = B * Hkv * D, B * Hq * D
        per = 2 * kv_el + q_el
        hin = torch.empty((K_e2e, layers, per), dtype=torch.bfloat16).pin_memory()
        for j in range(K_e2e):
            for layer in range(layers):
                hin[j, layer, :kv_el].copy_(rep.steps_k[layer][used + j].reshape(-1))
                hin[j, layer, kv_el:2 * kv_el].copy_(rep.steps_v[layer][used + j].reshape(-1))
                hin[j, layer, 2 * kv_el:].copy_(rep.qs[layer][j % (W_ + K)].reshape(-1))
        hout = torch.empty((K_e2e, layers, B, Hq, D), dtype=torch.bfloat16).pin_memory()
        din = torch.empty((2, layers, per), dtype=torch.bfloat16, device=device)
        dout = torch.empty((2, layers, B, Hq, D), dtype=torch.bfloat16, device=device)
        h2d, d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ready = [[torch.cuda.Event() for _ in range(layers)] for _ in range(2)]
        consumed = [[torch.cuda.Event() for _ in range(layers)] for _ in range(2)]
        written = [[torch.cuda.Event() for _ in range(layers)] for _ in range(2)]
        drained = [[torch.cuda.Event() for _ in range(layers)] for _ in range(2)]
        e0, e1 = ev(), ev()
        barrier()
        nvtx.push("kv4 e2e steps")
        e0.record(stream)
        h2d.wait_event(e0)
        d2h.wait_event(e0)
        for j in range(K_e2e):
            b = j & 1                                        # staging slot of this step
            for layer in range(layers):
                with torch.cuda.stream(h2d):
                    if j >= 2:
                        h2d.wait_event(consumed[b][layer])   # step j-2 has read this slot of the layer
                    din[b, layer].copy_(hin[j, layer], non_blocking=True)
                    ready[b][layer].record(h2d)
            for layer in range(layers):
                stream.wait_event(ready[b][layer])
                if j >= 2:
                    stream.wait_event(drained[b][layer])     # step j-2's output of the layer is on the host
                dk = din[b, layer, :kv_el].view(B, Hkv, D)
                dv = din[b, layer, kv_el:2 * kv_el].view(B, Hkv, D)
                dq = din[b, layer, 2 * kv_el:].view(B, Hq, D)
                if two:
                    cache.append(layer, rep.seq_ids, rep.cu_one, dk, dv, total_new=B, rope=rope)
                    cache.attention(layer, rep.seq_ids, dq, out=dout[b, layer], workspace=ws, mode=amode)
                else:
                    cache.decode_step(layer, rep.seq_ids, dk, dv, dq, out=dout[b, layer], workspace=ws, mode=amode)
                consumed[b][layer].record(stream)
                written[b][layer].record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(written[b][layer])
                    hout[j, layer].copy_(dout[b, layer], non_blocking=True)
                    drained[b][layer].record(d2h)
        for b in range(min(2, K_e2e)):
            for layer in range(layers):
                stream.wait_event(drained[b][layer])
        e1.record(stream)
        barrier()
        nvtx.pop()
        t_e2e = e0.elapsed_time(e1) / 1e3
        e2e_bytes = sum(rep.bytes_at(used + j + 1) * layers for j in range(K_e2e))
        e2e = {"t": t_e2e, "bytes": e2e_bytes, "steps": K_e2e, "h2d_bytes_per_step": int(layers * per * 2),
               "d2h_bytes_per_step": int(layers * B * Hq * D * 2)}
        used += K_e2e
        # diagnostic (outside the e2e figure): the same three pieces of a step one after another on one
        # stream, each between its own events -- the copy in, the library calls, the copy out
        nd = min(K_e2e, 5)
        ev3 = [[ev() for _ in range(4)] for _ in range(nd)]
        barrier()
        for j in range(nd):
            flush.fill_(j & 0xFF)
            ev3[j][0].record(stream)
            for layer in range(layers):
                din[0, layer].copy_(hin[j, layer], non_blocking=True)
            ev3[j][1].record(stream)
            for layer in range(layers):
                dk = din[0, layer, :kv_el].view(B, Hkv, D)
                dv = din[0, layer, kv_el:2 * kv_el].view(B, Hkv, D)
                dq = din[0, layer, 2 * kv_el:].view(B, Hq, D)
                cache.decode_step(layer, rep.seq_ids, dk, dv, dq, out=dout[0, layer], workspace=ws, mode=amode)
            ev3[j][2].record(stream)
            for layer in range(layers):
                hout[j, layer].copy_(dout[0, layer], non_blocking=True)
            ev3[j][3].record(stream)
        barrier()
        if nd:
            parts = [sum(ev3[j][i].elapsed_time(ev3[j][i + 1]) for j in range(nd)) / nd * 1e3 for i in range(3)]
            e2e["breakdown_us"] = {"h2d": round(parts[0], 2), "step": round(parts[1], 2), "d2h": round(parts[2], 2),
                                   "serial_sum": round(sum(parts), 2),
                                   "how": "%d steps with the three pieces serialised on one stream, each between "
                                          "its own CUDA events (not the e2e figure, which overlaps them)" % nd}
        used += nd
        del hin, hout, din, dout

    res = {"rep": rep, "setup_s": setup_s, "t_step": t_step, "bytes_timed": bytes_timed, "t_kern": t_kern,
           "t_kstep": t_kstep,
           "bytes_kern": bytes_kern, "e2e": e2e, "status": cache.status(), "used": used, "ws": ws, "out": out,
           "flush": flush}
    if do_cmp:
        res["compare"] = compare_int4_legs(torch, kv4, res, K)
    return res


def time_passes(torch, fn, K, layers, flush, q_of):
    """Attention-only passes over `layers` layers: 3 warm-up passes, then K passes with one event pair per
    layer call.  Returns the mean time of one call of each layer (s)."""
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for i in range(3):
        for layer in range(layers):
            fn(layer, q_of(layer, i))
    torch.cuda.synchronize()
    es = [[(ev(), ev()) for _ in range(layers)] for _ in range(K)]
    for i in range(K):
        flush.fill_(i & 0xFF)
        for layer in range(layers):
            es[i][layer][0].record()
            fn(layer, q_of(layer, i))
            es[i][layer][1].record()
    torch.cuda.synchronize()
    return [sum(es[i][layer][0].elapsed_time(es[i][layer][1]) for i in range(K)) / 1e3 / K for layer in range(layers)]


def compare_int4_legs(torch, kv4, res, K):
    """On the INT4 cache of `res`: the step as two calls against one call, attention alone in the protected and
    the INT4-only modes, and multi-token queries (attention-only figures are per layer call, summed over the
    layers)."""
    rep, ws, out, flush = res["rep"], res["ws"], res["out"], res["flush"]
    w, cache, layers, B = rep.w, rep.cache, rep.layers, rep.B
    Hkv, D = w["Hkv"], w["D"]
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    nq = rep.qs[0].shape[0]

    def time_steps(fn, t0):
        es = [(ev(), ev()) for _ in range(K)]
        for i in range(K):
            flush.fill_(i & 0xFF)
            es[i][0].record()
            for layer in range(layers):
                fn(layer, t0 + i, i % nq)
            es[i][1].record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in es) / 1e3 / K

    def two_calls(layer, i, qi):
        cache.append(layer, rep.seq_ids, rep.cu_one, rep.steps_k[layer][i], rep.steps_v[layer][i], total_new=B)
        cache.attention(layer, rep.seq_ids, rep.qs[layer][qi], out=out, workspace=ws)

    def one_call(layer, i, qi):
        cache.decode_step(layer, rep.seq_ids, rep.steps_k[layer][i], rep.steps_v[layer][i], rep.qs[layer][qi],
                          out=out, workspace=ws)

    used = res["used"]
    t_two = time_steps(two_calls, used)
    t_one = time_steps(one_call, used + K)
    used += 2 * K
    res["used"] = used
    q_of = lambda layer, i: rep.qs[layer][i % nq]  # noqa: E731
    per_int4 = time_passes(torch, lambda l, q: cache.attention(l, rep.seq_ids, q, out=out, workspace=ws), K, layers,
                           flush, q_of)
    per_only = time_passes(torch, lambda l, q: cache.attention(l, rep.seq_ids, q, out=out, workspace=ws,
                                                              mode=kv4.KV4_MODE_INT4_ONLY), K, layers, flush, q_of)
    b_prot, b_only = rep.bytes_at(used), rep.bytes_at(used, int4_only=True)
    t_int4, t_only = sum(per_int4), sum(per_only)
    cmp = {"step_as_two_calls": {"ms_per_step": round(t_two * 1e3, 4)},
           "step_as_one_call": {"ms_per_step": round(t_one * 1e3, 4)},
           "int4_protected": {"attention_ms": round(t_int4 * 1e3, 4), "layers": layers,
                              "kv_gbs": round(b_prot * layers / t_int4 / 1e9, 1)},
           "int4_only": {"attention_ms": round(t_only * 1e3, 4), "layers": layers,
                         "kv_gbs": round(b_only * layers / t_only / 1e9, 1)}}
    # multi-token query (speculative verification): the most query tokens whose heads fit one 8-column operand
    T = 8 // (w["Hq"] // Hkv)
    if T >= 2:
        gen = torch.Generator(device=rep.device).manual_seed(4242)
        qx = [torch.randn((B, T, w["Hq"], D), generator=gen, device=rep.device).to(torch.bfloat16) for _ in range(3)]
        outx = torch.empty((B, T, w["Hq"], D), dtype=torch.bfloat16, device=rep.device)
        wsx = cache.extend_workspace(B, T)
        per_ext = time_passes(torch, lambda l, q: cache.extend_attention(l, rep.seq_ids, q, out=outx, workspace=wsx),
                              K, layers, flush, lambda layer, i: qx[i % 3])
        t_ext = sum(per_ext)
        cmp["extend"] = {"q_len": T, "attention_ms": round(t_ext * 1e3, 4),
                         "kv_gbs": round(b_prot * layers / t_ext / 1e9, 1),
                         "query_tokens_per_s": round(B * T * layers / t_ext, 1)}
        del outx, wsx
    res["per_layer_int4_s"] = per_int4
    return cmp


def bf16_leg(torch, kv4, w, L, extra, used, layers_avail, per_layer_int4, K, device, flush):
    """The BF16-KV kernel on the same seeded tokens as the INT4 cache (positions 0 .. L_b - 2 + used of every
    sequence, drawn as the INT4 replica drew them), on as many of the first layers as fit in the free device
    memory (at most BF16_MAX_LAYERS); compared with the INT4 attention time of the same layers."""
    L_now = L - 1 + used
    need_layer = bf16_bytes(L_now, w["Hkv"], w["D"]) * 1.06
    free = torch.cuda.mem_get_info(device)[0]
    n = int(min(layers_avail, BF16_MAX_LAYERS, (free * 0.9 - 4e9) // need_layer))
    if n < 1:
        return {"skipped": "a BF16 layer cache of %.1f GB does not fit (%.1f GB free)" % (need_layer / 1e9, free / 1e9)}
    B = len(L_now)
    table, num_pages, mpps = workloads.block_table(w, L_now + 1, extra_tokens=0)
    cfg = workloads.cache_config(w, num_pages, mpps, layers=n)
    cache16 = kv4.BF16Cache(cfg, torch.from_numpy(table), device)
    for layer in range(n):   # identical tokens: the same per-(layer, sequence) streams up to the current length
        populate(torch, w, L, cache16.append, layer, extra, device, upto=used)
    ids = torch.arange(B, dtype=torch.int32, device=device)
    ws16 = cache16.workspace(B)
    out = torch.empty((B, w["Hq"], w["D"]), dtype=torch.bfloat16, device=device)
    qs = [workloads.queries(w, 0, 5000 + i, device=device) for i in range(3)]
    per = time_passes(torch, lambda l, q: cache16.attention(l, ids, q, out=out, workspace=ws16), K, n, flush,
                      lambda layer, i: qs[i % 3])
    t16, t4 = sum(per), sum(per_layer_int4[:n])
    b16 = bf16_bytes(L_now, w["Hkv"], w["D"]) * n
    res = {"attention_ms": round(t16 * 1e3, 4), "layers": n, "kv_gbs": round(b16 / t16 / 1e9, 1),
           "int4_protected_attention_ms_same_layers": round(t4 * 1e3, 4),
           "speedup_int4_protected_vs_bf16": round(t16 / t4, 3)}
    if n < layers_avail:
        res["note"] = ("%d of %d layer caches: the BF16 caches of all layers (%.0f GB) do not fit in HBM; the "
                       "INT4 time is that of the same %d layers" % (n, layers_avail, need_layer * layers_avail / 1e9, n))
    cache16.close()
    del cache16, ws16, out
    torch.cuda.empty_cache()
    return res


def format_leg(torch, kv4, fmt, w, L, extra, used, layers_avail, per_layer_int4, K, device, flush):
    """An alternative page format (NVFP4: the "KV Cache Quantization" topic page, item 3; INT2: its item 2) on
    the same seeded tokens as the INT4 cache, at the same lengths, on as many of the first layers as fit (at
    most BF16_MAX_LAYERS): decode attention in the protected mode, against the INT4 attention time of those
    layers."""
    L_now = L - 1 + used
    need_layer = kv_bytes(L_now, w["Hkv"], w["D"], w["S"], w["W"], fmt=fmt) * 1.08
    free = torch.cuda.mem_get_info(device)[0]
    n = int(min(layers_avail, BF16_MAX_LAYERS, (free * 0.9 - 4e9) // need_layer))
    if n < 1:
        return {"skipped": "a layer cache of %.1f GB does not fit (%.1f GB free)" % (need_layer / 1e9, free / 1e9)}
    B = len(L_now)
    table, num_pages, mpps = workloads.block_table(w, L_now + 1, extra_tokens=0)
    cfg = workloads.cache_config(w, num_pages, mpps, layers=n, page_format=fmt)
    cache = kv4.KV4Cache(cfg, torch.from_numpy(table), device)
    for layer in range(n):
        populate(torch, w, L, cache.append, layer, extra, device, upto=used)
    ids = torch.arange(B, dtype=torch.int32, device=device)
    ws = cache.workspace(B)
    out = torch.empty((B, w["Hq"], w["D"]), dtype=torch.bfloat16, device=device)
    qs = [workloads.queries(w, 0, 6000 + i, device=device) for i in range(3)]
    per = time_passes(torch, lambda l, q: cache.attention(l, ids, q, out=out, workspace=ws), K, n, flush,
                      lambda layer, i: qs[i % 3])
    status = cache.status()
    tf, t4 = sum(per), sum(per_layer_int4[:n])
    bf = kv_bytes(L_now, w["Hkv"], w["D"], w["S"], w["W"], fmt=fmt) * n
    res = {"attention_ms": round(tf * 1e3, 4), "layers": n, "kv_gbs": round(bf / tf / 1e9, 1),
           "kv_bytes_vs_int4": round(bf / (kv_bytes(L_now, w["Hkv"], w["D"], w["S"], w["W"]) * n), 4),
           "int4_protected_attention_ms_same_layers": round(t4 * 1e3, 4), "time_vs_int4": round(tf / t4, 3),
           "device_status": status}
    if n < layers_avail:
        res["note"] = "%d of %d layers (the caches of the INT4 run are freed first)" % (n, layers_avail)
    cache.close()
    del cache, ws, out
    torch.cuda.empty_cache()
    return res


def roofline_obj(achieved, hbm, peak_kind, traffic, bytes_per_launch, layers):
    return {"bound": "hbm", "achieved": round(achieved, 2), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "traffic": traffic,
            "kernel": "gattn_kernel: persistent stream-K attention over the INT4 pages and the INT8 store (the "
                      "events span it and the merge kernel, its programmatic dependent; with --two-calls also the "
                      "query-operand kernel before it)",
            "peak_source": peak_kind, "bytes_per_launch": int(bytes_per_launch),
            "launches_per_step": layers,
            "timing": "CUDA events recorded by the library around the kernels of every layer, over K steps that "
                      "follow the timed loop on the same workload"}


def sub_line(torch, kv4, name, args, device, clocks, hbm, peak_kind):
    """A single-layer workload: its step throughput, roofline fraction, INT4-only and BF16 comparisons."""
    w = workloads.workload(name)
    K = max(3, min(args.sub_steps, args.steps))
    r = measure(torch, kv4, w, 1, args, K, 3, device, clocks)
    rep = r["rep"]
    value = r["bytes_timed"] / r["t_step"] / 1e9
    achieved = r["bytes_kern"] / r["t_kern"] / 1e9
    line = {"value": round(value, 2), "unit": "GB/s", "ms_per_step": round(r["t_step"] / K * 1e3, 4),
            "tokens_per_s": round(rep.B * K / r["t_step"], 1), "steps": K,
            "config": {"batch": rep.B, "context": "%s" % (w["ctx"][0],), "page": w["P"], "recent_window": w["W"],
                       "kv_bytes_per_step_mb": round(r["bytes_timed"] / K / 1e6, 1),
                       "side_bytes_per_step": side_bytes(rep.L + 3, w, 1)},
            "roofline": roofline_obj(achieved, hbm, peak_kind, profiled_traffic(name), r["bytes_kern"] / K, 1),
            "device_status": r["status"]}
    if r["e2e"]:
        e = r["e2e"]
        line["e2e"] = {"value": round(e["bytes"] / e["t"] / 1e9, 2), "unit": "GB/s",
                       "h2d_bytes_per_step": e["h2d_bytes_per_step"], "d2h_bytes_per_step": e["d2h_bytes_per_step"],
                       "ms_per_step": round(e["t"] / e["steps"] * 1e3, 4), "breakdown_us": e.get("breakdown_us")}
    cmp = r.get("compare")
    if cmp:
        line["compare"] = cmp
        L0, extra, used = rep.L, rep.extra, r["used"]
        per = r["per_layer_int4_s"]
        flush = r["flush"]
        rep.cache.close()
        del r, rep
        torch.cuda.empty_cache()
        b16 = bf16_leg(torch, kv4, w, L0, extra, used, 1, per, K, device, flush)
        line["compare"]["bf16_kv"] = b16
        for key, fmt in (("nvfp4", kv4.KV4_FORMAT_NVFP4), ("int2", kv4.KV4_FORMAT_INT2)):
            line["compare"][key] = format_leg(torch, kv4, fmt, w, L0, extra, used, 1, per, K, device, flush)
        if "speedup_int4_protected_vs_bf16" in b16:
            line["speedup_int4_protected_vs_bf16"] = b16["speedup_int4_protected_vs_bf16"]
    return line


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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=900), device_id=device)

    W_, K = args.warmup, args.steps
    w = workloads.workload(args.workload)
    if rank > 0:
        w = workloads.workload(args.workload, seed=w["seed"] + 7919 * rank)   # independent sequences per rank
    layers = w["layers"] if args.layers <= 0 else min(args.layers, w["layers"])
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))

    with ClockSampler(device) as clocks:
        r = measure(torch, kv4, w, layers, args, K, W_, device, clocks, world=world, compare=True)
        rep = r["rep"]
        e2e = r["e2e"]
        t_e2e = e2e["t"] if e2e else float("nan")
        e2e_bytes = e2e["bytes"] if e2e else 0.0
        (t_step_all, t_e2e_all), (bytes_all, e2e_bytes_all) = reduce_over_ranks(
            [r["t_step"], t_e2e], [float(r["bytes_timed"]), float(e2e_bytes)], device, world)
        clk = clocks.summary()
        result = None
        if rank == 0:
            B = rep.B
            achieved = r["bytes_kern"] / r["t_kern"] / 1e9
            value = bytes_all / t_step_all / 1e9
            launches = (4 if args.two_calls else 3) * layers
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
                "dtype": "int4/int8 codes, fp16 scales, bf16 q/out, int8 and fp16 tensor-core operands, "
                         "fp32 accumulate",
                "data": "synthetic (seeded N(0,1) K/V with outlier K channels and a large-norm sink, bf16)",
                "config": {"workload": args.workload, "layers": layers, "batch": B, "q_heads": w["Hq"],
                           "kv_heads": w["Hkv"], "head_dim": w["D"], "page": w["P"], "hadamard_block": w["Bh"],
                           "sinks": w["S"], "recent_window": w["W"],
                           "context": "%s, mean %.0f at the first timed step" % (w["ctx"][0], float(np.mean(rep.L + W_))),
                           "step": "%d layers x one %s call (append one token per sequence, then attention)"
                                   % (layers, "two-call" if args.two_calls else "kv4_decode_step"),
                           "kv_bytes_per_step_mb": round(r["bytes_timed"] / K / 1e6, 1),
                           "side_bytes_per_step": side_bytes(rep.L + W_, w, layers),
                           "l2": "flushed before every step by a 256 MB write outside the timed events; each "
                                 "layer's KV also exceeds the 126 MB L2",
                           "parallelism": "replica per GPU" if world > 1 else "single GPU",
                           "rope": ("neox, rotary dim %d, base 1e6, fused into the append and query kernels" % w["D"]
                                    if args.rope else "none (keys arrive post-RoPE)")},
                "tokens_per_s": round(B * world * K / t_step_all, 1),
                "hbm_frac_of_%s" % peak_kind: round(value / hbm, 4),
                "attention_kv_gbs": round(achieved, 2),
                "api": ("two calls per layer: kv4_rotate_quantize_append + kv4_decode_attention" if args.two_calls
                        else "one call per layer: kv4_decode_step"),
                # step time outside the attention and merge kernels, all layers (append + query operands), from
                # the pass with the kernel events (its steps and its kernels under the same markers and clocks)
                ("append_us_per_step" if args.two_calls else "append_and_query_us_per_step"):
                    round(max(r["t_kstep"] - r["t_kern"], 0.0) / K * 1e6, 2),
                "roofline": roofline_obj(achieved, hbm, peak_kind, profiled_traffic(args.workload),
                                         r["bytes_kern"] / (K * layers), layers),
                "e2e": ({"value": round(e2e_bytes_all / t_e2e_all / 1e9, 2), "unit": "GB/s",
                         "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                         "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                         "tokens_per_s": round(B * world * e2e["steps"] / t_e2e_all, 1),
                         "ms_per_step": round(t_e2e_all / e2e["steps"] * 1e3, 4),
                         "breakdown_us": e2e.get("breakdown_us"),
                         "how": "per layer: new K, V and q copied from pinned host memory on a copy stream ahead "
                                "of the layer, the layer's output copied to pinned host memory on a second copy "
                                "stream behind it, device staging doubled so the copies of a step overlap the "
                                "previous step; one CUDA-event pair around all steps"} if e2e else None),
                # per layer: gstep_kernel, gattn_kernel, gmerge_kernel (two calls: append, gq, gattn, gmerge)
                "gpu_launches": launches * K,
                "clocks": clk,
                "device_status": r["status"],
                "setup_s": round(r["setup_s"], 1),
                "gpu": torch.cuda.get_device_name(device),
                "kernel_source_digest": kernel_source_hash(),
            }
            if "compare" in r:
                result["compare"] = r["compare"]
        cmp_ok = "compare" in r
        L0, extra, used = rep.L, rep.extra, r["used"]
        per = r.get("per_layer_int4_s")
        flush = r["flush"]
        rep.cache.close()
        del r, rep
        torch.cuda.empty_cache()
        if rank == 0 and cmp_ok:
            result["compare"]["bf16_kv"] = bf16_leg(torch, kv4, w, L0, extra, used, layers, per, K, device, flush)
            for key, fmt in (("nvfp4", kv4.KV4_FORMAT_NVFP4), ("int2", kv4.KV4_FORMAT_INT2)):
                result["compare"][key] = format_leg(torch, kv4, fmt, w, L0, extra, used, layers, per, K, device, flush)
        if (rank == 0 and world == 1 and not args.kernel_only and not args.no_sublines and not args.rope
                and args.workload not in SUBLINES):
            subs = {}
            for name in SUBLINES:
                subs[name] = sub_line(torch, kv4, name, args, device, clocks, hbm, peak_kind)
                torch.cuda.empty_cache()
            result["workloads"] = subs
        del flush
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# --------------------------------------------------------------------------- CPU oracle

def _oracle_proc(w, seq, steps, warm, rope, barrier, results):
    """One process of the CPU sample: the oracle on sequence `seq` of layer 0 of `w`: populate (untimed), wait
    for every process, then `warm` + `steps` decode steps (append one token, attend), timed with the
    system-wide monotonic clock.  Numpy only, one BLAS thread."""
    try:
        from threadpoolctl import threadpool_limits
        from oracle import OracleKV4Cache, decode_attention, ROPE_NEOX
        with threadpool_limits(1):
            L = int(workloads.context_lengths(w)[seq])
            n_steps = steps + warm
            one = dict(w, batch=1)
            table, num_pages, mpps = workloads.block_table(one, [L], extra_tokens=n_steps + 1)
            cfg = workloads.cache_config(w, num_pages, mpps, max_seqs=1, layers=1)
            orc = OracleKV4Cache(cfg, table)
            rp = (workloads.rope_cos_sin(L + n_steps + 1, w["D"]), w["D"], ROPE_NEOX) if rope else None
            k, v = workloads.kv_sequence_np(w, 0, seq, L - 1 + n_steps)
            orc.append(0, [0], [0, L - 1], k[:L - 1], v[:L - 1], rope=rp)
            barrier.wait(timeout=600)
            times, nbytes = [], 0
            for i in range(n_steps):
                q = workloads.queries_np(w, 0, i, n=1)
                t0 = time.perf_counter()
                orc.append(0, [0], [0, 1], k[L - 1 + i:L + i], v[L - 1 + i:L + i], rope=rp)
                decode_attention(orc, 0, [0], q, rope=rp)
                t1 = time.perf_counter()
                if i >= warm:
                    times.append((t0, t1))
                    nbytes += kv_bytes([L + i], w["Hkv"], w["D"], w["S"], w["W"])
            results.put((seq, times, nbytes, L))
    except Exception as e:   # reported by the parent
        results.put((seq, None, repr(e), 0))


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def oracle_sample(w, procs, steps, warm, rope=False):
    """The oracle on `procs` sequences of the workload's layer 0 at once, one process per sequence (spawned:
    no fork of a process that holds a CUDA context).  Returns (GB/s over the timed window, per-step wall times,
    mean context, processes)."""
    import multiprocessing as mp
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    ctx = mp.get_context("spawn")
    B = w["batch"]
    seqs = [int(s) for s in np.linspace(0, B - 1, procs).round().astype(int)] if procs <= B else \
        [s % B for s in range(procs)]
    barrier = ctx.Barrier(len(seqs))
    results = ctx.Queue()
    ps = [ctx.Process(target=_oracle_proc, args=(w, s, steps, warm, rope, barrier, results)) for s in seqs]
    for p in ps:
        p.start()
    got = [results.get(timeout=1800) for _ in ps]
    for p in ps:
        p.join(timeout=60)
    bad = [g for g in got if g[1] is None]
    if bad:
        raise RuntimeError("oracle process failed: %s" % (bad[0][2],))
    t0 = min(t[0] for g in got for t in g[1])
    t1 = max(t[1] for g in got for t in g[1])
    nbytes = sum(g[2] for g in got)
    # wall time of step i: from the first start to the last end of step i over the processes
    per_step = [max(g[1][i][1] for g in got) - min(g[1][i][0] for g in got) for i in range(steps)]
    return nbytes / (t1 - t0) / 1e9, per_step, float(np.mean([g[3] for g in got])), len(seqs)


def cpu_baseline(w, args):
    procs = args.cpu_procs or host_cores()
    gbs, per_step, mean_l, n = oracle_sample(w, procs, args.cpu_steps, 1, rope=args.rope)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": n, "kind": "oracle",
            "host_cores": host_cores(),
            "sample": "%d sequences of layer 0 (mean context %.0f), one per process, %d decode steps each (append "
                      "+ attention) after one warm-up step, numpy with one BLAS thread per process; K/V and q drawn "
                      "with numpy's generator from the workload's recipe; %.2f s per step over all processes"
                      % (n, mean_l, args.cpu_steps, float(np.mean(per_step)))}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    w = workloads.workload(args.workload)
    procs = args.cpu_procs or host_cores()
    gbs, per_step, mean_l, n = oracle_sample(w, procs, args.steps, args.warmup, rope=args.rope)
    t = sum(per_step)
    base = {"value": round(gbs, 4), "unit": "GB/s", "cores": n, "kind": "oracle", "host_cores": host_cores(),
            "sample": "%d sequences of layer 0 (mean context %.0f) per step, one per process, numpy with one BLAS "
                      "thread per process" % (n, mean_l)}
    return {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 attention, f32 codes",
            "data": "synthetic", "config": {"workload": args.workload, "batch_sample": n,
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
            res["cpu_baseline"] = cpu_baseline(workloads.workload(args.workload), args)
        print(json.dumps(res))


if __name__ == "__main__":
    main()
