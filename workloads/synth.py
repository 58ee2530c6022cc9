"""Seeded synthetic inputs (no arithmetic of the method lives here).

torch is imported only by the generators that return tensors, so CPU worker
processes that use the numpy generators (kv_sequence_np, queries_np) do not
load it."""

import math

import numpy as np

WORKLOADS = {
    "tiny": dict(index=0, layers=1, batch=2, Hq=4, Hkv=1, D=64, P=16, Bh=64, S=4, W=32,
                 ctx=("fixed", [200, 256]), n_outlier=2, outlier_factor=12.0, sink_factor=8.0,
                 drift_sigma=0.0, steps=4, max_chunk=1024),
    "qwen3_8b_layer": dict(index=1, layers=1, batch=64, Hq=32, Hkv=8, D=128, P=16, Bh=128, S=4, W=128,
                           ctx=("uniform", 1024, 8192), n_outlier=4, outlier_factor=15.0,
                           sink_factor=8.0, drift_sigma=0.0, steps=32, max_chunk=1024),
    "async_rl": dict(index=2, layers=1, batch=512, Hq=32, Hkv=8, D=128, P=16, Bh=128, S=4, W=128,
                     ctx=("lognormal", 3072, 1.0, 256, 32768), n_outlier=4, outlier_factor=15.0,
                     sink_factor=8.0, drift_sigma=0.0, steps=64, max_chunk=1024),
    "long_context": dict(index=3, layers=1, batch=8, Hq=32, Hkv=8, D=128, P=64, Bh=128, S=4, W=256,
                         ctx=("fixed", [131072] * 8), n_outlier=4, outlier_factor=15.0,
                         sink_factor=8.0, drift_sigma=0.01, steps=8, max_chunk=1024),
    "stack36": dict(index=4, layers=36, batch=256, Hq=32, Hkv=8, D=128, P=16, Bh=128, S=4, W=128,
                    ctx=("uniform", 4096, 16384), n_outlier=4, outlier_factor=15.0,
                    sink_factor=8.0, drift_sigma=0.0, steps=4, max_chunk=1024),
}


def workload(name, **overrides):
    w = dict(WORKLOADS[name])
    w["name"] = name
    w.update(overrides)
    w.setdefault("seed", 1000 + w["index"])
    return w


def make_seed(*parts):
    """63-bit seed derived from a tuple of non-negative integers."""
    ss = np.random.SeedSequence([int(p) for p in parts])
    return int(ss.generate_state(2, dtype=np.uint64)[0] & np.uint64(0x7FFFFFFFFFFFFFFF))


def context_lengths(w):
    """Context length per sequence at the first attention call (int64 [batch])."""
    kind = w["ctx"][0]
    rng = np.random.default_rng(make_seed(w["seed"], 1))
    B = w["batch"]
    if kind == "fixed":
        vals = list(w["ctx"][1])
        if len(vals) != B:
            vals = (vals * B)[:B]
        return np.asarray(vals, np.int64)
    if kind == "uniform":
        lo, hi = w["ctx"][1], w["ctx"][2]
        return rng.integers(lo, hi + 1, size=B).astype(np.int64)
    if kind == "lognormal":
        median, sigma, lo, hi = w["ctx"][1:]
        x = np.exp(math.log(median) + sigma * rng.standard_normal(B))
        return np.clip(np.rint(x), lo, hi).astype(np.int64)
    raise ValueError(kind)


def block_table(w, lengths, extra_tokens=None, spare=0.05):
    """Block table for the final lengths (lengths - 1 + steps, or + extra_tokens).

    Pages are a seeded permutation of the pool, handed out in order of need;
    unused entries are -1.  Returns (table int32 [batch, max_pages_per_seq],
    num_pages, max_pages_per_seq).
    """
    P = w["P"]
    extra = w["steps"] - 1 if extra_tokens is None else extra_tokens
    final = np.asarray(lengths, np.int64) + extra
    need = -(-final // P)
    total = int(need.sum())
    num_pages = total + max(1, int(math.ceil(spare * total)))
    max_pages = int(need.max()) if len(need) else 1
    rng = np.random.default_rng(make_seed(w["seed"], 2))
    perm = rng.permutation(num_pages).astype(np.int32)
    table = np.full((len(final), max_pages), -1, np.int32)
    k = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[k:k + n]
        k += n
    return table, num_pages, max_pages


def _outlier_channels(w, layer):
    rng = np.random.default_rng(make_seed(w["seed"], 3, layer))
    return [np.sort(rng.choice(w["D"], size=w["n_outlier"], replace=False)) for _ in range(w["Hkv"])]


def kv_sequence(w, layer, seq, length, device="cpu"):
    """K, V of one sequence, positions [0, length), as bf16 tensors [length, Hkv, D].

    K, V ~ N(0, 1) in fp32; K gets outlier channels (per KV head), the token at
    position 0 multiplied by sink_factor, and optionally a random-walk mean
    along the positions; both are then rounded to bf16.
    """
    import torch
    Hkv, D = w["Hkv"], w["D"]
    g = torch.Generator(device=device)
    g.manual_seed(make_seed(w["seed"], 4, layer, seq))
    k = torch.randn((length, Hkv, D), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((length, Hkv, D), generator=g, device=device, dtype=torch.float32)
    if w["n_outlier"] > 0:
        for h, ch in enumerate(_outlier_channels(w, layer)):
            idx = torch.as_tensor(ch, device=device, dtype=torch.long)
            k[:, h, idx] *= w["outlier_factor"]
    if length > 0 and w["sink_factor"] != 1.0:
        k[0] *= w["sink_factor"]
    if w["drift_sigma"] > 0:
        steps = torch.randn((length, Hkv, D), generator=g, device=device, dtype=torch.float32)
        k += torch.cumsum(steps * w["drift_sigma"], dim=0)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def queries(w, layer, step, n=None, device="cpu"):
    """bf16 queries [batch, Hq, D] ~ N(0, 1) for one decode step."""
    import torch
    B = w["batch"] if n is None else n
    g = torch.Generator(device=device)
    g.manual_seed(make_seed(w["seed"], 5, layer, step))
    return torch.randn((B, w["Hq"], w["D"]), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def _bf16_bits_np(x):
    """fp32 -> bf16 round-to-nearest-even, returned as fp32 values (numpy; finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def kv_sequence_np(w, layer, seq, length):
    """The recipe of kv_sequence drawn with numpy's generator (PCG64, same seed): fp32 arrays of bf16 values
    [length, Hkv, D].  Same shapes and distributions, different values from the torch generators; for CPU
    processes that time the oracle on a sample of a workload."""
    Hkv, D = w["Hkv"], w["D"]
    rng = np.random.default_rng(make_seed(w["seed"], 4, layer, seq))
    k = rng.standard_normal((length, Hkv, D), dtype=np.float32)
    v = rng.standard_normal((length, Hkv, D), dtype=np.float32)
    if w["n_outlier"] > 0:
        for h, ch in enumerate(_outlier_channels(w, layer)):
            k[:, h, ch] *= np.float32(w["outlier_factor"])
    if length > 0 and w["sink_factor"] != 1.0:
        k[0] *= np.float32(w["sink_factor"])
    if w["drift_sigma"] > 0:
        steps = rng.standard_normal((length, Hkv, D), dtype=np.float32)
        k += np.cumsum(steps * np.float32(w["drift_sigma"]), axis=0, dtype=np.float32)
    return _bf16_bits_np(k), _bf16_bits_np(v)


def queries_np(w, layer, step, n=None):
    """The recipe of queries drawn with numpy's generator: fp32 array of bf16 values [n, Hq, D]."""
    B = w["batch"] if n is None else n
    rng = np.random.default_rng(make_seed(w["seed"], 5, layer, step))
    return _bf16_bits_np(rng.standard_normal((B, w["Hq"], w["D"]), dtype=np.float32))


def cache_config(w, num_pages, max_pages_per_seq, max_seqs=None, layers=None, page_format=0):
    """The cache configuration (field names of the C-ABI struct) for a workload."""
    return dict(num_layers=w["layers"] if layers is None else layers,
                max_seqs=w["batch"] if max_seqs is None else max_seqs,
                num_q_heads=w["Hq"], num_kv_heads=w["Hkv"], head_dim=w["D"],
                page_size=w["P"], num_pages=num_pages, max_pages_per_seq=max_pages_per_seq,
                hadamard_block=w["Bh"], sink_tokens=w["S"], recent_window=w["W"], page_format=page_format)


def rope_cos_sin(max_pos, rotary_dim, base=1.0e6):
    """The model's RoPE angle table (an input of the fused append / query kernels):
    fp32 [max_pos][R], row p = cos(p * base^(-2i/R)) for i < R/2, then the sines.
    Angles in fp64, each entry rounded once to fp32 (Qwen3 uses base 1e6)."""
    half = rotary_dim // 2
    inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / rotary_dim)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)
