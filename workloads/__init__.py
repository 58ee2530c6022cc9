"""Seeded synthetic workloads for the paged INT4/INT8 KV cache.

This module is shared by the tests, the oracle-side checks and the benchmark.
It holds no arithmetic of the method (no rotation, quantization, placement or
attention): only the shapes and the value distributions of the inputs.

Workloads (one decode layer each unless stated):

* tiny            -- 1 layer, batch 2, 4 q heads / 1 KV head, head_dim 64,
                     contexts 200 and 256 at the first attention call, page 16,
                     Hadamard block 64, S=4 sinks, W=32 recent, 4 decode steps;
                     K, V ~ N(0,1) with 2 outlier K channels x12, K of token 0 x8.
* qwen3_8b_layer  -- batch 64, 32/8 heads (GQA 4), head_dim 128, contexts
                     uniform in [1024, 8192], page 16, block 128, S=4, W=128,
                     4 outlier K channels x15 per KV head, K of token 0 x8, 32 steps.
* async_rl        -- batch 512, contexts lognormal (median 3072, sigma 1.0)
                     clipped to [256, 32768], otherwise as qwen3_8b_layer, 64 steps.
* long_context    -- batch 8, context 131072, page 64, W=256, split into
                     chunks of at most 1024 tokens; K also carries a per-(seq,
                     head, channel) random-walk mean (step sigma 0.01), 8 steps.
* stack36         -- 36 independent layer caches, batch 256, contexts uniform in
                     [4096, 16384], page 16, S=4, W=128, 4 steps.

kv_sequence_np / queries_np draw the same recipe with numpy's generator (other
values, same distributions) for CPU processes that do not load torch.

rope_cos_sin(max_pos, R, base) gives the RoPE angle table that the fused
RoPE append and query kernels take as an input (the model's angles).

A context length L means: the cache is populated with L-1 tokens, then each
decode step appends one token per sequence and attends (so the first attention
call sees L tokens).  Token values are a function of (workload, layer,
sequence, position) only, whatever device generates them is used for both
sides of a comparison (values are copied, never regenerated, across devices).
"""

from .synth import (WORKLOADS, workload, context_lengths, block_table, kv_sequence,  # noqa: F401
                    queries, cache_config, make_seed, rope_cos_sin, kv_sequence_np, queries_np)
