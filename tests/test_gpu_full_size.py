"""GPU parity at the full sizes of the benchmark workloads, in the launch
configuration the benchmark times (the whole batch in one append call and one
attention call), checked on sampled sequences that the oracle recomputes one by
one: every INT4/INT8 byte those sequences own, and their attention rows.

Workloads (workloads/synth.py): the 64-sequence Qwen3-8B-shaped layer, the
512-sequence async-RL batch (lognormal contexts up to 32768), the long-context
batch (8 x 131072 tokens, page 64, W = 256, drifting K means) and the 36-layer
stack (256 sequences of 4096-16384 tokens; all 36 layer caches are allocated,
layers 0 and 35 are populated and checked)."""

import numpy as np
import pytest
import torch

import workloads
from oracle import OracleKV4Cache, decode_attention
from oracle.layout import tables, scale_offset, TILE
from kvhelpers import check_bf16_out, REL_L2

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _populate(w, cache, layer, lens, keep):
    """Append L_b - 1 tokens of every sequence (batched), return the last token of each
    sequence (for the decode step) and the full K/V of the sequences in `keep` (on the CPU)."""
    B = len(lens)
    last_k, last_v, kept = [], [], {}
    ks, vs, counts, ids, budget = [], [], [], [], 0

    def flush():
        nonlocal ks, vs, counts, ids, budget
        if not ids:
            return
        cu = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32, device="cuda")
        cache.append(layer, torch.tensor(ids, dtype=torch.int32, device="cuda"), cu, torch.cat(ks).contiguous(),
                     torch.cat(vs).contiguous(), total_new=int(sum(counts)))
        ks, vs, counts, ids, budget = [], [], [], [], 0

    for s in range(B):
        L = int(lens[s])
        k, v = workloads.kv_sequence(w, layer, s, L, device="cuda")
        if s in keep:
            kept[s] = (k.cpu(), v.cpu())
        last_k.append(k[L - 1])
        last_v.append(v[L - 1])
        ks.append(k[:L - 1])
        vs.append(v[:L - 1])
        counts.append(L - 1)
        ids.append(s)
        budget += L
        if budget > 4_000_000:
            flush()
    flush()
    return torch.stack(last_k).contiguous(), torch.stack(last_v).contiguous(), kept


def _compare_pages(pool, orc, table, layer, seq, L, D, P):
    """Bytes of every written INT4 position of `seq`: whole tiles where all 16 slots are written."""
    t4 = tables("int4", D)
    ar4 = np.arange(4)
    tiles_per_page = P // TILE
    full_tiles = L // TILE
    bad = 0
    for ti_abs in range(full_tiles):
        page = int(table[seq, (ti_abs * TILE) // P])
        ti = ti_abs % tiles_per_page
        bad += int(np.sum(pool[page, ti] != orc.pages[(layer, page)][ti]))
    for p in range(full_tiles * TILE, L):
        page = int(table[seq, p // P])
        ti, r = (p % P) // TILE, p % TILE
        idx = np.concatenate([t4.k_byte[r], 8 * D + t4.v_byte[r], 16 * D + scale_offset(r, 0) + ar4,
                              16 * D + scale_offset(r, 1) + ar4])
        bad += int(np.sum(pool[page, ti][:, idx] != orc.pages[(layer, page)][ti][:, idx]))
    return bad


def _compare_prot(prot, orc, layer, seq, L, S, W, D):
    t8 = tables("int8", D)
    ar4 = np.arange(4)
    bad = 0
    for slot in range(min(L, S + W)):
        ti, r = slot // TILE, slot % TILE
        idx = np.concatenate([t8.k_byte[r], 16 * D + t8.v_byte[r], 32 * D + scale_offset(r, 0) + ar4,
                              32 * D + scale_offset(r, 1) + ar4])
        bad += int(np.sum(prot[seq, ti][:, idx] != orc.prot[(layer, seq)][ti][:, idx]))
    return bad


def _check_layer(kv4, w, cache, table, cfg, layer, lens, sample):
    B = len(lens)
    last_k, last_v, kept = _populate(w, cache, layer, lens, set(sample))
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    cu_one = torch.arange(B + 1, dtype=torch.int32, device="cuda")
    cache.append(layer, ids, cu_one, last_k, last_v, total_new=B)            # the decode step's append
    q = workloads.queries(w, layer, 0, device="cuda")
    ws = cache.workspace(B)
    out = cache.attention(layer, ids, q, workspace=ws)                        # the whole batch, as timed
    torch.cuda.synchronize()
    assert cache.status() == 0
    D, P, S, W = w["D"], w["P"], w["S"], w["W"]
    lens_now = np.asarray(lens, np.int64)
    assert np.array_equal(cache.seq_lens()[layer].cpu().numpy()[:B], lens_now)
    pool = cache.pages(layer).cpu().numpy()
    prot = cache.protected(layer).cpu().numpy()
    orc = OracleKV4Cache(dict(cfg), table)
    qc = q.float().cpu().numpy()
    for s in sample:
        k, v = kept[s]
        L = int(lens[s])
        kf, vf = k.float().numpy(), v.float().numpy()
        orc.append(layer, [s], [0, L - 1], kf[:L - 1], vf[:L - 1])
        orc.append(layer, [s], [0, 1], kf[L - 1:L], vf[L - 1:L])
        assert _compare_pages(pool, orc, table, layer, s, L, D, P) == 0, ("int4 bytes", s)
        assert _compare_prot(prot, orc, layer, s, L, S, W, D) == 0, ("int8 bytes", s)
        ref = decode_attention(orc, layer, [s], qc[s:s + 1])
        rel, excess = check_bf16_out(out[s:s + 1], ref)
        assert rel <= REL_L2 and excess <= 0, (s, L, rel, excess)
        del orc.pages, orc.prot
        orc = OracleKV4Cache(dict(cfg), table)


def _sample(lens, extra):
    order = np.argsort(lens)
    return sorted({int(order[0]), int(order[-1]), *extra})


@pytest.mark.parametrize("name", ["qwen3_8b_layer", "async_rl", "long_context"])
def test_full_size_workload(kv4, name):
    w = workloads.workload(name)
    lens = workloads.context_lengths(w)
    table, num_pages, mpps = workloads.block_table(w, lens, extra_tokens=1)
    cfg = workloads.cache_config(w, num_pages, mpps)
    cache = kv4.KV4Cache(cfg, torch.from_numpy(table), "cuda")
    sample = _sample(lens, [len(lens) // 2]) if name != "long_context" else [3]
    _check_layer(kv4, w, cache, table, cfg, 0, lens, sample)


def test_full_size_36_layer_stack(kv4):
    w = workloads.workload("stack36")
    lens = workloads.context_lengths(w)
    table, num_pages, mpps = workloads.block_table(w, lens, extra_tokens=1)
    cfg = workloads.cache_config(w, num_pages, mpps)
    need = kv4.kv4_cache_required_bytes(kv4.make_config(**cfg))
    if need > 0.8 * torch.cuda.mem_get_info()[0]:
        pytest.skip("36-layer cache of %.0f GB does not fit this device" % (need / 1e9))
    cache = kv4.KV4Cache(cfg, torch.from_numpy(table), "cuda")
    for layer in (0, 35):
        _check_layer(kv4, w, cache, table, cfg, layer, lens, _sample(lens, [17 + layer]))
