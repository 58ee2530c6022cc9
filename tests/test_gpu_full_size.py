"""GPU parity at the full sizes of the benchmark workloads, in the launch
configuration the benchmark times: the whole batch populated by batched
appends, then one kv4_decode_step call (append of the decode token of every
sequence, then attention of the whole batch).  The oracle recomputes each
checked sequence in its own process (one process per host core) from the same
tokens, and the test compares every INT4/INT8 byte the sequence owns (codes,
scales, placement) and its attention rows.

Checked sequences: every sequence of the 64-sequence Qwen3-8B-shaped layer, of
the 512-sequence async-RL batch (lognormal contexts up to 32768) and of the
long-context batch (8 x 131072 tokens, page 64, W = 256, drifting K means);
on the 36-layer stack (256 sequences of 4096-16384 tokens, all 36 layer
caches allocated) 16 seeded sequences, with the shortest and the longest
among them, of each of layers 0, 17 and 35."""

import numpy as np
import pytest
import torch

import workloads
from oracle.layout import tables, scale_offset, TILE
from kvhelpers import check_bf16_out, REL_L2
from oracle_pool import OraclePool

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _bits(t):
    """bf16 tensor -> uint16 numpy bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _populate(w, cache, layer, lens):
    """Append L_b - 1 tokens of every sequence (batched, as the benchmark does); return the decode step's
    token of every sequence (the L_b-th, [B, Hkv, D] K and V)."""
    B = len(lens)
    last_k, last_v = [], []
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
        last_k.append(k[L - 1])
        last_v.append(v[L - 1])
        ks.append(k[:L - 1])
        vs.append(v[:L - 1])
        counts.append(L - 1)
        ids.append(s)
        budget += L
        if budget > 2_000_000:
            flush()
    flush()
    return torch.stack(last_k).contiguous(), torch.stack(last_v).contiguous()


def _page_bad(pool, pages, table, seq, L, D, P, t4):
    """Differing bytes over every written INT4 position of `seq`: whole tiles where all 16 slots are
    written, the written slots of the last tile."""
    ar4 = np.arange(4)
    tiles_per_page = P // TILE
    full_tiles = L // TILE
    bad = 0
    for ti_abs in range(full_tiles):
        page = int(table[seq, (ti_abs * TILE) // P])
        ti = ti_abs % tiles_per_page
        bad += int(np.sum(pool[page, ti] != pages[page][ti]))
    for p in range(full_tiles * TILE, L):
        page = int(table[seq, p // P])
        ti, r = (p % P) // TILE, p % TILE
        idx = np.concatenate([t4.k_byte[r], 8 * D + t4.v_byte[r], 16 * D + scale_offset(r, 0) + ar4,
                              16 * D + scale_offset(r, 1) + ar4])
        bad += int(np.sum(pool[page, ti][:, idx] != pages[page][ti][:, idx]))
    return bad


def _prot_bad(prot, oprot, seq, L, S, W, D, t8):
    ar4 = np.arange(4)
    bad = 0
    for slot in range(min(L, S + W)):
        ti, r = slot // TILE, slot % TILE
        idx = np.concatenate([t8.k_byte[r], 16 * D + t8.v_byte[r], 32 * D + scale_offset(r, 0) + ar4,
                              32 * D + scale_offset(r, 1) + ar4])
        bad += int(np.sum(prot[seq, ti][:, idx] != oprot[ti][:, idx]))
    return bad


def _check_layer(kv4, w, cache, table, cfg, layer, lens, check):
    B = len(lens)
    last_k, last_v = _populate(w, cache, layer, lens)
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    q = workloads.queries(w, layer, 0, device="cuda")
    out = cache.decode_step(layer, ids, last_k, last_v, q, workspace=cache.workspace(B))   # as the bench times it
    torch.cuda.synchronize()
    assert cache.status() == 0
    D, P, S, W = w["D"], w["P"], w["S"], w["W"]
    assert np.array_equal(cache.seq_lens()[layer].cpu().numpy()[:B], np.asarray(lens, np.int64))
    pool = cache.pages(layer).cpu().numpy()
    prot = cache.protected(layer).cpu().numpy()
    out_h = out.cpu()
    qc = q.float().cpu().numpy()
    t4, t8 = tables("int4", D), tables("int8", D)

    def jobs():
        for s in check:
            k, v = workloads.kv_sequence(w, layer, s, int(lens[s]), device="cuda")   # the tokens appended above
            yield layer, s, _bits(k), _bits(v), qc[s]

    seen = set()
    with OraclePool(cfg, table) as pool_o:
        for s, pages, oprot, ref in pool_o.run(jobs()):
            L = int(lens[s])
            assert _page_bad(pool, pages, table, s, L, D, P, t4) == 0, ("int4 bytes", layer, s)
            assert _prot_bad(prot, oprot, s, L, S, W, D, t8) == 0, ("int8 bytes", layer, s)
            rel, excess = check_bf16_out(out_h[s:s + 1], ref)
            assert rel <= REL_L2 and excess <= 0, (layer, s, L, rel, excess)
            seen.add(s)
    assert seen == set(check)


@pytest.mark.parametrize("name", ["qwen3_8b_layer", "async_rl", "long_context"])
def test_full_size_workload_every_sequence(kv4, name):
    w = workloads.workload(name)
    lens = workloads.context_lengths(w)
    table, num_pages, mpps = workloads.block_table(w, lens, extra_tokens=1)
    cfg = workloads.cache_config(w, num_pages, mpps)
    cache = kv4.KV4Cache(cfg, torch.from_numpy(table), "cuda")
    _check_layer(kv4, w, cache, table, cfg, 0, lens, list(range(len(lens))))


def test_full_size_36_layer_stack(kv4):
    w = workloads.workload("stack36")
    lens = workloads.context_lengths(w)
    table, num_pages, mpps = workloads.block_table(w, lens, extra_tokens=1)
    cfg = workloads.cache_config(w, num_pages, mpps)
    need = kv4.kv4_cache_required_bytes(kv4.make_config(**cfg))
    if need > 0.8 * torch.cuda.mem_get_info()[0]:
        pytest.skip("36-layer cache of %.0f GB does not fit this device" % (need / 1e9))
    cache = kv4.KV4Cache(cfg, torch.from_numpy(table), "cuda")
    order = np.argsort(lens)
    for layer in (0, 17, 35):
        rng = np.random.default_rng(workloads.make_seed(w["seed"], 9, layer))
        pick = set(int(x) for x in rng.choice(len(lens), size=14, replace=False))
        pick |= {int(order[0]), int(order[-1])}
        while len(pick) < 16:
            pick.add(int(rng.integers(len(lens))))
        _check_layer(kv4, w, cache, table, cfg, layer, lens, sorted(pick))
