"""The process pool that runs the oracle per sequence for the full-size GPU
tests: its results (tiles of each sequence, INT8 store, attention row) equal
those of one oracle cache fed the same tokens directly, in one append per
sequence plus the decode token."""

import numpy as np

from oracle import OracleKV4Cache, decode_attention
from oracle_pool import OraclePool


def test_pool_matches_a_direct_oracle_run():
    rng = np.random.default_rng(5)
    cfg = dict(num_layers=2, max_seqs=3, num_q_heads=4, num_kv_heads=2, head_dim=64, page_size=16, num_pages=40,
               max_pages_per_seq=12, hadamard_block=64, sink_tokens=4, recent_window=16)
    table = rng.permutation(40)[:36].reshape(3, 12).astype(np.int32)
    lens = [150, 1, 40]
    toks = {}
    for s, L in enumerate(lens):
        k = (rng.standard_normal((L, 2, 64)) * 2).astype(np.float32)
        v = rng.standard_normal((L, 2, 64)).astype(np.float32)
        # bf16 values and their bit patterns
        kb = (k.view(np.uint32) >> 16).astype(np.uint16)
        vb = (v.view(np.uint32) >> 16).astype(np.uint16)
        toks[s] = (kb, vb, rng.standard_normal((4, 64)).astype(np.float32))
    direct = OracleKV4Cache(cfg, table)
    f32 = lambda b: (b.astype(np.uint32) << 16).view(np.float32)  # noqa: E731
    for s, L in enumerate(lens):
        kb, vb, _ = toks[s]
        direct.append(1, [s], [0, L - 1], f32(kb[:L - 1]), f32(vb[:L - 1]))
        direct.append(1, [s], [0, 1], f32(kb[L - 1:]), f32(vb[L - 1:]))
    with OraclePool(cfg, table, procs=2) as pool:
        got = {s: (pages, prot, ref) for s, pages, prot, ref in
               pool.run(((1, s, toks[s][0], toks[s][1], toks[s][2]) for s in range(3)), batch=2)}
    assert sorted(got) == [0, 1, 2]
    for s, L in enumerate(lens):
        pages, prot, ref = got[s]
        own = {int(table[s, i]) for i in range(-(-L // 16))}
        assert set(pages) == own
        for pg in own:
            assert np.array_equal(pages[pg], direct.pages[(1, pg)])
        assert np.array_equal(prot, direct.prot[(1, s)])
        want = decode_attention(direct, 1, [s], toks[s][2][None])
        assert np.array_equal(ref["out_f64"], want["out_f64"])
        assert np.array_equal(ref["out_bf16"], want["out_bf16"])
