"""Host-side arithmetic of the multi-token path, checked without a GPU: the
passes of 8 // G query tokens and the operand-column -> (query token, query
head) -> output-row map of each pass cover every output row exactly once, and
each column's last visible position is L - q_len + (its query token).  The
formulas are those of launch_extend_attention (pass split) and q_row (row map)
in the library."""

import itertools

import pytest


def passes(q_len, G):
    chunk = min(q_len, 8 // G)
    return [(q0, min(chunk, q_len - q0)) for q0 in range(0, q_len, chunk)]


def q_row(b, h, c, Gh, qtot, q0, Hq):
    i, g = divmod(c, Gh)
    return (b * qtot + q0 + i) * Hq + h * Gh + g


@pytest.mark.parametrize("G,q_len", list(itertools.product([1, 2, 3, 4, 8], [1, 2, 3, 4, 5, 7, 8, 9])))
def test_passes_cover_every_output_row_once(G, q_len):
    n, Hkv = 3, 4
    Hq = G * Hkv
    seen = []
    for q0, qlen in passes(q_len, G):
        assert 1 <= qlen and qlen * G <= 8                       # one 8-column operand per KV head
        for b, h, c in itertools.product(range(n), range(Hkv), range(qlen * G)):
            seen.append(q_row(b, h, c, G, q_len, q0, Hq))
    assert sorted(seen) == list(range(n * q_len * Hq))


@pytest.mark.parametrize("G,q_len,L", [(4, 4, 10), (8, 3, 2), (1, 9, 100), (2, 5, 5)])
def test_each_column_sees_up_to_its_own_position(G, q_len, L):
    for q0, qlen in passes(q_len, G):
        vis = L - q_len + q0                                      # the kernel's per-pass visibility base
        for c in range(qlen * G):
            token = q0 + c // G
            assert vis + c // G == L - q_len + token              # last position the column's token sees
