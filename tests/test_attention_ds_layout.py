"""Host-side check of the stored-dS^T hand-over in the attention backward.

The dK/dV kernel writes dS^T in 4 KiB pieces (32 keys x 64 queries; piece
(j, i) holds query block j of 64 and key block i of 32), walking per 128-key
block the 64-query blocks from the causal diagonal on.  The dQ kernel reads,
per 256-query block, each 128-query half's pieces over the 64-key blocks that
half needs.  This restates both kernels' loop bounds and checks, over many
sequence lengths, that every piece the dQ kernel reads for a query block with
a valid query was written, and that all pieces lie inside the S_pad x S_pad
array the workspace holds per head (S_pad = seq rounded up to 128).  Pure
index arithmetic: no GPU.
"""
import pytest


def _cdiv(a, b):
    return (a + b - 1) // b


def written(S, causal):
    out = set()
    for kb in range(_cdiv(S, 128)):             # dK/dV items: 128-key blocks
        i0 = 2 * kb if causal else 0            # first 64-query block at or after the diagonal
        for j in range(i0, _cdiv(S, 64)):
            for quad in range(4):               # the four compute warps' 32-key pieces
                out.add((j, 4 * kb + quad))
    return out


def read(S, causal):
    out = set()
    nkb = _cdiv(S, 64)
    for qb in range(_cdiv(S, 256)):             # dQ items: 256-query blocks
        for half in range(2):
            qs = 256 * qb + 128 * half
            if qs >= S:
                continue
            nk = min(nkb, (qs + 128) // 64) if causal else nkb
            for k in range(nk):
                for c in range(2):
                    for p in range(2):
                        out.add((4 * qb + 2 * half + c, 2 * k + p))
    return out


@pytest.mark.parametrize("causal", [True, False])
def test_every_piece_read_was_written(causal):
    for S in list(range(1, 600)) + [1023, 1024, 1025, 2047, 2048, 2049, 4096]:
        s_pad = _cdiv(S, 128) * 128
        w, r = written(S, causal), read(S, causal)
        for (j, i) in r | w:
            assert 0 <= j < s_pad // 64 and 0 <= i < s_pad // 32, (S, j, i)
        # A piece read for a 64-query block with a valid query was written;
        # blocks wholly past S feed only dq rows that are never stored.
        missing = {(j, i) for (j, i) in r if 64 * j < S and (j, i) not in w}
        assert not missing, (S, sorted(missing)[:5])


def test_causal_reads_stay_on_or_below_the_diagonal():
    # Under the causal mask a half reads no key block that starts after its
    # last query.
    for S in (128, 300, 2048):
        for (j, i) in read(S, True):
            last_query_of_half = 128 * (j // 2) + 127
            assert 32 * i <= last_query_of_half, (S, j, i)
