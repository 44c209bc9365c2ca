"""Host model of the backward kernel's tensor-memory and shared-memory placement
(backward_kernels.cuh, bwd_main_kernel).

Each TMEM lane quarter (32 key rows) has two elementwise warps: part 0 takes a
block's queries [0, 64), part 1 queries [64, 128). Each reads its Sᵀ columns
(column c = query c) 32 at a time and writes the bf16 pairs of Pᵀ over columns
it has already read; the dV product then takes its A operand for the 16
queries of k-step k from TMEM column 8k + 32 (k >= 4). dSᵀ goes to shared
memory as two 64-query halves of 128-byte rows, 16-byte chunks swizzled by
(row & 7). These tests restate that placement and check what the kernel relies
on: no warp overwrites a column the other part still reads, each write follows
the writer's own read of that column, the dV A columns hold exactly the pairs of
their k-step's queries, and the dSᵀ stores of the two parts cover every 16-byte
chunk of the tile exactly once.
"""

QW, CH = 64, 2                      # queries per part, 32-query chunks per part


def p_events(part):
    """(step, kind, columns) of one part's TMEM accesses to the Sᵀ/Pᵀ columns, in order."""
    ev = []
    for cc in range(CH):
        c0 = QW * part + 32 * cc
        ev.append(("read", set(range(c0, c0 + 32))))
        ev.append(("write", set(range(QW * part + 16 * cc, QW * part + 16 * cc + 16))))
    return ev


def p_column(q):
    """TMEM column holding the bf16 pair of query q (pairs (2i, 2i + 1) share one)."""
    part, r = divmod(q, QW)
    return QW * part + r // 2


def dv_a_column(k):
    """First TMEM column of the dV product's A operand for k-step k (as the issuer forms it)."""
    return 8 * k + (QW // 2) * ((16 * k) // QW)


def test_writes_follow_own_reads_and_miss_the_other_part():
    for part in (0, 1):
        seen = set()
        for kind, cols in p_events(part):
            if kind == "read":
                seen |= cols
            else:
                assert cols <= seen, (part, sorted(cols - seen))
        other = set().union(*(c for k, c in p_events(1 - part) if k == "read"))
        written = set().union(*(c for k, c in p_events(part) if k == "write"))
        assert not written & other


def test_pairs_land_where_the_writes_put_them():
    for part in (0, 1):
        for cc in range(CH):
            for i in range(16):                  # pair i of chunk cc
                q = QW * part + 32 * cc + 2 * i
                assert p_column(q) == QW * part + 16 * cc + i
                assert p_column(q + 1) == p_column(q)


def test_dv_a_operand_holds_its_k_step():
    for k in range(8):
        cols = set(range(dv_a_column(k), dv_a_column(k) + 8))
        assert cols == {p_column(q) for q in range(16 * k, 16 * k + 16)}, k


def test_ds_chunks_cover_the_tile_once():
    HALF = 128 * 128
    hits = {}
    for t in range(128):                         # key row = TMEM lane
        for part in (0, 1):
            for cc in range(CH):
                c0 = QW * part + 32 * cc
                for ch in range(4):
                    chunk = 4 * cc + ch
                    addr = part * HALF + t * 128 + ((chunk ^ (t & 7)) * 16)
                    assert addr not in hits
                    hits[addr] = (t, c0 + 8 * ch)
    assert sorted(hits) == list(range(0, 2 * HALF, 16))
    # the unswizzled position of each chunk is (row t, queries c0 + 8 ch ..)
    for addr, (t, q) in hits.items():
        half, rest = divmod(addr, HALF)
        row, off = divmod(rest, 128)
        assert row == t and half == q // 64
        assert ((off // 16) ^ (t & 7)) == (q % 64) // 8
