"""A CPU model of how pass C stages a unit's prefix at head dim 32
(``pass_c_tc<32>`` in lcla_tc.cuh) and of its warp layout.

The table producer copies the quad's prefix states into the prefix buffer the
unit will use: head j's S (32 rows c of 32 fp32, 128 B each) at 4096 j, so raw
row m = 32 j + c sits at bytes [128 m, 128 m + 128).  The prologue converts
it in place into the MMA's A operand: row m as [P~hi 32 | P~lo 32] fp16 with
the 128-byte swizzle (16-byte chunk c of row m at c ^ (m & 7)).  Thread
(m = ptt >> 2, quarter qq = ptt & 3), ptt = (prologue thread) + 384 rep, reads
raw bytes [128 m + 32 qq, + 32) and writes hi to chunk qq and lo to chunk
4 + qq of the same row.

Checked: every (row, quarter) is converted exactly once; a row's four threads
are lanes of one warp, so the warp's lanes can all read before any writes; a
row's writes stay inside the 128 bytes it occupied raw; no two warps touch the
same row; and the warpgroup register split adds up (the prologue's three
warpgroups take no more registers than the epilogue's two and the producers'
one give up, launched at 80 a thread).  No GPU."""

NPC = 12           # prologue warps at d = 32 (three groups of four)
ROWS, QUARTERS = 128, 4


def staging_tasks():
    """(warp, lane, rep) -> (m, qq) for every task the staging loop runs."""
    tasks = {}
    for pw in range(NPC):
        for lane in range(32):
            pt = 32 * pw + lane
            rep = 0
            while 32 * NPC * rep < ROWS * QUARTERS:
                ptt = pt + 32 * NPC * rep
                if ptt >= ROWS * QUARTERS:   # the kernel leaves the loop for whole warps
                    break
                tasks[(pw, lane, rep)] = (ptt >> 2, ptt & 3)
                rep += 1
    return tasks


def chunk_bytes(m, c):
    return set(range(128 * m + 16 * (c ^ (m & 7)), 128 * m + 16 * (c ^ (m & 7)) + 16))


def test_every_row_quarter_converted_once():
    seen = {}
    for key, mq in staging_tasks().items():
        assert mq not in seen, (mq, seen[mq], key)
        seen[mq] = key
    assert sorted(seen) == [(m, q) for m in range(ROWS) for q in range(QUARTERS)]


def test_whole_warps_leave_the_staging_loop_together():
    tasks = staging_tasks()
    for pw in range(NPC):
        for rep in range(3):
            lanes = [lane for lane in range(32) if (pw, lane, rep) in tasks]
            assert lanes in ([], list(range(32))), (pw, rep, lanes)


def test_a_rows_four_threads_are_one_warp_and_rows_do_not_cross_warps():
    owner = {}
    for (pw, lane, rep), (m, qq) in staging_tasks().items():
        assert owner.setdefault(m, (pw, rep)) == (pw, rep), (m, owner[m], (pw, rep))


def test_in_place_writes_stay_within_the_raw_row():
    written = set()
    for (pw, lane, rep), (m, qq) in staging_tasks().items():
        read = set(range(128 * m + 32 * qq, 128 * m + 32 * qq + 32))
        assert read <= set(range(128 * m, 128 * m + 128))
        w = chunk_bytes(m, qq) | chunk_bytes(m, 4 + qq)
        assert w <= set(range(128 * m, 128 * m + 128))
        assert not (w & written)
        written |= w
    assert written == set(range(ROWS * 128))


def test_register_split_adds_up():
    launch, pro, epi, low = 80, 96, 72, 40
    warps = {"epilogue": 8, "prologue": NPC, "producers": 4}
    assert sum(warps.values()) * 32 * launch <= 65536   # 768 threads at the launch limit
    given = 32 * (warps["epilogue"] * (launch - epi) + warps["producers"] * (launch - low))
    taken = 32 * warps["prologue"] * (pro - launch)
    assert taken <= given
    assert all(w % 4 == 0 for w in warps.values())       # whole warpgroups
    for r in (launch, pro, epi, low):
        assert r % 8 == 0 and 24 <= r <= 256
