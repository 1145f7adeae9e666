"""A CPU model of the tensor-core prologues' shared-memory index map.

The model restates ``pair_offsets`` of ``lcla_tc.cuh`` (the prologue thread ->
row pair mapping shared by pass A and pass C) and the layouts it works on:

* a stage holds four 8 KB atoms of 64 rows x 128 B with the 128-byte swizzle
  (16-byte chunk c of row r at c ^ (r & 7)); TMA box b (64 tokens x heads
  2b, 2b+1, 64 B each) lands in atom b, so raw chunk j of a row is head 2b's
  quarter j (j < 4) or head 2b+1's quarter j - 4;
* after the prologue, atom a holds head 2(a & 1) + (a >> 1) as [hi 32 | lo 32]
  bf16 per row: hi quarter f in chunk f, lo quarter f in chunk 4 + f;
* a rotary table tile is 64 rows x 64 B with the 64-byte swizzle (chunk c of
  row r at c ^ ((r >> 1) & 3)).

Checked: the 512 prologue threads cover every (row, head pair, quarter) once;
every 16-byte chunk of a stage is written exactly once; a thread overwrites
raw chunks only where it has read them (in place), so no thread's write lands
on another thread's unread input; and every 8-lane phase of each 128-bit
access touches 8 different 16-byte bank groups.  No GPU."""


def pair_offsets(pw, lane):
    f = lane & 3
    g = (lane >> 3) & 1
    pr = ((lane >> 4) << 1) | ((lane >> 2) & 1)
    r = 8 * (pw >> 1) + 2 * (pw & 1) + (pr >> 1) + (pr & 1) * (5 - 2 * (pr >> 1))
    sw = r & 7
    row = r * 128
    return dict(g=g, f=f, r=r,
                in0=g * 8192 + row + ((f ^ sw) << 4),
                in1=g * 8192 + row + (((4 + f) ^ sw) << 4),
                out2=(2 + g) * 8192 + row + ((f ^ sw) << 4),
                out3=(2 + g) * 8192 + row + (((4 + f) ^ sw) << 4),
                tab=r * 64 + ((f ^ ((r >> 1) & 3)) << 4))


NPRO = 16
THREADS = [(pw, lane) for pw in range(NPRO) for lane in range(32)]


def atom_of(h):
    return (h >> 1) + 2 * (h & 1)


def test_threads_cover_every_row_pair_and_quarter_once():
    seen = {}
    for pw, lane in THREADS:
        o = pair_offsets(pw, lane)
        key = (o["r"], o["g"], o["f"])
        assert 0 <= o["r"] < 64
        assert key not in seen, (key, seen.get(key), (pw, lane))
        seen[key] = (pw, lane)
    assert len(seen) == 64 * 2 * 4


def test_every_stage_chunk_written_once_and_in_place():
    written = {}
    for pw, lane in THREADS:
        o = pair_offsets(pw, lane)
        for k in ("in0", "in1", "out2", "out3"):
            off = o[k]
            assert 0 <= off < 4 * 8192 and off % 16 == 0
            assert off not in written, (k, off)
            written[off] = (pw, lane)
    assert len(written) == 4 * 8192 // 16
    # the raw boxes occupy atoms 0 and 1; a thread writes there only the two chunks it read
    for pw, lane in THREADS:
        o = pair_offsets(pw, lane)
        reads = {o["in0"], o["in1"]}
        writes_raw = {off for off in (o["in0"], o["in1"], o["out2"], o["out3"]) if off < 2 * 8192}
        assert writes_raw == reads


def test_raw_chunks_read_are_the_heads_and_quarter_of_the_thread():
    # box g, row r: chunk j < 4 is head 2g's quarter j, chunk 4 + j is head 2g+1's (128-byte swizzle)
    for pw, lane in THREADS:
        o = pair_offsets(pw, lane)
        r, g, f = o["r"], o["g"], o["f"]
        assert o["in0"] == g * 8192 + r * 128 + ((f ^ (r & 7)) << 4)
        assert o["in1"] == g * 8192 + r * 128 + (((4 + f) ^ (r & 7)) << 4)
        # and the operand chunks: head 2g -> atom g (hi f, lo 4+f), head 2g+1 -> atom 2+g
        assert atom_of(2 * g) == g and atom_of(2 * g + 1) == 2 + g
        assert o["out2"] == atom_of(2 * g + 1) * 8192 + r * 128 + ((f ^ (r & 7)) << 4)


def test_every_eight_lane_phase_hits_eight_bank_groups():
    for pw in range(NPRO):
        for k, size in (("in0", None), ("in1", None), ("out2", None), ("out3", None), ("tab", None)):
            for phase in range(4):
                lanes = range(8 * phase, 8 * phase + 8)
                groups = {(pair_offsets(pw, lane)[k] >> 4) & 7 for lane in lanes}
                assert len(groups) == 8, (pw, k, phase, groups)


def test_table_offsets_in_bounds():
    for pw, lane in THREADS:
        o = pair_offsets(pw, lane)
        assert 0 <= o["tab"] < 64 * 64 and o["tab"] % 16 == 0
        # row r's chunk f of the 64-byte-swizzled tile holds table columns 4f .. 4f+3
        assert (o["tab"] - o["r"] * 64) >> 4 == o["f"] ^ ((o["r"] >> 1) & 3)
