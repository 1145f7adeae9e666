"""A CPU model of the chunk-mode kernel's work split (pass_c_chunk_ffma in
lcla_ffma.cuh): 512 threads over a 64-token tile of two heads.

The model restates the kernel's thread -> work maps and checks that each phase
covers its work exactly once, and that the shared-memory accesses that once
conflicted now spread over the bank groups: the key rows of the score tiles
(token stride CHUNK_QK_TS = 68 floats) and the per-token-group state partials
(rows of CHUNK_RED_TS = 33 floats).  No GPU."""
import itertools

THREADS = 512
T, HG, D = 64, 2, 32
QK_TS = HG * D + 4      # floats per token row of the rotated features
RED_TS = D + 1          # floats per row of the state partials


def test_outputs_cover_tile_once():
    seen = set()
    for tid in range(THREADS):
        w, lane = tid >> 5, tid & 31
        ohh, otq, c0 = w >> 3, (w & 7) * 8 + (lane >> 3) * 2, (lane & 7) * 4
        for a, c in itertools.product(range(2), range(4)):
            key = (ohh, otq + a, c0 + c)
            assert key not in seen
            seen.add(key)
    assert len(seen) == HG * T * D
    # the 8 lanes that share two tokens (lane bits 3-4 equal) split the key dims of the normaliser
    for lane in range(32):
        assert {(l & 7) * 4 for l in range(32) if l >> 3 == lane >> 3} == set(range(0, D, 4))


def test_scores_cover_pairs_once_and_key_rows_spread_over_bank_groups():
    seen = set()
    for blkid in range(HG * 16 * 16):
        hh, ib, jb = blkid >> 8, (blkid >> 4) & 15, blkid & 15
        for ii, jj in itertools.product(range(4), range(4)):
            key = (hh, ib * 4 + ii, jb + 16 * jj)
            assert key not in seen
            seen.add(key)
    assert len(seen) == HG * T * T
    # one warp's 128-bit key loads: each 8-lane phase on 8 different 16-byte bank groups
    for warp in range(THREADS // 32):
        for x in range(4):
            for e4 in range(D // 4):
                for phase in range(4):
                    groups = set()
                    for lane in range(8 * phase, 8 * phase + 8):
                        blkid = 32 * warp + lane
                        hh, jb = blkid >> 8, blkid & 15
                        addr = ((jb + 16 * x) * QK_TS + hh * D + e4 * 4) * 4
                        groups.add((addr >> 4) & 7)
                    assert len(groups) == 8


def test_state_partials_cover_once_and_stores_spread():
    seen = set()
    for tid in range(THREADS):
        w, lane = tid >> 5, tid & 31
        shh, tg, half = w >> 3, (w >> 1) & 3, w & 1
        rc0, re0 = half * 16 + (lane >> 2) * 2, (lane & 3) * 8
        for ii, j in itertools.product(range(2), range(8)):
            key = (shh, tg, rc0 + ii, re0 + j)
            assert key not in seen
            seen.add(key)
    assert len(seen) == HG * 4 * D * D
    # the scalar stores of a warp at fixed (ii, j): at most 2 lanes per bank
    for w in range(THREADS // 32):
        shh, tg, half = w >> 3, (w >> 1) & 3, w & 1
        for ii, j in itertools.product(range(2), range(8)):
            banks = {}
            for lane in range(32):
                rc0, re0 = half * 16 + (lane >> 2) * 2, (lane & 3) * 8
                addr = ((shh * 4 + tg) * D + rc0 + ii) * RED_TS + re0 + j
                banks[addr % 32] = banks.get(addr % 32, 0) + 1
            assert max(banks.values()) <= 2
    # the partials fit the score buffer they reuse
    assert (HG * 4 * D) * RED_TS <= HG * T * (T + 4)


def test_key_sum_runs_and_final_reduction():
    runs = set()
    for tid in range(THREADS):
        col, r = tid & (HG * D - 1), tid // (HG * D)
        for u in range(8):
            key = (col, r * 8 + u)
            assert key not in runs
            runs.add(key)
    assert len(runs) == HG * D * T
    cells = set()
    for x in range(HG * D * D):
        hh, ec = x >> 10, x & 1023
        e, c = ec >> 5, ec & 31
        assert (hh, e, c) not in cells
        cells.add((hh, e, c))
    assert len(cells) == HG * D * D
    # a warp's read-modify-writes of the prefix rows: consecutive c, so 32 different banks
    for base in range(0, HG * D * D, 32):
        banks = {((x >> 10) * D * D + ((x & 1023) >> 5) * D + (x & 31)) % 32 for x in range(base, base + 32)}
        assert len(banks) == 32
