"""A CPU model of pass C's epilogue (pass_c_tc in lcla_tc.cuh): tensor memory
-> registers -> stmatrix.trans -> 64-byte-swizzled [32 token][32 channel]
bf16 box -> TMA store.

Restated here:
* the register fragment the kernel's 16x256b loads give a lane:
  v[16 L + 4 j + i] = D[c = 16 L + lane / 4 + 8 (i >> 1)][tok = 8 j + 2 (lane % 4) + (i & 1)];
* the kernel packs (v[4j], v[4j+1]), (v[4j+2], v[4j+3]), (v[16+4j], v[16+4j+1]),
  (v[16+4j+2], v[16+4j+3]) as the four registers of stmatrix.x4.trans, and
  lane l gives the address of row l & 7 of matrix l >> 3: token 8 j + (l & 7),
  16-byte chunk l >> 3 (channels 8 (l >> 3) .. +8), swizzled by ((tok >> 1) & 3);
* stmatrix with .trans: lane t's register r holds row t / 4, columns
  2 (t % 4), 2 (t % 4) + 1 of 8 x 8 matrix r, stored transposed;
* the 64-byte swizzle of the TMA box: chunk m of the 64-byte row r sits at
  m ^ ((r >> 1) & 3).
Checked: after the TMA store reads the box back unswizzled, row tok, column c
is D[c][tok] -- the output for token tok, channel c.  No GPU."""
import numpy as np


def test_stmatrix_transpose_writes_the_output_box():
    rng = np.random.default_rng(3)
    D = rng.standard_normal((32, 32))           # accumulator block: [channel c][token], one head, 32 tokens
    box = np.full((32, 4, 8), np.nan)           # smem box: [row][16-byte chunk][bf16 element]
    for j in range(4):                          # the four stmatrix.x4.trans calls
        regs = {}
        for lane in range(32):
            v = {}
            for L in range(2):
                for jj in range(4):
                    for i in range(4):
                        v[16 * L + 4 * jj + i] = D[16 * L + lane // 4 + 8 * (i >> 1), 8 * jj + 2 * (lane % 4) + (i & 1)]
            regs[lane] = [(v[4 * j], v[4 * j + 1]), (v[4 * j + 2], v[4 * j + 3]),
                          (v[16 + 4 * j], v[16 + 4 * j + 1]), (v[16 + 4 * j + 2], v[16 + 4 * j + 3])]
        # row addresses: lane l -> matrix l >> 3, row l & 7
        row_addr = {}
        for lane in range(32):
            m, k = lane >> 3, lane & 7
            tok = 8 * j + k
            row_addr[(m, k)] = (tok, m ^ ((tok >> 1) & 3))
        # .trans: element (row t/4, col 2 (t%4) + h) of matrix r goes to matrix row (2 (t%4) + h), column t/4
        for t in range(32):
            for r in range(4):
                for h in range(2):
                    mrow, mcol = 2 * (t % 4) + h, t // 4
                    tok, chunk = row_addr[(r, mrow)]
                    assert np.isnan(box[tok, chunk, mcol])          # each element written once
                    box[tok, chunk, mcol] = regs[t][r][h]
    assert not np.isnan(box).any()
    # the TMA store reads the box with the 64-byte swizzle undone
    out = np.empty((32, 32))
    for tok in range(32):
        for m in range(4):
            out[tok, 8 * m:8 * m + 8] = box[tok, m ^ ((tok >> 1) & 3)]
    np.testing.assert_array_equal(out, D.T)
