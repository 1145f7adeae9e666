"""A CPU model of how the tensor-core passes serve head dim 64 (pass_a_tc<64>
and pass_c_tc<64> in lcla_tc.cuh).

A quad work unit holds two 64-dim heads as four 32-dim virtual heads
(vh = 2 R + half).  The model restates the operand layouts with numpy
products in place of the MMAs and checks:

* pass A: the quad product D[(vh', c)][(vh, e)] = sum_tok v[tok][vh', c]
  k~[tok][vh, e] holds, in the blocks of a head's two halves, the whole
  64 x 64 state, which the drain of virtual head q assembles as row 32 a + c
  from the column blocks of virtual heads q & ~1 and q | 1;
* pass C: the stage's operand atoms hold virtual heads 0, 2, 1, 3; the first
  MMA set multiplies the prefix's first key half by the stage operand, the
  second set the second key half by the operand window two atoms on (virtual
  heads 1, 3, then two atoms past the stage that feed unread columns); column
  block R of the sum is head R's output, the block the epilogue reads
  (64 * (q >> 1)).  No GPU."""
import numpy as np

T = 64
rng = np.random.default_rng(7)


def atom_of(h):
    return (h >> 1) + 2 * (h & 1)


def test_pass_a_quad_products_hold_the_64_dim_states():
    v = rng.standard_normal((T, 4, 32))        # [tok][virtual head][c]
    k = rng.standard_normal((T, 4, 32))        # rotated keys
    # D[(vh', c)][(vh, e)] over the quad: every block, as the MMA computes it
    D = np.einsum("tac,tbe->acbe", v, k)       # [vh'][c][vh][e]
    for R in range(2):                         # the two heads of the quad
        v64 = np.concatenate([v[:, 2 * R], v[:, 2 * R + 1]], axis=1)
        k64 = np.concatenate([k[:, 2 * R], k[:, 2 * R + 1]], axis=1)
        S = v64.T @ k64                        # the 64 x 64 state of head R
        for q in (2 * R, 2 * R + 1):           # drain warps of the head's two virtual heads
            a = q & 1
            rows = np.concatenate([D[q, :, (q & ~1) + hb, :] for hb in range(2)], axis=1)   # [c][64]
            np.testing.assert_allclose(rows, S[32 * a:32 * a + 32], rtol=1e-12, atol=1e-12)


def test_pass_c_two_key_halves_land_in_column_block_R():
    P = rng.standard_normal((2, 64, 64))       # prefix states of the quad's two heads [R][row][key]
    qt = rng.standard_normal((T, 4, 32))       # normalised rotated queries [tok][virtual head][e]
    # the stage: atom a holds virtual head 2 (a & 1) + (a >> 1); rows (atom, tok), K = e; two atoms of
    # whatever follows the stage in shared memory
    atoms = [qt[:, 2 * (a & 1) + (a >> 1)] for a in range(4)]
    beyond = [rng.standard_normal((T, 32)) for _ in range(2)]
    B1 = np.concatenate(atoms, axis=0)                         # 256 rows
    B2 = np.concatenate(atoms[2:] + beyond, axis=0)            # the window two atoms on
    # A operands: rows (virtual head q, c) = row 32 (q & 1) + c of head q >> 1, key half kh
    A = [np.concatenate([P[q >> 1, 32 * (q & 1):32 * (q & 1) + 32, 32 * kh:32 * kh + 32] for q in range(4)], axis=0)
         for kh in range(2)]
    D = A[0] @ B1.T + A[1] @ B2.T                              # [128 rows][256 columns]
    for q in range(4):
        R, a = q >> 1, q & 1
        q64 = np.concatenate([qt[:, 2 * R], qt[:, 2 * R + 1]], axis=1)      # head R's 64 dims per token
        want = (P[R] @ q64.T)[32 * a:32 * a + 32]                          # rows 32 a + c, columns tok
        ocol = 64 * (q >> 1)                                                # the epilogue's column block
        got = D[32 * q:32 * q + 32, ocol:ocol + T]
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # at head width 32 the epilogue reads the diagonal atom instead
    assert [atom_of(q) for q in range(4)] == [0, 2, 1, 3]
