// lcla_plan.h -- how one call is cut into work units (host and device).
//
// Tokens of one (b, h) form blocks of block_len tokens; a token attends to
// its own block and every earlier block ("Implementing Block Causal Linear
// Attention for Long Video Generation with Sana", section "Chunk-Wise
// Causality").  The kernels cut the sequence into *segments*, contiguous token
// ranges that either
//   - lie inside one block (block mode: block_len >= LCLA_T, explicit block
//     offsets, and every block length at head dim 64): every token of the
//     segment uses the inclusive prefix state of its block; or
//   - hold whole blocks only (chunk mode, block_len < LCLA_T at d = 32): tiles of
//     T = (LCLA_T / block_len) * block_len tokens, where a token uses the
//     exclusive prefix at the tile start plus a masked term inside the tile.
// Pass A reduces each segment to a partial state, the scan turns partials
// into prefixes, pass C produces the outputs.
#pragma once
#include <stddef.h>

#define LCLA_D 32                              // head dim of the tensor-core and tiled CUDA-core kernels
#define LCLA_D_WIDE 64                         // the other head dim served (generic CUDA-core kernels)
#define LCLA_HG 2                              // heads per CTA (CUDA-core path)
#define LCLA_T 64                              // tokens per tile (CUDA-core path)
#define LCLA_TC_T 64                           // tokens per tile (tensor-core path)
#define LCLA_TC_HQ 4                           // heads per work unit (tensor-core path)
#define LCLA_TC_CTAS LCLA_SMS                  // persistent tensor-core CTAs (one per SM)
#define LCLA_SZ ((LCLA_D + 1) * LCLA_D)        // floats per (S, z) state at LCLA_D
#define LCLA_SMS 148                           // B200 streaming multiprocessors
#define LCLA_TARGET_CTAS (LCLA_SMS * 4)        // CTAs per pass the CUDA-core plan aims for

struct LclaPlan {
    int B, H, N, L, dtype;
    int d, sz;     // head dim and floats per (S, z) state, (d + 1) * d
    int chunk;     // 0: block mode, 1: chunk mode
    int tc;        // 1: tensor-core kernels (bf16, block mode), 0: CUDA-core kernels
    int T;         // chunk mode: tokens per tile (whole blocks); block mode: tile tokens
    int nb;        // blocks
    int nsb;       // block mode: segments per block
    int tps;       // chunk mode: tiles per segment
    int nseg;      // segments
    int npref;     // prefix entries: block mode nb, chunk mode nseg
    int ngroups;   // head groups of LCLA_HG heads (CUDA-core grid)
    int nquads;    // head groups of LCLA_TC_HQ heads (tensor-core work units)
    int scs, nch;  // scan over many groups: segments per scan chunk (whole groups) and chunks; nch = 0: one pass
    const int *boff;   // explicit blocks: device array of nb + 1 token offsets (block b = [boff[b], boff[b+1]));
                       // null: uniform blocks of L tokens
    size_t part_off, pref_off, ctot_off, ws_bytes;   // workspace layout (bytes)
};

struct LclaSeg {
    int t0, t1;    // token range [t0, t1), possibly empty
    int blk;       // block mode: block index; chunk mode: -1
};

#ifdef __CUDACC__
#define LCLA_HD __host__ __device__ __forceinline__
#else
#define LCLA_HD inline
#endif

LCLA_HD int lcla_min_i(int a, int b) { return a < b ? a : b; }

// Token range of segment s.  All arithmetic fits in 32 bits: N <= 2^30 (the
// API rejects larger N), so block starts, token counts and j * per stay below
// 2^30 before the final multiply by the tile length, which is bounded by the
// block length.
LCLA_HD LclaSeg lcla_segment(const LclaPlan &p, int s)
{
    LclaSeg g;
    if (!p.chunk) {
        g.blk = s / p.nsb;
        const int j = s - g.blk * p.nsb;
        int b0, bl;
        if (p.boff) {   // explicit blocks (device code only): clamped into [0, N], an inverted pair is empty
            b0 = lcla_min_i(p.boff[g.blk] > 0 ? p.boff[g.blk] : 0, p.N);
            const int b1 = lcla_min_i(p.boff[g.blk + 1] > 0 ? p.boff[g.blk + 1] : 0, p.N);
            bl = b1 > b0 ? b1 - b0 : 0;
        } else {
            b0 = g.blk * p.L;
            bl = lcla_min_i(p.L, p.N - b0);
        }
        const int nt = (bl + p.T - 1) / p.T;               // tiles in this block
        const int per = (nt + p.nsb - 1) / p.nsb;          // tiles per segment
        g.t0 = b0 + lcla_min_i(lcla_min_i(j * per, nt) * p.T, bl);
        g.t1 = b0 + lcla_min_i(lcla_min_i((j + 1) * per, nt) * p.T, bl);
    } else {
        const int span = p.tps * p.T;
        g.t0 = s < p.nseg ? lcla_min_i(s * span, p.N) : p.N;   // (nseg - 1) * span < N + T
        g.t1 = lcla_min_i(g.t0 + span, p.N);
        g.blk = -1;
    }
    return g;
}
