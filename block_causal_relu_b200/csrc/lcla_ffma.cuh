// lcla_ffma.cuh -- CUDA-core (FFMA) kernels for every dtype and block length.
//
// Pass A: per segment, the partial state
//           S[c][e] = sum_j v_j[c] (R_j phi(k_j))[e],  z[e] = sum_j phi(k_j)[e]
//         ("Implementing Block Causal Linear Attention for Long Video
//          Generation with Sana", section "The Linear Attention Kernel":
//          vk = v k_rotated^T and the key sum of the normaliser).
// Pass C: out_i = (P S) R_i phi(q_i) / (P_z . phi(q_i) + eps) with P the
//         prefix state the token sees (same section: out = vk q_rotated,
//         output = out * z).  Chunk mode adds the masked in-tile term.
// phi = ReLU applied to q and k only; the rotary embedding R acts on the
// ReLU features, interleaved pairs (same page, "Rotary Position Embeddings").
//
// Both passes stream [tile][head group] slices of the [B, N, H, d] inputs
// through shared memory with cp.async (16-byte chunks, zero fill for ragged
// tiles and missing heads, so padding contributes exact zeros), keep all
// arithmetic in fp32 and reduce in a fixed order (no atomics).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "lcla_common.cuh"
#include "lcla_plan.h"

namespace lcla {

// ---------------------------------------------------------------------------
// Pass A: segment partial states.  grid (nseg, ngroups, B), 256 threads.
// part layout: [nseg][B][H][D+1][D] fp32.
// ---------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(256)
pass_a_ffma(const Tin *__restrict__ k, const Tin *__restrict__ v, const float *__restrict__ rcos,
            const float *__restrict__ rsin, const LclaPlan p, float *__restrict__ part)
{
    using G = Geo<Tin>;
    constexpr int STAGE = 2 * G::TILE_IN + 2 * G::TILE_TAB;
    extern __shared__ __align__(128) unsigned char sm[];
    float *kt = reinterpret_cast<float *>(sm + 2 * STAGE);   // [T][HG][D] rotated features

    const int s = blockIdx.x / p.ngroups, h0 = (blockIdx.x % p.ngroups) * LCLA_HG, b = blockIdx.y;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const LclaSeg g = lcla_segment(p, s);
    const int ntile = (g.t1 - g.t0 + LCLA_T - 1) / LCLA_T;

    // outer-product micro tile: warp w -> head w>>2, 16 tokens of each tile;
    // lane -> value dims c0..c0+3, key dims e0..e0+7
    const int ohh = w >> 2, otq = (w & 3) * 16;
    const int c0 = (lane >> 2) * 4, e0 = (lane & 3) * 8;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    float zacc[8];   // key-sum partial of (head (tid>>2)&1, dims (tid&3)*8..+8)
#pragma unroll
    for (int i = 0; i < 8; ++i) zacc[i] = 0.f;

    auto issue = [&](int st, int i) {
        unsigned char *buf = sm + st * STAGE;
        const int t = g.t0 + i * LCLA_T, nt = min(LCLA_T, g.t1 - t);
        issue_rows<Tin>(buf, k, p, b, t, nt, h0, tid, 256);
        issue_rows<Tin>(buf + G::TILE_IN, v, p, b, t, nt, h0, tid, 256);
        issue_table(buf + 2 * G::TILE_IN, rcos, t, nt, tid, 256);
        issue_table(buf + 2 * G::TILE_IN + G::TILE_TAB, rsin, t, nt, tid, 256);
        cp_async_commit();
    };

    if (ntile > 0) issue(0, 0);
    for (int i = 0; i < ntile; ++i) {
        if (i + 1 < ntile) {
            issue((i + 1) & 1, i + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const unsigned char *buf = sm + (i & 1) * STAGE;
        const Tin *kraw = reinterpret_cast<const Tin *>(buf);
        const Tin *vraw = reinterpret_cast<const Tin *>(buf + G::TILE_IN);
        const float *ct = reinterpret_cast<const float *>(buf + 2 * G::TILE_IN);
        const float *st = reinterpret_cast<const float *>(buf + 2 * G::TILE_IN + G::TILE_TAB);

        // prologue: phi, rotary, key sum
        for (int it = tid; it < LCLA_T * LCLA_HG * 4; it += 256) {
            const int tok = it >> 3, hh = (it >> 2) & 1, qtr = it & 3;
            float x[8], f[8], y[8];
            load8(kraw + (tok * LCLA_HG + hh) * LCLA_D + qtr * 8, x);
            const float4 c4 = reinterpret_cast<const float4 *>(ct + tok * (LCLA_D / 2))[qtr];
            const float4 s4 = reinterpret_cast<const float4 *>(st + tok * (LCLA_D / 2))[qtr];
            relu_rope8(x, c4, s4, f, y);
#pragma unroll
            for (int j = 0; j < 8; ++j) zacc[j] += f[j];
            float4 *dst = reinterpret_cast<float4 *>(kt + (tok * LCLA_HG + hh) * LCLA_D + qtr * 8);
            dst[0] = make_float4(y[0], y[1], y[2], y[3]);
            dst[1] = make_float4(y[4], y[5], y[6], y[7]);
        }
        __syncthreads();

        // outer products over this warp's 16 tokens
#pragma unroll 4
        for (int t = 0; t < 16; ++t) {
            const int tok = otq + t;
            float vv[4];
            load4(vraw + (tok * LCLA_HG + ohh) * LCLA_D + c0, vv);
            const float4 ka = *reinterpret_cast<const float4 *>(kt + (tok * LCLA_HG + ohh) * LCLA_D + e0);
            const float4 kb = *reinterpret_cast<const float4 *>(kt + (tok * LCLA_HG + ohh) * LCLA_D + e0 + 4);
            const float kk[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[ii][j] = fmaf(vv[ii], kk[j], acc[ii][j]);
        }
        __syncthreads();
    }

    pdl_trigger();
    // fixed-order reduction of the 4 warps of each head and of the key sums
    float *red = reinterpret_cast<float *>(sm);                 // [8][D][D]
    float *zred = red + 8 * LCLA_D * LCLA_D;                     // [256][8]
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int j = 0; j < 8; ++j) red[w * LCLA_D * LCLA_D + (c0 + ii) * LCLA_D + e0 + j] = acc[ii][j];
#pragma unroll
    for (int j = 0; j < 8; ++j) zred[tid * 8 + j] = zacc[j];
    __syncthreads();
    for (int x = tid; x < LCLA_HG * LCLA_SZ; x += 256) {
        const int hh = x / LCLA_SZ, e = x - hh * LCLA_SZ;
        float val;
        if (e < LCLA_D * LCLA_D) {
            const float *r = red + (hh * 4) * LCLA_D * LCLA_D + e;
            val = ((r[0] + r[LCLA_D * LCLA_D]) + r[2 * LCLA_D * LCLA_D]) + r[3 * LCLA_D * LCLA_D];
        } else {
            const int ez = e - LCLA_D * LCLA_D, qtr = ez >> 3, jj = ez & 7;
            const int t0 = hh * 4 + qtr;      // threads t0, t0+8, ... hold this key-sum slot
            val = 0.f;
            for (int m = 0; m < 32; ++m) val += zred[(t0 + 8 * m) * 8 + jj];
        }
        if (h0 + hh < p.H)
            part[(((size_t)s * p.B + b) * p.H + (h0 + hh)) * LCLA_SZ + e] = val;
    }
}

// ---------------------------------------------------------------------------
// Pass C, block mode: every token of the segment uses its block's inclusive
// prefix.  grid (nseg, ngroups, B), 256 threads.
// pref layout: [npref][B][H][D+1][D] fp32.
// ---------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(256)
pass_c_ffma(const Tin *__restrict__ q, const float *__restrict__ rcos, const float *__restrict__ rsin,
            const LclaPlan p, const float *__restrict__ pref, const float eps, Tin *__restrict__ out)
{
    using G = Geo<Tin>;
    constexpr int STAGE = G::TILE_IN + 2 * G::TILE_TAB;
    extern __shared__ __align__(128) unsigned char sm[];
    float *qt = reinterpret_cast<float *>(sm + 2 * STAGE);            // [T][HG][D]
    float *PT = qt + LCLA_T * LCLA_HG * LCLA_D;                       // [HG][D e][D c]
    float *zz = PT + LCLA_HG * LCLA_D * LCLA_D;                       // [HG][D]
    float *inv = zz + LCLA_HG * LCLA_D;                               // [T][HG]

    const int s = blockIdx.x / p.ngroups, h0 = (blockIdx.x % p.ngroups) * LCLA_HG, b = blockIdx.y;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const LclaSeg g = lcla_segment(p, s);
    const int ntile = (g.t1 - g.t0 + LCLA_T - 1) / LCLA_T;
    if (ntile <= 0) return;
    pdl_wait();

    // prefix state of this block, transposed to [e][c]
    for (int x = tid; x < LCLA_HG * LCLA_SZ; x += 256) {
        const int hh = x / LCLA_SZ, e = x - hh * LCLA_SZ;
        float val = 0.f;
        if (h0 + hh < p.H) val = pref[(((size_t)g.blk * p.B + b) * p.H + (h0 + hh)) * LCLA_SZ + e];
        if (e < LCLA_D * LCLA_D) PT[hh * LCLA_D * LCLA_D + (e & 31) * LCLA_D + (e >> 5)] = val;
        else zz[hh * LCLA_D + (e - LCLA_D * LCLA_D)] = val;
    }

    const int ohh = w >> 2, otq = (w & 3) * 16 + (lane >> 3) * 4;   // 4 tokens per lane
    const int c0 = (lane & 7) * 4;

    auto issue = [&](int st, int i) {
        unsigned char *buf = sm + st * STAGE;
        const int t = g.t0 + i * LCLA_T, nt = min(LCLA_T, g.t1 - t);
        issue_rows<Tin>(buf, q, p, b, t, nt, h0, tid, 256);
        issue_table(buf + G::TILE_IN, rcos, t, nt, tid, 256);
        issue_table(buf + G::TILE_IN + G::TILE_TAB, rsin, t, nt, tid, 256);
        cp_async_commit();
    };

    issue(0, 0);
    for (int i = 0; i < ntile; ++i) {
        if (i + 1 < ntile) {
            issue((i + 1) & 1, i + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const unsigned char *buf = sm + (i & 1) * STAGE;
        const Tin *qraw = reinterpret_cast<const Tin *>(buf);
        const float *ct = reinterpret_cast<const float *>(buf + G::TILE_IN);
        const float *st = reinterpret_cast<const float *>(buf + G::TILE_IN + G::TILE_TAB);
        const int t = g.t0 + i * LCLA_T, nt = min(LCLA_T, g.t1 - t);

        // prologue: phi, rotary, denominator (4 lanes per (token, head))
        for (int it = tid; it < LCLA_T * LCLA_HG * 4; it += 256) {
            const int tok = it >> 3, hh = (it >> 2) & 1, qtr = it & 3;
            float x[8], f[8], y[8];
            load8(qraw + (tok * LCLA_HG + hh) * LCLA_D + qtr * 8, x);
            const float4 c4 = reinterpret_cast<const float4 *>(ct + tok * (LCLA_D / 2))[qtr];
            const float4 s4 = reinterpret_cast<const float4 *>(st + tok * (LCLA_D / 2))[qtr];
            relu_rope8(x, c4, s4, f, y);
            float dp = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) dp = fmaf(f[j], zz[hh * LCLA_D + qtr * 8 + j], dp);
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            dp += __shfl_xor_sync(0xffffffffu, dp, 2);
            if (qtr == 0) inv[tok * LCLA_HG + hh] = 1.0f / (dp + eps);
            float4 *dst = reinterpret_cast<float4 *>(qt + (tok * LCLA_HG + hh) * LCLA_D + qtr * 8);
            dst[0] = make_float4(y[0], y[1], y[2], y[3]);
            dst[1] = make_float4(y[4], y[5], y[6], y[7]);
        }
        __syncthreads();

        // outputs: 4 tokens x 4 value dims per lane
        float acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll
        for (int e4 = 0; e4 < LCLA_D / 4; ++e4) {
            float4 qv[4], pv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
                qv[a] = *reinterpret_cast<const float4 *>(qt + ((otq + a) * LCLA_HG + ohh) * LCLA_D + e4 * 4);
#pragma unroll
            for (int m = 0; m < 4; ++m)
                pv[m] = *reinterpret_cast<const float4 *>(PT + ohh * LCLA_D * LCLA_D + (e4 * 4 + m) * LCLA_D + c0);
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float qq[4] = {qv[a].x, qv[a].y, qv[a].z, qv[a].w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    acc[a][0] = fmaf(qq[m], pv[m].x, acc[a][0]);
                    acc[a][1] = fmaf(qq[m], pv[m].y, acc[a][1]);
                    acc[a][2] = fmaf(qq[m], pv[m].z, acc[a][2]);
                    acc[a][3] = fmaf(qq[m], pv[m].w, acc[a][3]);
                }
            }
        }
        if (h0 + ohh < p.H) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int tok = otq + a;
                if (tok < nt) {
                    const float r = inv[tok * LCLA_HG + ohh];
                    float o[4] = {acc[a][0] * r, acc[a][1] * r, acc[a][2] * r, acc[a][3] * r};
                    store4(out + (((size_t)b * p.N + (size_t)(t + tok)) * p.H + (h0 + ohh)) * LCLA_D + c0, o);
                }
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Pass C, chunk mode (block_len <= LCLA_T): tiles of whole blocks.  Each
// segment walks its tiles in order with a running state R (exclusive prefix
// at the tile start):
//   num_i = R_S q~_i + sum_{j in tile, blk(j) <= blk(i)} v_j (k~_j . q~_i)
//   den_i = (R_z + sum_{same j} phi(k_j)) . phi(q_i) + eps
// then R += the tile's (S, z).  grid (nseg * ngroups, B), CHUNK_THREADS threads.
// ---------------------------------------------------------------------------
constexpr int CHUNK_THREADS = 512;   // 16 warps: one CTA fills an SM's shared memory, so the warps are the latency hiding
// Rows of the rotated features (token stride) and of the score matrix are padded by 4 floats: a
// 128-bit shared access is served eight lanes at a time, and with 17 16-byte chunks per row the
// rows of consecutive tokens fall on different bank groups.
constexpr int CHUNK_QK_TS = LCLA_HG * LCLA_D + 4;   // floats per token row of qt / kt
constexpr int CHUNK_SC_TS = LCLA_T + 4;             // floats per score row
constexpr int CHUNK_RED_TS = LCLA_D + 1;           // floats per row of the per-token-group state partials
// bytes beyond the unpadded layout: row padding, a second v tile (the next tile's v lands while this one's is
// in use) and the key-sum run totals
template <typename Tin>
constexpr int chunk_smem_extra() { return (2 * LCLA_T * 4 + LCLA_HG * LCLA_T * 4 + 8 * LCLA_HG * LCLA_D) * 4 + Geo<Tin>::TILE_IN; }

template <typename Tin>
__global__ void __launch_bounds__(CHUNK_THREADS)
pass_c_chunk_ffma(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const float *__restrict__ rcos, const float *__restrict__ rsin, const LclaPlan p,
                  const float *__restrict__ pref, const float eps, Tin *__restrict__ out)
{
    using G = Geo<Tin>;
    extern __shared__ __align__(128) unsigned char sm[];
    unsigned char *qraw_b = sm;
    unsigned char *kraw_b = qraw_b + G::TILE_IN;
    unsigned char *vraw_b = kraw_b + G::TILE_IN;                       // two v tiles: this one, the next
    unsigned char *ct_b = vraw_b + 2 * G::TILE_IN;
    unsigned char *st_b = ct_b + G::TILE_TAB;
    float *qt = reinterpret_cast<float *>(st_b + G::TILE_TAB);        // [T][CHUNK_QK_TS] rotated q: [HG][D] + pad
    float *kt = qt + LCLA_T * CHUNK_QK_TS;                            // rotated k, same rows
    float *fq = kt + LCLA_T * CHUNK_QK_TS;                            // [T][HG][D] phi(q)
    float *fk = fq + LCLA_T * LCLA_HG * LCLA_D;                       // phi(k), then its running sum
    float *sc = fk + LCLA_T * LCLA_HG * LCLA_D;                       // [HG][T j][CHUNK_SC_TS] scores / reduction
    float *RT = sc + LCLA_HG * LCLA_T * CHUNK_SC_TS;                  // [HG][D e][D c]
    float *Rz = RT + LCLA_HG * LCLA_D * LCLA_D;                       // [HG][D]
    float *ktot = Rz + LCLA_HG * LCLA_D;                              // [8 runs][HG][D] key-sum run totals

    const int s = blockIdx.x / p.ngroups, h0 = (blockIdx.x % p.ngroups) * LCLA_HG, b = blockIdx.y;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const LclaSeg g = lcla_segment(p, s);
    const int T = p.T, L = p.L;
    const int ntile = (g.t1 - g.t0 + T - 1) / T;
    if (ntile <= 0) return;
    pdl_wait();

    for (int x = tid; x < LCLA_HG * LCLA_SZ; x += CHUNK_THREADS) {
        const int hh = x / LCLA_SZ, e = x - hh * LCLA_SZ;
        float val = 0.f;
        if (h0 + hh < p.H) val = pref[(((size_t)s * p.B + b) * p.H + (h0 + hh)) * LCLA_SZ + e];
        if (e < LCLA_D * LCLA_D) RT[hh * LCLA_D * LCLA_D + (e & 31) * LCLA_D + (e >> 5)] = val;
        else Rz[hh * LCLA_D + (e - LCLA_D * LCLA_D)] = val;
    }

    // outputs: warp w -> head w / 8 and tokens [8 (w % 8), +8); lane -> 2 tokens (lane / 8) and 4 channels
    const int ohh = w >> 3, otq = (w & 7) * 8 + (lane >> 3) * 2;
    const int c0 = (lane & 7) * 4;

    // one cp.async group per tile: q, k and the tables (free once the tile's prologue is done) and v into
    // the v tile the tile before last used
    auto issue_tile = [&](int ii) {
        const int tt = g.t0 + ii * T, ntt = min(T, g.t1 - tt);
        issue_rows<Tin>(qraw_b, q, p, b, tt, ntt, h0, tid, CHUNK_THREADS);
        issue_rows<Tin>(kraw_b, k, p, b, tt, ntt, h0, tid, CHUNK_THREADS);
        issue_rows<Tin>(vraw_b + (ii & 1) * G::TILE_IN, v, p, b, tt, ntt, h0, tid, CHUNK_THREADS);
        issue_table(ct_b, rcos, tt, ntt, tid, CHUNK_THREADS);
        issue_table(st_b, rsin, tt, ntt, tid, CHUNK_THREADS);
        cp_async_commit();
    };
    issue_tile(0);
    for (int i = 0; i < ntile; ++i) {
        const int t = g.t0 + i * T, nt = min(T, g.t1 - t);
        cp_async_wait<0>();
        __syncthreads();
        const Tin *qraw = reinterpret_cast<const Tin *>(qraw_b);
        const Tin *kraw = reinterpret_cast<const Tin *>(kraw_b);
        const Tin *vraw = reinterpret_cast<const Tin *>(vraw_b + (i & 1) * G::TILE_IN);
        const float *ct = reinterpret_cast<const float *>(ct_b);
        const float *st = reinterpret_cast<const float *>(st_b);

        // prologue for q and k (rows past nt are zero-filled, so they give zeros)
        for (int it = tid; it < LCLA_T * LCLA_HG * 4; it += CHUNK_THREADS) {
            const int tok = it >> 3, hh = (it >> 2) & 1, qtr = it & 3;
            const float4 c4 = reinterpret_cast<const float4 *>(ct + tok * (LCLA_D / 2))[qtr];
            const float4 s4 = reinterpret_cast<const float4 *>(st + tok * (LCLA_D / 2))[qtr];
            const int o = (tok * LCLA_HG + hh) * LCLA_D + qtr * 8;
            const int ot = tok * CHUNK_QK_TS + hh * LCLA_D + qtr * 8;
            float x[8], f[8], y[8];
            load8(qraw + o, x);
            relu_rope8(x, c4, s4, f, y);
#pragma unroll
            for (int j = 0; j < 8; ++j) { fq[o + j] = f[j]; qt[ot + j] = y[j]; }
            load8(kraw + o, x);
            relu_rope8(x, c4, s4, f, y);
#pragma unroll
            for (int j = 0; j < 8; ++j) { fk[o + j] = f[j]; kt[ot + j] = y[j]; }
        }
        __syncthreads();
        if (i + 1 < ntile) issue_tile(i + 1);   // the prologue has consumed q, k and the tables

        // scores sc[hh][j][i] = [blk(j) <= blk(i)] (k~_j . q~_i); a thread takes queries ib*4..+3 and keys
        // jb, jb+16, jb+32, jb+48, so that the lanes of a warp read consecutive key rows
        for (int blkid = tid; blkid < LCLA_HG * 16 * 16; blkid += CHUNK_THREADS) {
            const int hh = blkid >> 8, ib = (blkid >> 4) & 15, jb = blkid & 15;
            float a[4][4];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) a[ii][jj] = 0.f;
#pragma unroll
            for (int e4 = 0; e4 < LCLA_D / 4; ++e4) {
                float4 qv[4], kv[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    qv[x] = *reinterpret_cast<const float4 *>(qt + (ib * 4 + x) * CHUNK_QK_TS + hh * LCLA_D + e4 * 4);
                    kv[x] = *reinterpret_cast<const float4 *>(kt + (jb + 16 * x) * CHUNK_QK_TS + hh * LCLA_D + e4 * 4);
                }
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        a[ii][jj] += qv[ii].x * kv[jj].x + qv[ii].y * kv[jj].y +
                                     qv[ii].z * kv[jj].z + qv[ii].w * kv[jj].w;
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = jb + 16 * jj;
                float o4[4];
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    const int i2 = ib * 4 + ii;
                    o4[ii] = (j < nt && (j / L) <= (i2 / L)) ? a[ii][jj] : 0.f;
                }
                *reinterpret_cast<float4 *>(sc + (hh * LCLA_T + j) * CHUNK_SC_TS + ib * 4) =
                    make_float4(o4[0], o4[1], o4[2], o4[3]);
            }
        }
        // running key sum over the tile in token order: 8 runs of 8 tokens per (head, dim) column, run r in
        // warps 2r, 2r+1 (consecutive lanes take consecutive columns), then each run adds the earlier runs' totals
        {
            const int col = tid & (LCLA_HG * LCLA_D - 1), r = tid / (LCLA_HG * LCLA_D);
            const int hh = col / LCLA_D, e = col % LCLA_D;
            float run[8], acc = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                acc += fk[((r * 8 + u) * LCLA_HG + hh) * LCLA_D + e];
                run[u] = acc;
            }
            ktot[r * LCLA_HG * LCLA_D + col] = acc;
            __syncthreads();
            float off = 0.f;
            for (int r2 = 0; r2 < r; ++r2) off += ktot[r2 * LCLA_HG * LCLA_D + col];
#pragma unroll
            for (int u = 0; u < 8; ++u) fk[((r * 8 + u) * LCLA_HG + hh) * LCLA_D + e] = run[u] + off;
        }
        __syncthreads();

        // outputs
        float acc[2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
        for (int e4 = 0; e4 < LCLA_D / 4; ++e4) {      // carried state
            float4 qv[2], pv[4];
#pragma unroll
            for (int a = 0; a < 2; ++a)
                qv[a] = *reinterpret_cast<const float4 *>(qt + (otq + a) * CHUNK_QK_TS + ohh * LCLA_D + e4 * 4);
#pragma unroll
            for (int m = 0; m < 4; ++m)
                pv[m] = *reinterpret_cast<const float4 *>(RT + ohh * LCLA_D * LCLA_D + (e4 * 4 + m) * LCLA_D + c0);
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const float qq[4] = {qv[a].x, qv[a].y, qv[a].z, qv[a].w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    acc[a][0] = fmaf(qq[m], pv[m].x, acc[a][0]);
                    acc[a][1] = fmaf(qq[m], pv[m].y, acc[a][1]);
                    acc[a][2] = fmaf(qq[m], pv[m].z, acc[a][2]);
                    acc[a][3] = fmaf(qq[m], pv[m].w, acc[a][3]);
                }
            }
        }
        for (int j = 0; j < nt; ++j) {                 // masked in-tile term
            const float2 sv = *reinterpret_cast<const float2 *>(sc + (ohh * LCLA_T + j) * CHUNK_SC_TS + otq);
            float vv[4];
            load4(vraw + (j * LCLA_HG + ohh) * LCLA_D + c0, vv);
            const float ss[2] = {sv.x, sv.y};
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(ss[a], vv[c], acc[a][c]);
        }
        // denominators: the 8 lanes sharing these 2 tokens split the key dims
        float den[2];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            const int tok = otq + a;
            const int last = min(nt, (tok / L + 1) * L) - 1;   // last in-tile token of tok's block
            const int lc = last < 0 ? 0 : last;
            float dp = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int e = c0 + m;
                const float zt = Rz[ohh * LCLA_D + e] + fk[(lc * LCLA_HG + ohh) * LCLA_D + e];
                dp = fmaf(zt, fq[(tok * LCLA_HG + ohh) * LCLA_D + e], dp);
            }
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            dp += __shfl_xor_sync(0xffffffffu, dp, 2);
            dp += __shfl_xor_sync(0xffffffffu, dp, 4);
            den[a] = dp + eps;
        }
        if (h0 + ohh < p.H) {
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                const int tok = otq + a;
                if (tok < nt) {
                    const float r = 1.0f / den[a];
                    float o[4] = {acc[a][0] * r, acc[a][1] * r, acc[a][2] * r, acc[a][3] * r};
                    store4(out + (((size_t)b * p.N + (size_t)(t + tok)) * p.H + (h0 + ohh)) * LCLA_D + c0, o);
                }
            }
        }
        __syncthreads();

        // R += tile state: warp w -> head w / 8, tokens [16 ((w / 2) % 4), +16), value dims [16 (w % 2), +16);
        // lane -> 2 value dims x 8 key dims; the four token groups of a head are summed in a fixed order
        {
            const int shh = w >> 3, tg = (w >> 1) & 3, half = w & 1;
            const int rc0 = half * 16 + (lane >> 2) * 2, re0 = (lane & 3) * 8, rtq = tg * 16;
            float ra[2][8];
#pragma unroll
            for (int ii = 0; ii < 2; ++ii)
#pragma unroll
                for (int j = 0; j < 8; ++j) ra[ii][j] = 0.f;
            for (int tt = 0; tt < 16; ++tt) {
                const int tok = rtq + tt;
                const Tin *vp = vraw + (tok * LCLA_HG + shh) * LCLA_D + rc0;
                float vv[2];
                if constexpr (sizeof(Tin) == 2) {
                    const uint32_t u = *reinterpret_cast<const uint32_t *>(vp);
                    vv[0] = bf_lo(u);
                    vv[1] = bf_hi(u);
                } else {
                    const float2 f2 = *reinterpret_cast<const float2 *>(vp);
                    vv[0] = f2.x;
                    vv[1] = f2.y;
                }
                const float4 ka = *reinterpret_cast<const float4 *>(kt + tok * CHUNK_QK_TS + shh * LCLA_D + re0);
                const float4 kb = *reinterpret_cast<const float4 *>(kt + tok * CHUNK_QK_TS + shh * LCLA_D + re0 + 4);
                const float kk[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
#pragma unroll
                for (int ii = 0; ii < 2; ++ii)
#pragma unroll
                    for (int j = 0; j < 8; ++j) ra[ii][j] = fmaf(vv[ii], kk[j], ra[ii][j]);
            }
            float *red = sc;                                 // [2 heads][4 token groups][D c][CHUNK_RED_TS]
#pragma unroll
            for (int ii = 0; ii < 2; ++ii)
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    red[((shh * 4 + tg) * LCLA_D + rc0 + ii) * CHUNK_RED_TS + re0 + j] = ra[ii][j];
        }
        __syncthreads();
        for (int x = tid; x < LCLA_HG * LCLA_D * LCLA_D; x += CHUNK_THREADS) {   // lanes: consecutive c
            const int hh = x >> 10, ec = x & 1023, e = ec >> 5, c = ec & 31;
            constexpr int G4 = LCLA_D * CHUNK_RED_TS;    // one token group's partial
            const float *r = sc + (hh * 4) * G4 + c * CHUNK_RED_TS + e;
            const float add = ((r[0] + r[G4]) + r[2 * G4]) + r[3 * G4];
            RT[hh * LCLA_D * LCLA_D + e * LCLA_D + c] += add;
        }
        if (tid < LCLA_HG * LCLA_D && nt > 0) {
            const int hh = tid >> 5, e = tid & 31;
            Rz[hh * LCLA_D + e] += fk[((nt - 1) * LCLA_HG + hh) * LCLA_D + e];
        }
        __syncthreads();
    }
}

}  // namespace lcla
