// lcla_gen.cuh -- CUDA-core passes for head dim 64 (linear_head_dim 64 of
// the "[feat] LongSANA" configuration), whole-block (block) mode.
//
// The same two passes as the d = 32 kernels, one (segment, head, batch entry)
// per CTA:
//   pass A: S[c][e] = sum over the segment of v[c] * (R phi(k))[e] and
//           z[e] = sum of phi(k)[e] ("Implementing Block Causal Linear
//           Attention for Long Video Generation with Sana", section "The
//           Linear Attention Kernel": vk = v k_rotated^T and the key sum);
//   pass C: out[c] = sum_e P[c][e] (R phi(q))[e] / (z . phi(q) + eps) with P,
//           z the inclusive prefix of the token's block.
// Tokens are staged 32 at a time in shared memory as fp32 features and the
// state is accumulated in fp32 registers.  A 128-bit shared load is served
// eight lanes at a time, so the inner loops read what a whole warp shares as
// one broadcast and give each lane a distinct 64-bit slice: pass A, warp w
// owns key dims [8w, 8w + 8) and lane l value dims 2l, 2l + 1; pass C (64-token
// tiles), warp w owns tokens [8w, 8w + 8) and lane l output channels 2l, 2l + 1.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "lcla_common.cuh"
#include "lcla_plan.h"

namespace lcla {
namespace gen {

constexpr int THREADS = 256;
constexpr int TT = 32;   // tokens per shared-memory tile: 8 lanes x 8 dims cover one 64-dim head row
// resident CTAs per SM (-Xptxas -v: pass A 80 registers -> 3 x 256 threads; pass C 55 registers and
// 33.8 KB of shared memory -> 4), used by the planner to fill whole waves
constexpr int RES_A = 3, RES_C = 4;

// 8 consecutive elements of a head row, fetched raw (held in registers across a tile) and widened later
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void fetch(const __nv_bfloat16 *p) { u = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void widen(float *x) const
    {
        x[0] = bf_lo(u.x); x[1] = bf_hi(u.x); x[2] = bf_lo(u.y); x[3] = bf_hi(u.y);
        x[4] = bf_lo(u.z); x[5] = bf_hi(u.z); x[6] = bf_lo(u.w); x[7] = bf_hi(u.w);
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void fetch(const float *p)
    {
        a = reinterpret_cast<const float4 *>(p)[0];
        b = reinterpret_cast<const float4 *>(p)[1];
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void widen(float *x) const
    {
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};

__device__ __forceinline__ void store2(__nv_bfloat16 *p, float a, float b)
{
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void store2(float *p, float a, float b)
{
    *reinterpret_cast<float2 *>(p) = make_float2(a, b);
}

template <typename Tin, int D>
__global__ void __launch_bounds__(THREADS)
pass_a_gen(const Tin *__restrict__ k, const Tin *__restrict__ v, const float *__restrict__ rc,
           const float *__restrict__ rs, const LclaPlan p, float *__restrict__ part)
{
    static_assert(D == 64, "thread mapping: 8 lanes x 8 dims per token row; 8 warps x 8 key dims, 32 lanes x 2 value dims");
    __shared__ __align__(16) float kt[TT][D];   // rotated key features
    __shared__ __align__(16) float vt[TT][D];
    __shared__ float zw[THREADS / 32][D];      // key-sum parts per warp
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const LclaSeg g = lcla_segment(p, s);
    const int tok = tid >> 3, j = tid & 7, e0 = j * 8;        // loader: token row and 8 dims
    // state: warp w owns key dims [8w, 8w + 8) (read as a broadcast), lane l value dims 2l, 2l + 1
    const int ew = (tid >> 5) * 8, cl = (tid & 31) * 2;
    float acc[2][8] = {};
    float zacc[8] = {};
    // the next tile's raw rows are fetched into registers before this tile's products, so the global
    // latency overlaps them
    Raw8<Tin> rk, rv;
    float4 c4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = c4;
    auto fetch = [&](int t) {
        const int n = t + tok;
        if (n < g.t1) {
            const size_t row = (((size_t)b * p.N + n) * p.H + h) * D + e0;
            rk.fetch(k + row);
            rv.fetch(v + row);
            c4 = *reinterpret_cast<const float4 *>(rc + (size_t)n * (D / 2) + j * 4);
            s4 = *reinterpret_cast<const float4 *>(rs + (size_t)n * (D / 2) + j * 4);
        } else {
            rk.zero();
            rv.zero();
        }
    };
    if (g.t0 < g.t1) fetch(g.t0);
    for (int t = g.t0; t < g.t1; t += TT) {
        float kx[8], vx[8], f[8], y[8];
        rk.widen(kx);
        rv.widen(vx);
        relu_rope8(kx, c4, s4, f, y);   // rows past the segment are zeros: phi and its rotation stay zero
#pragma unroll
        for (int i = 0; i < 8; ++i) zacc[i] += f[i];
        store4(&kt[tok][e0], y);
        store4(&kt[tok][e0 + 4], y + 4);
        store4(&vt[tok][e0], vx);
        store4(&vt[tok][e0 + 4], vx + 4);
        __syncthreads();
        if (t + TT < g.t1) fetch(t + TT);
        const int nt = min(TT, g.t1 - t);
        for (int u = 0; u < nt; ++u) {
            const float2 vv = *reinterpret_cast<const float2 *>(&vt[u][cl]);
            const float4 k0 = *reinterpret_cast<const float4 *>(&kt[u][ew]);
            const float4 k1 = *reinterpret_cast<const float4 *>(&kt[u][ew + 4]);
            const float va[2] = {vv.x, vv.y}, ka[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(va[a], ka[c], acc[a][c]);
        }
        __syncthreads();
    }
    // key sum: the four token rows of a warp (lanes j, j+8, j+16, j+24), then the warps in order
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        zacc[i] += __shfl_xor_sync(0xffffffffu, zacc[i], 8);
        zacc[i] += __shfl_xor_sync(0xffffffffu, zacc[i], 16);
    }
    if ((tid & 31) < 8)
#pragma unroll
        for (int i = 0; i < 8; ++i) zw[tid >> 5][e0 + i] = zacc[i];
    __syncthreads();
    float *dst = part + (((size_t)s * p.B + b) * p.H + h) * p.sz;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        store4(dst + (size_t)(cl + a) * D + ew, acc[a]);
        store4(dst + (size_t)(cl + a) * D + ew + 4, acc[a] + 4);
    }
    if (tid < D) {
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < THREADS / 32; ++w) z += zw[w][tid];
        dst[D * D + tid] = z;
    }
}

template <typename Tin, int D>
__global__ void __launch_bounds__(THREADS)
pass_c_gen(const Tin *__restrict__ q, const float *__restrict__ rc, const float *__restrict__ rs,
           const LclaPlan p, const float *__restrict__ pref, const float eps, Tin *__restrict__ out)
{
    constexpr int TC = 2 * TT;   // 64 tokens per tile: two token rows per loader thread, 8 per warp in the products
    static_assert(D == 64 && TC == 64, "thread mapping: 8 lanes x 8 dims per token row; 8 warps x 8 tokens, "
                                       "32 lanes x 2 channels");
    __shared__ __align__(16) float PT[D][D + 2];   // PT[e][c] = P[c][e]; rows padded for the transposing fill
    __shared__ float zs[D];
    // rotated query features transposed, qf[e][tok ^ 4 (e / 8)]: the fill (8 lanes per token, 8 dims each)
    // hits 32 banks, and the 8 tokens of a warp stay one 8-aligned group, its halves swapped when e / 8 is odd
    __shared__ __align__(16) float qf[D][TC];
    __shared__ float inv[TC];                  // 1 / (z . phi(q) + eps)
    const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const LclaSeg g = lcla_segment(p, s);
    pdl_wait();   // the prefixes come from the scan
    if (g.t1 <= g.t0) return;
    const float *P = pref + (((size_t)g.blk * p.B + b) * p.H + h) * p.sz;
    for (int x = tid; x < D * D; x += THREADS) PT[x % D][x / D] = P[x];
    if (tid < D) zs[tid] = P[D * D + tid];
    __syncthreads();
    const int j = tid & 7, e0 = j * 8;                      // features: 8 dims of token rows tid / 8 and + 32
    const int wg = tid >> 5, cl = (tid & 31) * 2;            // outputs: tokens [8 wg, 8 wg + 8), channels cl, cl + 1
    for (int t = g.t0; t < g.t1; t += TC) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int tok = (tid >> 3) + TT * r, n = t + tok;
            float x[8] = {}, f[8] = {}, y[8] = {};
            float dz = 0.f;
            if (n < g.t1) {
                load8(q + (((size_t)b * p.N + n) * p.H + h) * D + e0, x);
                const float4 c4 = *reinterpret_cast<const float4 *>(rc + (size_t)n * (D / 2) + j * 4);
                const float4 s4 = *reinterpret_cast<const float4 *>(rs + (size_t)n * (D / 2) + j * 4);
                relu_rope8(x, c4, s4, f, y);
#pragma unroll
                for (int i = 0; i < 8; ++i) dz = fmaf(f[i], zs[e0 + i], dz);
            }
            // z . phi(q) over the 8 lanes of this token row
            dz += __shfl_xor_sync(0xffffffffu, dz, 1);
            dz += __shfl_xor_sync(0xffffffffu, dz, 2);
            dz += __shfl_xor_sync(0xffffffffu, dz, 4);
#pragma unroll
            for (int i = 0; i < 8; ++i) qf[e0 + i][tok ^ (4 * j)] = y[i];   // rows e0..e0+7 have e / 8 = j
            if (j == 0) inv[tok] = 1.f / (dz + eps);
        }
        __syncthreads();
        float acc[8][2] = {};
#pragma unroll 8
        for (int e = 0; e < D; ++e) {
            const int g8 = 8 * (wg ^ (e >> 4)), hs = 4 * ((e >> 3) & 1);
            const float4 qa = *reinterpret_cast<const float4 *>(&qf[e][g8 + hs]);        // tokens 8 wg + 0..3
            const float4 qb = *reinterpret_cast<const float4 *>(&qf[e][g8 + (hs ^ 4)]);  // tokens 8 wg + 4..7
            const float2 pv = *reinterpret_cast<const float2 *>(&PT[e][cl]);
            const float qa8[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                acc[a][0] = fmaf(qa8[a], pv.x, acc[a][0]);
                acc[a][1] = fmaf(qa8[a], pv.y, acc[a][1]);
            }
        }
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int tk = 8 * wg + a, m = t + tk;
            if (m < g.t1) {
                const float r = inv[tk];
                store2(out + (((size_t)b * p.N + m) * p.H + h) * D + cl, acc[a][0] * r, acc[a][1] * r);
            }
        }
        __syncthreads();
    }
}

}  // namespace gen
}  // namespace lcla
