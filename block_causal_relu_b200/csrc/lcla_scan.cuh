// lcla_scan.cuh -- the block scan: segment partial states -> prefix states
// (inclusive per block in block mode, exclusive per segment in chunk mode),
// with the carried state in and the total out.
#pragma once
#include <stdint.h>

#include "lcla_common.cuh"
#include "lcla_plan.h"

namespace lcla {

// ---------------------------------------------------------------------------
// Scan: partials -> prefixes, one thread per 4 consecutive state elements
// (b, h, x..x+3) with x < (D+1)*D; the segment partials are loaded as float4
// in batches of independent loads and summed in a fixed order.
// Block mode: pref[blk] = state_in + sum of all segments of blocks <= blk.
// Chunk mode: pref[s]   = state_in + sum of segments < s.
// state_out (may equal state_in) receives the total.
// ---------------------------------------------------------------------------
constexpr int SCAN_THREADS = 128;
constexpr int SCAN_VEC = 4;   // elements per thread (a state's (d + 1) * d floats are a multiple of 4 for even d)

__device__ __forceinline__ void add4(float4 &a, const float4 &b)
{
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
}

// Chunked scan, for more groups than the grouped scan holds: the segments are
// cut into chunks of p.scs segments (whole groups).  scan_chunk_totals sums
// each chunk in segment order (grid: column blocks x chunks) and copies
// state_in after the chunk totals; scan_chunk_prefix starts each chunk from
// state_in plus the totals of the chunks before it, walks the chunk's
// segments and writes the same prefixes as the one-pass scans, and the last
// chunk writes the total.  Only the first kernel reads state_in, so state_out
// may alias it.
// ---------------------------------------------------------------------------
constexpr int SCAN_CHUNK_GROUPS = 32;

__global__ void __launch_bounds__(SCAN_THREADS)
scan_chunk_totals(const LclaPlan p, const float *__restrict__ part, const float *state_in, float *__restrict__ ctot)
{
    constexpr int BATCH = 16;
    const size_t n4 = (size_t)p.B * p.H * (p.sz / SCAN_VEC);
    const size_t x = (size_t)blockIdx.x * SCAN_THREADS + threadIdx.x;
    const int c = blockIdx.y;
    pdl_wait();
    pdl_trigger();
    if (x >= n4) return;
    const float4 *part4 = reinterpret_cast<const float4 *>(part);
    float4 *ctot4 = reinterpret_cast<float4 *>(ctot);
    const int s0 = c * p.scs, s1 = min(s0 + p.scs, p.nseg);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sb = s0; sb < s1; sb += BATCH) {
        float4 v[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j)
            if (sb + j < s1) v[j] = __ldcg(part4 + (size_t)(sb + j) * n4 + x);
#pragma unroll
        for (int j = 0; j < BATCH; ++j)
            if (sb + j < s1) add4(acc, v[j]);
    }
    ctot4[(size_t)c * n4 + x] = acc;
    if (c == 0)
        ctot4[(size_t)p.nch * n4 + x] = state_in ? reinterpret_cast<const float4 *>(state_in)[x]
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void __launch_bounds__(SCAN_THREADS)
scan_chunk_prefix(const LclaPlan p, const float *__restrict__ part, const float *__restrict__ ctot,
                  float *__restrict__ pref, float *state_out)
{
    constexpr int BATCH = 16;
    const size_t n4 = (size_t)p.B * p.H * (p.sz / SCAN_VEC);
    const size_t x = (size_t)blockIdx.x * SCAN_THREADS + threadIdx.x;
    const int c = blockIdx.y;
    pdl_wait();
    pdl_trigger();
    if (x >= n4) return;
    const float4 *part4 = reinterpret_cast<const float4 *>(part);
    const float4 *ctot4 = reinterpret_cast<const float4 *>(ctot);
    float4 *pref4 = reinterpret_cast<float4 *>(pref);
    float4 acc = __ldcg(ctot4 + (size_t)p.nch * n4 + x);   // state_in
    for (int cb = 0; cb < c; cb += BATCH) {
        float4 v[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j)
            if (cb + j < c) v[j] = __ldcg(ctot4 + (size_t)(cb + j) * n4 + x);
#pragma unroll
        for (int j = 0; j < BATCH; ++j)
            if (cb + j < c) add4(acc, v[j]);
    }
    const int s0 = c * p.scs, s1 = min(s0 + p.scs, p.nseg);
    for (int sb = s0; sb < s1; sb += BATCH) {
        float4 v[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j)
            if (sb + j < s1) v[j] = __ldcg(part4 + (size_t)(sb + j) * n4 + x);
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            const int sg = sb + j;
            if (sg < s1) {
                if (p.chunk) pref4[(size_t)sg * n4 + x] = acc;
                add4(acc, v[j]);
                if (!p.chunk && (sg + 1) % p.nsb == 0) pref4[(size_t)(sg / p.nsb) * n4 + x] = acc;
            }
        }
    }
    if (state_out && c == p.nch - 1) reinterpret_cast<float4 *>(state_out)[x] = acc;
}

// Grouped scan: the same prefixes in two phases, for up to SCANG_MAX_GROUPS
// groups (block mode: a block's nsb segments; chunk mode: one segment).  A
// CTA owns 32 float4 columns of the state slice; phase 1 has its 8 warps sum
// the groups' segment partials in parallel (all loads of a group in flight)
// into shared memory; phase 2 has one warp run the prefix over the group sums
// in group order and write pref (inclusive per block in block mode,
// exclusive per segment in chunk mode) and the total.
// ---------------------------------------------------------------------------
constexpr int SCANG_WARPS = 8;
constexpr int SCANG_MAX_GROUPS = 256;   // shared memory: groups x 32 x 16 B

__device__ __forceinline__ void st_v4_keep(float4 *p, float4 v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;"
                 ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}

__global__ void __launch_bounds__(32 * SCANG_WARPS)
scan_states_grouped(const LclaPlan p, const float *__restrict__ part, float *__restrict__ pref,
                    const float *state_in, float *state_out)
{
    extern __shared__ float4 gsum[];   // [groups][32]
    const size_t n4 = (size_t)p.B * p.H * (p.sz / SCAN_VEC);
    const int lane = threadIdx.x & 31, wg = threadIdx.x >> 5;
    const size_t x = (size_t)blockIdx.x * 32 + lane;
    const bool live = x < n4;
    const int ngroups = p.chunk ? p.nseg : p.nb, per = p.chunk ? 1 : p.nsb;
    const float4 *part4 = reinterpret_cast<const float4 *>(part);
    pdl_wait();
    pdl_trigger();
    for (int gi = wg; gi < ngroups; gi += SCANG_WARPS) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (live) {
            constexpr int BATCH = 8;
            for (int s0 = 0; s0 < per; s0 += BATCH) {
                float4 v[BATCH];
#pragma unroll
                for (int j = 0; j < BATCH; ++j)
                    if (s0 + j < per) v[j] = __ldcg(part4 + ((size_t)gi * per + s0 + j) * n4 + x);
#pragma unroll
                for (int j = 0; j < BATCH; ++j)
                    if (s0 + j < per) add4(acc, v[j]);
            }
        }
        gsum[gi * 32 + lane] = acc;
    }
    __syncthreads();
    if (wg == 0 && live) {
        float4 *pref4 = reinterpret_cast<float4 *>(pref);
        float4 acc = state_in ? reinterpret_cast<const float4 *>(state_in)[x] : make_float4(0.f, 0.f, 0.f, 0.f);
        uint64_t keep;   // the prefixes are read back by the next kernel: keep them in L2
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
        for (int gi = 0; gi < ngroups; ++gi) {
            const float4 v = gsum[gi * 32 + lane];
            if (p.chunk) st_v4_keep(pref4 + (size_t)gi * n4 + x, acc, keep);
            add4(acc, v);
            if (!p.chunk) st_v4_keep(pref4 + (size_t)gi * n4 + x, acc, keep);
        }
        if (state_out) reinterpret_cast<float4 *>(state_out)[x] = acc;
    }
}

}  // namespace lcla
