// lcla_common.cuh -- device helpers shared by the kernels: cp.async staging,
// programmatic dependent launch, ReLU, bf16 unpacking, 8- and 4-element loads
// and stores, phi plus the rotary embedding on 8 elements, and the tile
// geometry and row staging of the CUDA-core passes.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "lcla_plan.h"

namespace lcla {

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Programmatic dependent launch: wait until the preceding kernel of the
// stream has completed (no-op when launched without the attribute), and let
// the next kernel of the stream start its launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ReLU written as a comparison so that NaN passes through.
__device__ __forceinline__ float relu(float x) { return x < 0.f ? 0.f : x; }

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 8 consecutive elements -> fp32
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *x)
{
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    x[0] = bf_lo(u.x); x[1] = bf_hi(u.x); x[2] = bf_lo(u.y); x[3] = bf_hi(u.y);
    x[4] = bf_lo(u.z); x[5] = bf_hi(u.z); x[6] = bf_lo(u.w); x[7] = bf_hi(u.w);
}
__device__ __forceinline__ void load8(const float *p, float *x)
{
    const float4 a = reinterpret_cast<const float4 *>(p)[0];
    const float4 b = reinterpret_cast<const float4 *>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// 4 consecutive elements -> fp32
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float *x)
{
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    x[0] = bf_lo(u.x); x[1] = bf_hi(u.x); x[2] = bf_lo(u.y); x[3] = bf_hi(u.y);
}
__device__ __forceinline__ void load4(const float *p, float *x)
{
    const float4 a = *reinterpret_cast<const float4 *>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
// 4 fp32 -> 4 consecutive outputs (bf16 round-to-nearest-even)
__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float *x)
{
    __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}
__device__ __forceinline__ void store4(float *p, const float *x)
{
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}

// phi then the rotary embedding on 8 consecutive elements (4 pairs) of a head
// row; x holds the raw values on entry, f the ReLU features and y the rotated
// features on exit.  c4/s4 are the 4 table entries of these pairs.
__device__ __forceinline__ void relu_rope8(const float *x, const float4 &c4, const float4 &s4,
                                           float *f, float *y)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = relu(x[i]);
    const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
    const float ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float a = f[2 * p], b = f[2 * p + 1];
        y[2 * p] = a * cc[p] - b * ss[p];
        y[2 * p + 1] = a * ss[p] + b * cc[p];
    }
}

// Tile geometry for one input type.
template <typename Tin>
struct Geo {
    static constexpr int EB = (int)sizeof(Tin);
    static constexpr int ROWB = LCLA_D * EB;                  // bytes of one head row
    static constexpr int CPR = ROWB / 16;                     // 16-byte chunks per head row
    static constexpr int TILE_IN = LCLA_T * LCLA_HG * ROWB;   // one input tile [T][HG][D]
    static constexpr int TILE_TAB = LCLA_T * (LCLA_D / 2) * 4; // one table tile [T][D/2] fp32
    static constexpr int TILE_F = LCLA_T * LCLA_HG * LCLA_D * 4; // fp32 tile [T][HG][D]
};

// Queue cp.async copies of rows [t, t + nt) of an input tensor for heads
// h0, h0+1 into buf ([T][HG][D] elements); rows and heads outside the valid
// range are zero-filled without reading global memory.
template <typename Tin>
__device__ __forceinline__ void issue_rows(unsigned char *buf, const Tin *src, const LclaPlan &p,
                                           int b, int t, int nt, int h0, int tid, int nthr)
{
    using G = Geo<Tin>;
    for (int c = tid; c < LCLA_T * LCLA_HG * G::CPR; c += nthr) {
        const int tok = c / (LCLA_HG * G::CPR);
        const int rem = c - tok * (LCLA_HG * G::CPR);
        const int hh = rem / G::CPR;
        const int part = rem - hh * G::CPR;
        const bool ok = tok < nt && h0 + hh < p.H;
        const size_t off = ok ? ((((size_t)b * p.N + (size_t)(t + tok)) * p.H + (size_t)(h0 + hh)) *
                                     LCLA_D) * G::EB + (size_t)part * 16
                              : 0;
        cp_async16(buf + (size_t)c * 16, reinterpret_cast<const unsigned char *>(src) + off, ok);
    }
}

// Same for the [N, D/2] fp32 tables.
__device__ __forceinline__ void issue_table(unsigned char *buf, const float *tab, int t, int nt,
                                            int tid, int nthr)
{
    for (int c = tid; c < LCLA_T * 4; c += nthr) {
        const int tok = c >> 2, part = c & 3;
        const bool ok = tok < nt;
        const size_t off = ok ? (size_t)(t + tok) * (LCLA_D / 2) * 4 + (size_t)part * 16 : 0;
        cp_async16(buf + (size_t)c * 16, reinterpret_cast<const unsigned char *>(tab) + off, ok);
    }
}

}  // namespace lcla
