// lcla_tconv.cu -- causal temporal convolution of the Mix-FFN with a cached
// last frame (lcla_temporal_conv in include/lcla.h).
//
// The pages put a causal Mix-FFN after the attention of each block and say it
// keeps the previous block's last frame for its temporal convolution ("Block
// Causal Linear Attention", section "What SANA-Video Actually Uses"; "[feat]
// LongSANA" pull request: causal computation for the linear attention and for
// the Mix-FFN, the convolution in the MLP).  The kernel size is not on the
// pages; a single retained frame is read as a causal depthwise convolution of
// size 2 over latent frames:
//   y[b, f, s, c] = w[0][c] x[b, f, s, c] + w[1][c] x[b, f-1, s, c] + bias[c]
// with x[b, -1, s, c] the cached frame (zeros without one); with save the
// cache becomes x[b, F-1, s, c].
//
// Layout: x, y [B, F * S, C] token-major (token f * S + s), cache [B, S, C],
// weight [2][C] and bias [C] fp32.  One thread owns 8 consecutive channels of
// one (b, s) and walks the frames in order with the previous frame in
// registers: x is read once, y written once, the cache read and written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lcla.h"

namespace {

constexpr int kVec = 8;        // channels per thread
constexpr int kThreads = 256;

struct V8 {
    float x[kVec];
};

__device__ __forceinline__ V8 load8(const float *p)
{
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    return V8{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}
__device__ __forceinline__ V8 load8(const __nv_bfloat16 *p)
{
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    V8 r;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        r.x[2 * j] = __uint_as_float(w[j] << 16);
        r.x[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
    return r;
}
__device__ __forceinline__ void store8(float *p, const V8 &v)
{
    reinterpret_cast<float4 *>(p)[0] = make_float4(v.x[0], v.x[1], v.x[2], v.x[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v.x[4], v.x[5], v.x[6], v.x[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const V8 &v)
{
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v.x[2 * j], v.x[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
temporal_conv_k2(const T *__restrict__ x, int B, int F, int S, int C, const float *__restrict__ weight,
                 const float *__restrict__ bias, const T *cache_in, T *cache_out, T *__restrict__ y)
{
    const int nv = C / kVec;
    const long long idx = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (idx >= (long long)B * S * nv) return;
    const int cv = (int)(idx % nv);
    const long long bs = idx / nv;
    const int s = (int)(bs % S), b = (int)(bs / S), c0 = cv * kVec;
    const V8 w0 = load8(weight + c0), w1 = load8(weight + C + c0);
    V8 bb = {{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}};
    if (bias) bb = load8(bias + c0);
    const size_t cache_at = ((size_t)b * S + s) * C + c0;
    V8 prev = {{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}};
    if (cache_in) prev = load8(cache_in + cache_at);
    const size_t frame = (size_t)S * C;
    size_t at = ((size_t)b * F * S + s) * C + c0;
    for (int f = 0; f < F; ++f, at += frame) {
        const V8 cur = load8(x + at);
        V8 out;
#pragma unroll
        for (int j = 0; j < kVec; ++j) out.x[j] = fmaf(w0.x[j], cur.x[j], fmaf(w1.x[j], prev.x[j], bb.x[j]));
        store8(y + at, out);
        prev = cur;
    }
    // the last frame's widened values are exact, so the cache round-trips bit for bit
    if (cache_out && F > 0) store8(cache_out + cache_at, prev);
}

bool misaligned16(const void *p) { return ((uintptr_t)p & 15u) != 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    if (!a || !b || !na || !nb) return false;
    const uintptr_t a0 = (uintptr_t)a, a1 = a0 + na, b0 = (uintptr_t)b, b1 = b0 + nb;
    return a0 < b1 && b0 < a1;
}

}  // namespace

extern "C" int lcla_temporal_conv(const void *x, int B, int F, int S, int C, const float *weight,
                                  const float *bias, void *cache, int save, void *y, int dtype, void *stream)
{
    if (B < 1 || F < 0 || S < 1 || C < kVec || (C % kVec) != 0) return LCLA_ERR_INVALID_ARG;
    if (dtype != LCLA_BF16 && dtype != LCLA_F32) return LCLA_ERR_INVALID_ARG;
    if ((long long)B * F * S > (1ll << 31) || (long long)B * S * C > (1ll << 40)) return LCLA_ERR_UNSUPPORTED;
    if (F == 0) return LCLA_OK;   // no frames: nothing to write, the cache keeps its frame
    if (!x || !y || !weight) return LCLA_ERR_INVALID_ARG;
    if (misaligned16(x) || misaligned16(y) || misaligned16(weight) || (bias && misaligned16(bias)) ||
        (cache && misaligned16(cache)))
        return LCLA_ERR_MISALIGNED;
    const size_t esz = dtype == LCLA_BF16 ? 2 : 4;
    const size_t nx = (size_t)B * F * S * C * esz, nc = (size_t)B * S * C * esz;
    if (overlaps(y, nx, x, nx) || overlaps(y, nx, cache, nc) || overlaps(y, nx, weight, 2 * C * 4) ||
        overlaps(y, nx, bias, C * 4) || overlaps(cache, nc, x, nx))
        return LCLA_ERR_INVALID_ARG;
    const long long nthreads = (long long)B * S * (C / kVec);
    const dim3 grid((unsigned)((nthreads + kThreads - 1) / kThreads));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == LCLA_BF16) {
        __nv_bfloat16 *c = static_cast<__nv_bfloat16 *>(cache);
        temporal_conv_k2<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(x), B, F, S, C, weight, bias, c, save ? c : nullptr,
            static_cast<__nv_bfloat16 *>(y));
    } else {
        float *c = static_cast<float *>(cache);
        temporal_conv_k2<float><<<grid, kThreads, 0, st>>>(static_cast<const float *>(x), B, F, S, C, weight,
                                                            bias, c, save ? c : nullptr, static_cast<float *>(y));
    }
    return cudaGetLastError() == cudaSuccess ? LCLA_OK : LCLA_ERR_CUDA;
}
