// lcla_tc.cuh -- tensor-core (tcgen05 + TMA) kernels: bf16 inputs, block mode.
//
// Same two passes as the CUDA-core path ("Implementing Block Causal Linear
// Attention for Long Video Generation with Sana", section "The Linear
// Attention Kernel": vk = v k_rotated^T, out = vk q_rotated, normaliser from
// the unrotated key sum; section "Rotary Position Embeddings": rotary on the
// ReLU features), with the d x d contractions on the 5th-generation tensor
// cores:
//
// Two CTAs of 256 threads reside on each SM (about 105 KB of shared memory
// each), so one CTA's barriers overlap the other's work.  Tiles hold 64
// tokens; two threads share each (token, head) row, 16 elements each.
//
// Pass A, per CTA = (segment inside one block, head pair, batch entry).  The
// rotated keys are split into bf16 hi + lo parts
// (k~ = hi + lo to 2^-16 relative) and stacked as the 128 rows of the MMA's A
// operand, [hi_h0; lo_h0; hi_h1; lo_h1] (MN-major, written by the threads);
// V of the two heads is the B operand exactly as TMA lands it (MN-major,
// 128-byte swizzle).  D[128 x 64] in tensor memory holds
//   D[part*32 + e][c] = sum_tok part(k~)[tok][e] * v[tok][c]
// for both heads (the off-diagonal head blocks are unused).  Each tile's D is
// read back and added into fp32 registers, so no long accumulation chain runs
// inside the tensor core.  The unrotated key sum z is accumulated on the CUDA
// cores from the same ReLU features.
//
// Pass C, per CTA = (segment, head pair, batch entry): the block's prefix
// state P of both heads is split once into bf16 hi + lo and staged as the B
// operand (K-major rows (head, c) = [P hi | P lo]); per 64-token tile the
// rotated queries of both heads, split into hi + lo, are the 128 rows
// (head, token) of the A operand (K-major) and
//   D[(h,tok)][(h',c)] = q~hi.Phi + q~lo.Phi + q~hi.Plo   (6 MMAs of K = 16)
// (blocks h = h' used) is scaled by 1 / (z . phi(q) + eps) and stored
// through TMA.
//
// Every wait on an mbarrier is bounded (LCLA_TC_WAIT_NS of globaltimer); a
// timeout is voted across the CTA, the CTA waits (bounded) for its own
// copies and MMAs in flight, frees its tensor memory, poisons its partial
// state with NaN, sets the caller-visible status word and returns.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lcla_ffma.cuh"
#include "lcla_plan.h"

#define LCLA_TC_WAIT_NS 1000000000ull   // 1 s: far above any legitimate wait

namespace lcla {
namespace tc {

constexpr int T = LCLA_TC_T;

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t s32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t gtimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase with the given parity to complete.
__device__ __noinline__ bool bar_wait(uint32_t bar, uint32_t parity)
{
    if (bar_try(bar, parity)) return true;
    const uint64_t t0 = gtimer();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (bar_try(bar, parity)) return true;
        if (gtimer() - t0 > LCLA_TC_WAIT_NS) return false;
    }
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tma_load3(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tma_load2(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tma_store3(const CUtensorMap *map, uint32_t src, int x, int y, int z)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
                 ::"l"((uint64_t)map), "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier when every MMA issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 32 lanes x 16 columns of 32 bits: thread t of the warp gets lane (quarter*32 + t).
__device__ __forceinline__ void tmem_ld16(uint32_t ta, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(ta));
}
__device__ __forceinline__ void tmem_ld32(uint32_t ta, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(ta));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout, version 1).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D.
constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }

// Rotate 16 pairs of ReLU features and split each rotated value into bf16 hi + lo.
__device__ __forceinline__ void rope_split(const float *f, const float *cv, const float *sv, uint32_t *hi, uint32_t *lo)
{
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        const float a = f[2 * p], b = f[2 * p + 1];
        const float y0 = a * cv[p] - b * sv[p];
        const float y1 = a * sv[p] + b * cv[p];
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
        const float2 hf = __bfloat1622float2(h2);
        hi[p] = bf2_bits(h2);
        lo[p] = bf2_bits(__floats2bfloat162_rn(y0 - hf.x, y1 - hf.y));
    }
}

// ReLU on two packed bf16 (NaN passes through).
__device__ __forceinline__ uint32_t relu2(uint32_t w)
{
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&w);
    x = __hmax2_nan(x, __floats2bfloat162_rn(0.f, 0.f));
    return bf2_bits(x);
}

// Elements [16f, 16f+16) of head h in row r of a [64][64] bf16 tile with
// 128-byte swizzle, as 8 packed bf16 pairs.
__device__ __forceinline__ void load_half_row(const unsigned char *tile, int r, int h, int f, uint32_t *w)
{
    const int sw = r & 7;
    const uint4 a = *reinterpret_cast<const uint4 *>(tile + r * 128 + (((4 * h + 2 * f) ^ sw) << 4));
    const uint4 b = *reinterpret_cast<const uint4 *>(tile + r * 128 + (((4 * h + 2 * f + 1) ^ sw) << 4));
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}
// Pairs [8f, 8f+8) of row r of a [64][16] fp32 table tile with 64-byte swizzle.
__device__ __forceinline__ void load_half_table(const unsigned char *tile, int r, int f, float *x)
{
    const int sw = (r >> 1) & 3;
    const float4 a = *reinterpret_cast<const float4 *>(tile + r * 64 + (((2 * f) ^ sw) << 4));
    const float4 b = *reinterpret_cast<const float4 *>(tile + r * 64 + (((2 * f + 1) ^ sw) << 4));
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// Rotate 8 pairs of (packed bf16) ReLU features and split each rotated value
// into bf16 hi + lo (packed pairs).
__device__ __forceinline__ void rope_split8(const uint32_t *fw, const float *cv, const float *sv, uint32_t *hi,
                                            uint32_t *lo)
{
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const float a = bf_lo(fw[p]), b = bf_hi(fw[p]);
        const float y0 = a * cv[p] - b * sv[p];
        const float y1 = a * sv[p] + b * cv[p];
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
        const float2 hf = __bfloat1622float2(h2);
        hi[p] = bf2_bits(h2);
        lo[p] = bf2_bits(__floats2bfloat162_rn(y0 - hf.x, y1 - hf.y));
    }
}
// Half f of operand row r (128 B, 128-byte swizzle): hi -> chunks 2f, 2f+1; lo -> chunks 4+2f, 5+2f.
__device__ __forceinline__ void store_half_hi_lo(unsigned char *tile, int r, int f, const uint32_t *hi,
                                                 const uint32_t *lo)
{
    const int sw = r & 7;
    unsigned char *row = tile + r * 128;
    *reinterpret_cast<uint4 *>(row + (((2 * f) ^ sw) << 4)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4 *>(row + (((2 * f + 1) ^ sw) << 4)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
    *reinterpret_cast<uint4 *>(row + (((4 + 2 * f) ^ sw) << 4)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint4 *>(row + (((5 + 2 * f) ^ sw) << 4)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
}

// ---------------------------------------------------------------------------
// Pass A
// ---------------------------------------------------------------------------
struct LayA {
    static constexpr int STAGES = 3;
    static constexpr int K_OFF = 0, V_OFF = 8192, C_OFF = 16384, S_OFF = 20480, STAGE = 24576;
    static constexpr int A_OFF = STAGES * STAGE, A_BYTES = 16384;   // per buffer: head 0 | head 1, [64 tok][128 B]
    static constexpr int CTRL = A_OFF + 2 * A_BYTES;
    static constexpr int BYTES = CTRL + 128 + 1024;                 // + alignment slack
    static constexpr uint32_t TX = STAGE;
    static constexpr uint32_t IDESC = idesc_bf16(128, 64, 1, 1);
};

__global__ void __launch_bounds__(256, 2)
pass_a_tc(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
          const __grid_constant__ CUtensorMap mc, const __grid_constant__ CUtensorMap ms,
          const LclaPlan p, float *__restrict__ part, int *__restrict__ status)
{
    using L = LayA;
    extern __shared__ unsigned char smraw[];
    const uint32_t raw = s32(smraw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    unsigned char *sm = smraw + pad;
    const uint32_t sb = raw + pad;
    const uint32_t full0 = sb + L::CTRL, done0 = full0 + 8 * L::STAGES;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::CTRL + 64);

    const int s = blockIdx.x / p.ngroups, hp = blockIdx.x % p.ngroups, b = blockIdx.y;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const LclaSeg g = lcla_segment(p, s);
    const int ntile = g.t1 > g.t0 ? (g.t1 - g.t0 + T - 1) / T : 0;

    if (tid == 0) {
        for (int i = 0; i < L::STAGES; ++i) bar_init(full0 + 8 * i, 1);
        for (int i = 0; i < 2; ++i) bar_init(done0 + 8 * i, 1);
        bar_fence_init();
    }
    if (w == 0) {
        tmem_alloc(s32(tslot), 128);
        tmem_relinquish();
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tslot;

    const int r = tid & 63, h = (tid >> 6) & 1, f = tid >> 7;   // prologue: token row, head, half
    const int q4 = w & 3, ch = w >> 2;                            // drain: lane quarter, column half

    float zacc[16], sacc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) zacc[j] = sacc[j] = 0.f;
    int loaded = 0, consumed = 0, issued = 0, drained = 0;
    bool bad = false;

    auto load = [&](int i) {
        const int st = i % L::STAGES;
        const uint32_t base = sb + st * L::STAGE, fb = full0 + 8 * st;
        const int t = g.t0 + i * T;
        bar_expect_tx(fb, L::TX);
        tma_load3(base + L::K_OFF, &mk, fb, 64 * hp, t, b);
        tma_load3(base + L::V_OFF, &mv, fb, 64 * hp, t, b);
        tma_load2(base + L::C_OFF, &mc, fb, 0, t);
        tma_load2(base + L::S_OFF, &ms, fb, 0, t);
    };
    auto drain = [&](int buf) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(q4 * 32) << 16) + buf * 64 + (q4 >> 1) * 32 + ch * 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) sacc[j] += __uint_as_float(v[j]);
    };

    if (tid == 0)
        for (; loaded < L::STAGES - 1 && loaded < ntile; ++loaded) load(loaded);

    for (int i = 0; i < ntile; ++i) {
        const int st = i % L::STAGES, ab = i & 1;
        unsigned char *stg = sm + st * L::STAGE;
        const int t = g.t0 + i * T, nt = min(T, g.t1 - t);

        bool ok = bar_wait(full0 + 8 * st, (uint32_t)((i / L::STAGES) & 1));
        {   // phi, key sum, rotary, hi/lo split -> A operand (MN-major) of token r, head h, half f
            const bool valid = ok && r < nt;
            uint32_t fw[8], hi[8], lo[8];
            float cv[8], sv[8];
            load_half_row(stg + L::K_OFF, r, h, f, fw);
            load_half_table(stg + L::C_OFF, r, f, cv);
            load_half_table(stg + L::S_OFF, r, f, sv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                fw[j] = valid ? relu2(fw[j]) : 0u;
                zacc[2 * j] += bf_lo(fw[j]);
                zacc[2 * j + 1] += bf_hi(fw[j]);
            }
            rope_split8(fw, cv, sv, hi, lo);
            store_half_hi_lo(sm + L::A_OFF + ab * L::A_BYTES + h * 8192, r, f, hi, lo);
            if (!valid) {   // rows past the segment belong to another CTA: zero this half of V
                const int sw = r & 7;
                *reinterpret_cast<uint4 *>(stg + L::V_OFF + r * 128 + (((4 * h + 2 * f) ^ sw) << 4)) =
                    make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(stg + L::V_OFF + r * 128 + (((4 * h + 2 * f + 1) ^ sw) << 4)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
        }
        fence_async_smem();
        if (__syncthreads_or(!ok)) { bad = true; break; }
        consumed = i + 1;

        if (tid == 0) {
            tc_after();
            const uint32_t d = tmem + ab * 64;
            const uint32_t a0 = sb + L::A_OFF + ab * L::A_BYTES;
            const uint32_t v0 = sb + st * L::STAGE + L::V_OFF;
#pragma unroll
            for (int j = 0; j < T / 16; ++j)
                mma_bf16(d, desc_sw128(a0 + 2048 * j, 8192, 1024), desc_sw128(v0 + 2048 * j, 8192, 1024),
                         L::IDESC, j > 0);
            mma_commit(done0 + 8 * ab);
        }
        issued = i + 1;

        ok = true;
        if (i >= 1) {
            ok = bar_wait(done0 + 8 * ((i - 1) & 1), (uint32_t)(((i - 1) >> 1) & 1));
            if (ok) {
                tc_after();
                drain((i - 1) & 1);
            }
        }
        tc_before();
        if (__syncthreads_or(!ok)) { bad = true; break; }
        drained = i;
        if (tid == 0 && loaded < ntile) { load(loaded); ++loaded; }
    }
    if (!bad && ntile > 0) {
        const bool ok = bar_wait(done0 + 8 * ((ntile - 1) & 1), (uint32_t)(((ntile - 1) >> 1) & 1));
        if (ok) {
            tc_after();
            drain((ntile - 1) & 1);
        }
        if (__syncthreads_or(!ok)) bad = true;
        else drained = ntile;
    }
    if (bad && tid == 0) {   // let this CTA's own copies and MMAs finish before leaving
        if (issued > drained) bar_wait(done0 + 8 * ((issued - 1) & 1), (uint32_t)(((issued - 1) >> 1) & 1));
        for (int j = consumed; j < loaded; ++j) bar_wait(full0 + 8 * (j % L::STAGES), (uint32_t)((j / L::STAGES) & 1));
    }
    tc_before();
    __syncthreads();

    pdl_trigger();
    // fixed-order reduction: S from the hi and lo quarters, z over the 64 threads of each (head, half)
    float *red = reinterpret_cast<float *>(sm);          // [4 quarters][32 e][32 c]
    float *zred = red + 4 * 32 * 32;                      // [256 threads][17]
#pragma unroll
    for (int j = 0; j < 16; ++j) red[(q4 * 32 + lane) * 32 + ch * 16 + j] = sacc[j];
#pragma unroll
    for (int j = 0; j < 16; ++j) zred[tid * 17 + j] = zacc[j];
    __syncthreads();
    const float nanv = __int_as_float(0x7fc00000);
    for (int x = tid; x < LCLA_HG * LCLA_SZ; x += 256) {
        const int hh = x / LCLA_SZ, e = x - hh * LCLA_SZ;
        float val;
        if (e < LCLA_D * LCLA_D) {
            const int c = e >> 5, ee = e & 31;
            val = red[((2 * hh) * 32 + ee) * 32 + c] + red[((2 * hh + 1) * 32 + ee) * 32 + c];
        } else {
            const int ez = e - LCLA_D * LCLA_D, ff = ez >> 4, j = ez & 15;
            const float *zr = zred + (ff * 128 + hh * 64) * 17 + j;
            val = 0.f;
            for (int rr = 0; rr < 64; ++rr) val += zr[rr * 17];
        }
        const int head = LCLA_HG * hp + hh;
        if (head < p.H) part[(((size_t)s * p.B + b) * p.H + head) * LCLA_SZ + e] = bad ? nanv : val;
    }
    if (bad && tid == 0) atomicOr(status, 1);
    tc_before();
    __syncthreads();
    if (w == 0) {
        tc_after();
        tmem_dealloc(tmem, 128);
    }
}

// ---------------------------------------------------------------------------
// Pass C
// ---------------------------------------------------------------------------
struct LayC {
    static constexpr int STAGES = 4;
    static constexpr int Q_OFF = 0, C_OFF = 8192, S_OFF = 12288, STAGE = 16384;
    static constexpr int A_OFF = STAGES * STAGE;          // [128 rows (head, token)][q~hi | q~lo]
    static constexpr int O_OFF = A_OFF + 16384;           // out tiles, 2 x [64 tok][128 B]
    static constexpr int B_OFF = O_OFF + 2 * 8192;        // [64 rows (head, c)][P hi | P lo]
    static constexpr int D_OFF = B_OFF + 8192;            // denominator halves [2 parity][2 h][2 f][64 r]
    static constexpr int CTRL = D_OFF + 2048;
    static constexpr int BYTES = CTRL + 128 + 1024;
    static constexpr uint32_t TX = STAGE;
    static constexpr uint32_t IDESC = idesc_bf16(128, 64, 0, 0);
};

__global__ void __launch_bounds__(256, 2)
pass_c_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mc,
          const __grid_constant__ CUtensorMap ms, const __grid_constant__ CUtensorMap mo,
          const LclaPlan p, const float *__restrict__ pref, const float eps,
          __nv_bfloat16 *__restrict__ out, int *__restrict__ status)
{
    using L = LayC;
    extern __shared__ unsigned char smraw[];
    const uint32_t raw = s32(smraw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    unsigned char *sm = smraw + pad;
    const uint32_t sb = raw + pad;
    const uint32_t full0 = sb + L::CTRL, done0 = full0 + 8 * L::STAGES;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::CTRL + 64);
    float *dens = reinterpret_cast<float *>(sm + L::D_OFF);

    const int s = blockIdx.x / p.ngroups, hp = blockIdx.x % p.ngroups, b = blockIdx.y;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const LclaSeg g = lcla_segment(p, s);
    const int ntile = g.t1 > g.t0 ? (g.t1 - g.t0 + T - 1) / T : 0;
    if (ntile == 0) return;

    if (tid == 0) {
        for (int i = 0; i < L::STAGES; ++i) bar_init(full0 + 8 * i, 1);
        for (int i = 0; i < 2; ++i) bar_init(done0 + 8 * i, 1);
        bar_fence_init();
    }
    if (w == 0) {
        tmem_alloc(s32(tslot), 128);
        tmem_relinquish();
    }
    int loaded = 0;
    auto load = [&](int i) {
        const int st = i % L::STAGES;
        const uint32_t base = sb + st * L::STAGE, fb = full0 + 8 * st;
        const int t = g.t0 + i * T;
        bar_expect_tx(fb, L::TX);
        tma_load3(base + L::Q_OFF, &mq, fb, 64 * hp, t, b);
        tma_load2(base + L::C_OFF, &mc, fb, 0, t);
        tma_load2(base + L::S_OFF, &ms, fb, 0, t);
    };
    if (tid == 0) {   // q and the tables are inputs: start streaming them before the prefixes exist
        for (; loaded < L::STAGES - 1 && loaded < ntile; ++loaded) load(loaded);
    }
    pdl_wait();
    const size_t pbase = ((size_t)g.blk * p.B + b) * p.H;
    // prefix state of this block -> B operand rows (head, c) = [P hi | P lo] (K-major)
    for (int x = tid; x < 64 * 8; x += 256) {
        const int n = x >> 3, j = x & 7, hh = n >> 5, c = n & 31;
        const int head = LCLA_HG * hp + hh;
        const float *P = pref + (pbase + (head < p.H ? head : 0)) * LCLA_SZ + c * LCLA_D + 8 * (j & 3);
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float y0 = head < p.H ? P[2 * m] : 0.f, y1 = head < p.H ? P[2 * m + 1] : 0.f;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
            const float2 hf = __bfloat1622float2(h2);
            hi[m] = bf2_bits(h2);
            lo[m] = bf2_bits(__floats2bfloat162_rn(y0 - hf.x, y1 - hf.y));
        }
        *reinterpret_cast<uint4 *>(sm + L::B_OFF + n * 128 + ((j ^ (n & 7)) << 4)) =
            j < 4 ? make_uint4(hi[0], hi[1], hi[2], hi[3]) : make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    fence_async_smem();
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tslot;

    const int r = tid & 63, h = (tid >> 6) & 1, f = tid >> 7;   // prologue: token row, head, half
    const int q4 = w & 3, ch = w >> 2;                            // epilogue: lane quarter, column half
    const int er = ((q4 & 1) << 5) | lane, eh = q4 >> 1;          // epilogue: token row, head
    const int ehead = LCLA_HG * hp + eh;
    float zr[16];
    {
        const int head = LCLA_HG * hp + h;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            zr[j] = head < p.H ? pref[(pbase + head) * LCLA_SZ + LCLA_D * LCLA_D + 16 * f + j] : 0.f;
    }
    int consumed = 0, issued = 0, drained = 0;
    bool bad = false;

    // outputs of tile i: this thread's 16 values of (token er, head eh), scaled and
    // written to the tile's out buffer (full tile, stored by TMA) or to global
    auto epilogue = [&](int i) {
        const int t = g.t0 + i * T, nt = min(T, g.t1 - t), par = i & 1;
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(q4 * 32) << 16) + par * 64 + eh * 32 + ch * 16, v);
        const float den = dens[((par * 2 + eh) * 2 + 0) * 64 + er] + dens[((par * 2 + eh) * 2 + 1) * 64 + er];
        const float inv = 1.0f / (den + eps);
        tmem_wait_ld();
        uint32_t o[8];
#pragma unroll
        for (int m = 0; m < 8; ++m)
            o[m] = bf2_bits(__floats2bfloat162_rn(__uint_as_float(v[2 * m]) * inv, __uint_as_float(v[2 * m + 1]) * inv));
        if (nt == T) {
            unsigned char *row = sm + L::O_OFF + par * 8192 + er * 128;
            const int sw = er & 7;
            *reinterpret_cast<uint4 *>(row + (((4 * eh + 2 * ch) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4 *>(row + (((4 * eh + 2 * ch + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        } else if (er < nt && ehead < p.H) {
            uint4 *dst = reinterpret_cast<uint4 *>(out + (((size_t)b * p.N + (size_t)(t + er)) * p.H + ehead) * LCLA_D +
                                                   16 * ch);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
    };
    auto store_tile = [&](int i) {   // thread 0: TMA store of a full tile's outputs
        const int t = g.t0 + i * T;
        if (g.t1 - t >= T) tma_store3(&mo, sb + L::O_OFF + (i & 1) * 8192, 64 * hp, t, b);
        bulk_commit();
    };

    for (int i = 0; i < ntile; ++i) {
        const int st = i % L::STAGES, par = i & 1;
        unsigned char *stg = sm + st * L::STAGE;

        bool ok = bar_wait(full0 + 8 * st, (uint32_t)((i / L::STAGES) & 1));
        if (i >= 1)   // the single A buffer is free once MMA(i-1) is done
            ok = bar_wait(done0 + 8 * ((i - 1) & 1), (uint32_t)(((i - 1) >> 1) & 1)) && ok;
        {   // phi, denominator half, rotary, hi/lo split -> A operand row (head h, token r)
            uint32_t fw[8], hi[8], lo[8];
            float cv[8], sv[8];
            load_half_row(stg + L::Q_OFF, r, h, f, fw);
            load_half_table(stg + L::C_OFF, r, f, cv);
            load_half_table(stg + L::S_OFF, r, f, sv);
            float den = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                fw[j] = relu2(fw[j]);
                den = fmaf(bf_lo(fw[j]), zr[2 * j], den);
                den = fmaf(bf_hi(fw[j]), zr[2 * j + 1], den);
            }
            dens[((par * 2 + h) * 2 + f) * 64 + r] = den;
            rope_split8(fw, cv, sv, hi, lo);
            store_half_hi_lo(sm + L::A_OFF, 64 * h + r, f, hi, lo);
        }
        fence_async_smem();
        if (__syncthreads_or(!ok)) { bad = true; break; }
        consumed = i + 1;

        if (tid == 0) {
            tc_after();
            const uint32_t d = tmem + par * 64;
            const uint32_t a0 = sb + L::A_OFF, b0 = sb + L::B_OFF;
#pragma unroll
            for (int j = 0; j < 4; ++j)      // q~hi.P hi + q~lo.P hi
                mma_bf16(d, desc_sw128(a0 + 32 * j, 16, 1024), desc_sw128(b0 + 32 * (j & 1), 16, 1024), L::IDESC, j > 0);
#pragma unroll
            for (int j = 0; j < 2; ++j)      // + q~hi.P lo
                mma_bf16(d, desc_sw128(a0 + 32 * j, 16, 1024), desc_sw128(b0 + 64 + 32 * j, 16, 1024), L::IDESC, 1);
            mma_commit(done0 + 8 * par);
        }
        issued = i + 1;

        if (i >= 1) {   // MMA(i-1) completion was observed above by every thread
            tc_after();
            epilogue(i - 1);
        }
        fence_async_smem();
        tc_before();
        __syncthreads();
        drained = i;
        if (tid == 0) {
            if (i >= 1) {
                store_tile(i - 1);
                bulk_wait_read1();   // the out buffer written next has been read by its store
            }
            if (loaded < ntile) { load(loaded); ++loaded; }
        }
    }
    if (!bad) {
        const bool ok = bar_wait(done0 + 8 * ((ntile - 1) & 1), (uint32_t)(((ntile - 1) >> 1) & 1));
        if (ok) {
            tc_after();
            epilogue(ntile - 1);
        }
        fence_async_smem();
        tc_before();
        if (__syncthreads_or(!ok)) {
            bad = true;
        } else {
            drained = ntile;
            if (tid == 0) store_tile(ntile - 1);
        }
    }
    if (tid == 0) {
        if (bad) {
            if (issued > drained) bar_wait(done0 + 8 * ((issued - 1) & 1), (uint32_t)(((issued - 1) >> 1) & 1));
            for (int j = consumed; j < loaded; ++j) bar_wait(full0 + 8 * (j % L::STAGES), (uint32_t)((j / L::STAGES) & 1));
            atomicOr(status, 2);
        }
        bulk_wait_all();
    }
    tc_before();
    __syncthreads();
    if (w == 0) {
        tc_after();
        tmem_dealloc(tmem, 128);
    }
}

}  // namespace tc
}  // namespace lcla
