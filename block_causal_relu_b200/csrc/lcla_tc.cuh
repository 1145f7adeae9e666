// lcla_tc.cuh -- tensor-core (tcgen05 + TMA) kernels: bf16 inputs, block mode.
//
// Same two passes as the CUDA-core path ("Implementing Block Causal Linear
// Attention for Long Video Generation with Sana", section "The Linear
// Attention Kernel": vk = v k_rotated^T, out = vk q_rotated, normaliser from
// the unrotated key sum; section "Rotary Position Embeddings": rotary on the
// ReLU features), with the d x d contractions on the 5th-generation tensor
// cores.
//
// Both kernels are persistent (one CTA per SM, looping over work units =
// (segment, head pair, batch entry), head pair fastest) and warp-specialised:
//   producer warp   TMA loads of 64-token tiles into a deep ring of stages;
//   MMA warp        one thread issues tcgen05.mma and tcgen05.commit;
//   prologue warps  ReLU, rotary, bf16 hi/lo split into the MMA operand;
//   drain/epilogue  tensor memory -> registers -> partial states / outputs.
// Roles talk only through mbarriers, so loads run as far ahead as the ring
// allows, independently of the compute.
//
// Pass A.  The rotated keys k~ of a head pair are split into bf16 hi + lo
// (k~ = hi + lo to 2^-16 relative) and stacked as the 128 rows of the A
// operand, [hi_h0; lo_h0; hi_h1; lo_h1] (MN-major, written by the threads);
// V of the two heads is the B operand exactly as TMA lands it (MN-major,
// 128-byte swizzle):  D[part*32 + e][c] = sum_tok part(k~)[tok][e] v[tok][c].
// The unrotated key sum comes from the tensor cores as well: the prologue
// writes phi(k) back into the K tile in place and an all-ones A operand sums
// it over the tile's tokens.  Every tile's result is read back and added into
// fp32 registers (no long accumulation chain inside the tensor core).
//
// Pass C.  The block's prefix state P of both heads is split once per unit
// into bf16 hi + lo and staged as the B operand (K-major rows (head, c) =
// [P hi | P lo]); per tile the rotated queries of both heads, split into
// hi + lo, are the 128 rows (head, token) of the A operand (K-major) and
//   D[(h,tok)][(h',c)] = q~hi.Phi + q~lo.Phi + q~hi.Plo   (6 MMAs of K = 16)
// (blocks h = h' used) is scaled by 1 / (z . phi(q) + eps); each epilogue
// warp stores its 32 x 32 output block through TMA.
//
// Every mbarrier wait is bounded (LCLA_TC_WAIT_NS of globaltimer) and also
// gives up when another role has set the CTA's abort flag; the multi-warp
// roles vote after each wait (named-barrier OR), so an abort is uniform within
// a role and no barrier can deadlock.  An aborting CTA waits (bounded) for
// its own copies and MMAs in flight, frees its tensor memory, writes NaN
// partial states (pass A), sets the caller-visible status word and returns.
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
// One try-wait on the phase with the given parity; the thread may sleep in
// the barrier for up to ~20 us before the attempt reports failure.
__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase with the given parity to complete; gives up when
// the CTA's abort flag is set.  Sets the flag itself on timeout.
__device__ __noinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
    if (bar_try(bar, parity)) return true;
    const uint64_t t0 = gtimer();
    for (;;) {
        if (bar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (gtimer() - t0 > LCLA_TC_WAIT_NS) {
            *abort_flag = 1;
            return false;
        }
    }
}
// Position in a ring of N barrier-guarded slots: index and the parity of the
// phase to wait for.  Consumers of "filled" slots start at phase 0; producers
// waiting for "freed" slots start at phase 1 (the first round is free).
struct Ring {
    int idx;
    uint32_t phase;
};
template <int N>
__device__ __forceinline__ void ring_next(Ring &r)
{
    if (++r.idx == N) {
        r.idx = 0;
        r.phase ^= 1u;
    }
}
__device__ __forceinline__ void bar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// OR of x over the `nthreads` threads that use named barrier `id` (also a barrier).
__device__ __forceinline__ bool vote_any(int id, int nthreads, bool x)
{
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.cta.red.or.pred q, %2, %3, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)x), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
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
__device__ __forceinline__ void tmem_ld8(uint32_t ta, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
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

// ReLU on two packed bf16 (NaN passes through).
__device__ __forceinline__ uint32_t relu2(uint32_t w)
{
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&w);
    x = __hmax2_nan(x, __floats2bfloat162_rn(0.f, 0.f));
    return bf2_bits(x);
}

// Elements [8f, 8f+8) of head h in row r of a [64][64] bf16 tile (128-byte
// swizzle), as 4 packed bf16 pairs.
__device__ __forceinline__ uint4 load_quarter_row(const unsigned char *tile, int r, int h, int f)
{
    return *reinterpret_cast<const uint4 *>(tile + r * 128 + (((4 * h + f) ^ (r & 7)) << 4));
}
// Pairs [4f, 4f+4) of row r of a [64][16] fp32 table tile (64-byte swizzle).
__device__ __forceinline__ float4 load_quarter_table(const unsigned char *tile, int r, int f)
{
    return *reinterpret_cast<const float4 *>(tile + r * 64 + ((f ^ ((r >> 1) & 3)) << 4));
}
// Rotate 4 pairs of (packed bf16) ReLU features, split into bf16 hi + lo.
__device__ __forceinline__ void rope_split4(const uint32_t *fw, const float4 &c4, const float4 &s4, uint32_t *hi,
                                            uint32_t *lo)
{
    const float cv[4] = {c4.x, c4.y, c4.z, c4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float a = bf_lo(fw[p]), b = bf_hi(fw[p]);
        const float y0 = a * cv[p] - b * sv[p];
        const float y1 = a * sv[p] + b * cv[p];
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
        const float2 hf = __bfloat1622float2(h2);
        hi[p] = bf2_bits(h2);
        lo[p] = bf2_bits(__floats2bfloat162_rn(y0 - hf.x, y1 - hf.y));
    }
}
// Quarter f of operand row r (128 B, 128-byte swizzle): hi -> chunk f, lo -> chunk 4+f.
__device__ __forceinline__ void store_quarter_hi_lo(unsigned char *tile, int r, int f, const uint32_t *hi,
                                                    const uint32_t *lo)
{
    unsigned char *row = tile + r * 128;
    *reinterpret_cast<uint4 *>(row + ((f ^ (r & 7)) << 4)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4 *>(row + (((4 + f) ^ (r & 7)) << 4)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}

// ---------------------------------------------------------------------------
// Work units of a persistent CTA: unit u = (segment, head pair, batch entry),
// head pair fastest; CTA c takes units c, c + gridDim.x, ...
// ---------------------------------------------------------------------------
struct Unit {
    int s, hp, b;       // segment, head pair, batch entry
    int t0, t1, blk;    // token range [t0, t1) and its block
    int ntile;          // 64-token tiles
};

__device__ __forceinline__ Unit unit_at(const LclaPlan &p, long long u)
{
    Unit x;
    x.hp = (int)(u % p.ngroups);
    const long long rest = u / p.ngroups;
    x.s = (int)(rest % p.nseg);
    x.b = (int)(rest / p.nseg);
    const LclaSeg g = lcla_segment(p, x.s);
    x.t0 = g.t0;
    x.t1 = g.t1;
    x.blk = g.blk;
    x.ntile = g.t1 > g.t0 ? (g.t1 - g.t0 + T - 1) / T : 0;
    return x;
}

// Bounded wait that ignores the abort flag (used to let in-flight work land).
__device__ __forceinline__ void bar_wait_quiet(uint32_t bar, uint32_t parity)
{
    volatile int never = 0;
    bar_wait(bar, parity, &never);
}

// ---------------------------------------------------------------------------
// Pass A
// ---------------------------------------------------------------------------
struct LayA {
    static constexpr int STAGES = 6;                                // TMA ring
    static constexpr int NA = 3;                                    // A-operand ring
    static constexpr int NTM = 4;                                   // tensor-memory ring
    static constexpr int K_OFF = 0, V_OFF = 8192, C_OFF = 16384, S_OFF = 20480, STAGE = 24576;
    static constexpr int A_OFF = STAGES * STAGE, A_BYTES = 16384;   // [64 tok][128 B] head 0 | head 1
    static constexpr int RED_OFF = A_OFF + NA * A_BYTES;            // [4 quarters][32 e][33] fp32
    static constexpr int Z_OFF = RED_OFF + 4 * 32 * 33 * 4;         // key-sum parts [2 unit parity][16 warps][8]
    static constexpr int CTRL = Z_OFF + 2 * 16 * 8 * 4;
    static constexpr int BYTES = CTRL + 512 + 1024;
    static constexpr int NTHREADS = 704;                            // drain 0-3, producer 4, MMA 5, prologue 6-21
    static constexpr int W_PROD = 4, W_MMA = 5, W_PRO0 = 6, NPRO = 512;
    static constexpr uint32_t TX = STAGE;
    static constexpr uint32_t IDESC = idesc_bf16(128, 64, 1, 1);
    static constexpr int TMEM_COLS = NTM * 64;
};

__global__ void __launch_bounds__(LayA::NTHREADS, 1)
pass_a_tc(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
          const __grid_constant__ CUtensorMap mc, const __grid_constant__ CUtensorMap ms,
          const LclaPlan p, float *__restrict__ part, int *__restrict__ status)
{
    using L = LayA;
    constexpr int S = L::STAGES, NA = L::NA, NTM = L::NTM;
    extern __shared__ __align__(1024) unsigned char smraw[];
    const uint32_t raw = s32(smraw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    unsigned char *sm = smraw + pad;
    const uint32_t sb = raw + pad;
    const uint32_t FULL = sb + L::CTRL, EMPTY = FULL + 8 * S, AREADY = EMPTY + 8 * S, AFREE = AREADY + 8 * NA,
                   TFULL = AFREE + 8 * NA, TFREE = TFULL + 8 * NTM, ZREADY = TFREE + 8 * NTM, ZFREE = ZREADY + 16;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::CTRL + 8 * (2 * S + 2 * NA + 2 * NTM + 4));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    float *zbuf = reinterpret_cast<float *>(sm + L::Z_OFF);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const long long nunits = (long long)p.nseg * p.ngroups * p.B;

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            bar_init(FULL + 8 * i, 1);
            bar_init(EMPTY + 8 * i, 1);
        }
        for (int i = 0; i < NA; ++i) {
            bar_init(AREADY + 8 * i, L::NPRO / 32);
            bar_init(AFREE + 8 * i, 1);
        }
        for (int i = 0; i < NTM; ++i) {
            bar_init(TFULL + 8 * i, 1);
            bar_init(TFREE + 8 * i, 4);
        }
        for (int i = 0; i < 2; ++i) {
            bar_init(ZREADY + 8 * i, L::NPRO / 32);
            bar_init(ZFREE + 8 * i, 1);
        }
        *abort_flag = 0;
        bar_fence_init();
    }
    if (w == L::W_MMA) {
        tmem_alloc(s32(tslot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tslot;

    if (w == L::W_PROD) {
        // ---------------- producer: TMA loads into the ring ----------------
        if (lane == 0) {
            Ring er = {0, 1u};
            int issued = 0;
            bool ok = true;
            for (long long u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const Unit x = unit_at(p, u);
                for (int i = 0; i < x.ntile; ++i) {
                    if (!bar_wait(EMPTY + 8 * er.idx, er.phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t base = sb + er.idx * L::STAGE, fb = FULL + 8 * er.idx;
                    const int t = x.t0 + i * T;
                    bar_expect_tx(fb, L::TX);
                    tma_load3(base + L::K_OFF, &mk, fb, 64 * x.hp, t, x.b);
                    tma_load3(base + L::V_OFF, &mv, fb, 64 * x.hp, t, x.b);
                    tma_load2(base + L::C_OFF, &mc, fb, 0, t);
                    tma_load2(base + L::S_OFF, &ms, fb, 0, t);
                    ring_next<S>(er);
                    ++issued;
                }
            }
            if (!ok)   // let the copies already issued land before the CTA releases its memory
                for (int j = issued > S ? issued - S : 0; j < issued; ++j)
                    bar_wait_quiet(FULL + 8 * (j % S), (uint32_t)((j / S) & 1));
        }
    } else if (w == L::W_MMA) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            Ring sr = {0, 0u}, ar = {0, 0u}, tr = {0, 1u};   // stage, A-ready, TMEM-free
            const uint64_t adesc0 = desc_sw128(sb + L::A_OFF, 8192, 1024);
            const uint64_t vdesc0 = desc_sw128(sb + L::V_OFF, 8192, 1024);
            int issued = 0, last_tb = 0;
            uint32_t last_phase = 0;
            bool ok = true;
            for (long long u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const Unit x = unit_at(p, u);
                for (int i = 0; i < x.ntile; ++i) {
                    if (!bar_wait(AREADY + 8 * ar.idx, ar.phase, abort_flag) ||
                        !bar_wait(TFREE + 8 * tr.idx, tr.phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_after();
                    const uint32_t d = tmem + tr.idx * 64;
                    // descriptor start addresses advance in 16-byte units
                    const uint64_t ad = adesc0 + (uint64_t)((ar.idx * L::A_BYTES) >> 4);
                    const uint64_t vd = vdesc0 + (uint64_t)((sr.idx * L::STAGE) >> 4);
#pragma unroll
                    for (int j = 0; j < T / 16; ++j)   // [hi; lo] k~ (x) v
                        mma_bf16(d, ad + (uint64_t)(128 * j), vd + (uint64_t)(128 * j), L::IDESC, j > 0);
                    mma_commit(TFULL + 8 * tr.idx);
                    mma_commit(AFREE + 8 * ar.idx);
                    mma_commit(EMPTY + 8 * sr.idx);
                    last_tb = tr.idx;
                    last_phase = tr.phase ^ 1u;   // TFULL runs one phase behind TFREE's producer-side parity
                    ring_next<S>(sr);
                    ring_next<NA>(ar);
                    ring_next<NTM>(tr);
                    ++issued;
                }
            }
            if (!ok && issued > 0) bar_wait_quiet(TFULL + 8 * last_tb, last_phase);
        }
    } else if (w >= L::W_PRO0) {
        // ---------------- prologue: phi, key sum, rotary, hi/lo split ----------------
        const int pt = tid - 32 * L::W_PRO0, pw = pt >> 5;
        const int r = pt & 63, h = (pt >> 6) & 1, f = pt >> 7;   // token row, head, quarter of the row
        Ring fr = {0, 0u}, ar = {0, 1u}, zr2 = {0, 1u};   // stage-full, A-free, key-sum buffer free
        bool ok = true;
        for (long long u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
            const Unit x = unit_at(p, u);
            float zacc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) zacc[j] = 0.f;
            for (int i = 0; i < x.ntile; ++i) {
                const int st = fr.idx, ab = ar.idx;
                bool fine = bar_wait(FULL + 8 * fr.idx, fr.phase, abort_flag);
                fine = bar_wait(AFREE + 8 * ar.idx, ar.phase, abort_flag) && fine;
                if (vote_any(1, L::NPRO, !fine)) {
                    ok = false;
                    break;
                }
                ring_next<S>(fr);
                ring_next<NA>(ar);
                unsigned char *stg = sm + st * L::STAGE;
                const int t = x.t0 + i * T, nt = min(T, x.t1 - t);
                const bool valid = r < nt;
                const uint4 kq = load_quarter_row(stg + L::K_OFF, r, h, f);
                const float4 c4 = load_quarter_table(stg + L::C_OFF, r, f);
                const float4 s4 = load_quarter_table(stg + L::S_OFF, r, f);
                uint32_t fw[4] = {kq.x, kq.y, kq.z, kq.w}, hi[4], lo[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    fw[j] = valid ? relu2(fw[j]) : 0u;
                    zacc[2 * j] += bf_lo(fw[j]);
                    zacc[2 * j + 1] += bf_hi(fw[j]);
                }
                rope_split4(fw, c4, s4, hi, lo);
                store_quarter_hi_lo(sm + L::A_OFF + ab * L::A_BYTES + h * 8192, r, f, hi, lo);
                if (!valid)   // rows past the segment belong to another unit: zero this quarter of V
                    *reinterpret_cast<uint4 *>(stg + L::V_OFF + r * 128 + (((4 * h + f) ^ (r & 7)) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) bar_arrive(AREADY + 8 * ab);
            }
            if (!ok) break;
            // unit done: key-sum parts of this warp (32 rows of one (head, quarter)) for the drain
#pragma unroll
            for (int j = 0; j < 8; ++j) {
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) zacc[j] += __shfl_xor_sync(0xffffffffu, zacc[j], m);
            }
            const int zb = zr2.idx;
            if (!bar_wait(ZFREE + 8 * zr2.idx, zr2.phase, abort_flag)) {
                ok = false;
                break;
            }
            ring_next<2>(zr2);
            if (lane == 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j) zbuf[(zb * 16 + pw) * 8 + j] = zacc[j];
                bar_arrive(ZREADY + 8 * zb);
            }
        }
    } else {
        // ---------------- drain: tensor memory -> registers -> partial states ----------------
        const int q4 = w;   // lane quarter: hi_h0, lo_h0, hi_h1, lo_h1
        float *red = reinterpret_cast<float *>(sm + L::RED_OFF);
        const float nanv = __int_as_float(0x7fc00000);
        Ring tr = {0, 0u}, zr2 = {0, 0u};   // TMEM-full, key-sum ready
        bool ok = true;
        for (long long u = blockIdx.x; u < nunits; u += gridDim.x) {
            const Unit x = unit_at(p, u);
            float sacc[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) sacc[j] = 0.f;
            for (int i = 0; ok && i < x.ntile; ++i) {
                const int tb = tr.idx;
                const bool fine = bar_wait(TFULL + 8 * tr.idx, tr.phase, abort_flag);
                ring_next<NTM>(tr);
                if (vote_any(2, 128, !fine)) {
                    ok = false;
                    break;
                }
                tc_after();
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + tb * 64 + (q4 >> 1) * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) sacc[j] += __uint_as_float(v[j]);
                tc_before();
                __syncwarp();
                if (lane == 0) bar_arrive(TFREE + 8 * tb);
            }
            // unit done: S = hi quarter + lo quarter (fixed order); z from the prologue's parts
            const size_t pbase = ((size_t)x.s * p.B + x.b) * p.H;
            const int zb = zr2.idx;
            bool zok = ok && bar_wait(ZREADY + 8 * zr2.idx, zr2.phase, abort_flag);
            ring_next<2>(zr2);
            if (ok) {
#pragma unroll
                for (int j = 0; j < 32; ++j) red[(q4 * 32 + lane) * 33 + j] = sacc[j];
            }
            if (vote_any(2, 128, !zok)) ok = false;
            for (int xx = tid; xx < LCLA_HG * LCLA_SZ; xx += 128) {
                const int hh = xx / LCLA_SZ, e = xx - hh * LCLA_SZ;
                const int head = LCLA_HG * x.hp + hh;
                float val = nanv;
                if (ok) {
                    if (e < LCLA_D * LCLA_D) {
                        const int c = e >> 5, ee = e & 31;
                        val = red[((2 * hh) * 32 + ee) * 33 + c] + red[((2 * hh + 1) * 32 + ee) * 33 + c];
                    } else {   // z[hh][8f + j]: warps 2*(2f + hh) and +1 of the prologue
                        const int ez = e - LCLA_D * LCLA_D, ff = ez >> 3, j = ez & 7;
                        const int w0 = 2 * (2 * ff + hh);
                        val = zbuf[(zb * 16 + w0) * 8 + j] + zbuf[(zb * 16 + w0 + 1) * 8 + j];
                    }
                }
                if (head < p.H) part[(pbase + head) * LCLA_SZ + e] = val;
            }
            vote_any(2, 128, false);
            if (tid == 0 && zok) bar_arrive(ZFREE + 8 * zb);
        }
    }

    pdl_trigger();
    tc_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicOr(status, 1);
    if (w == L::W_MMA) {
        tc_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Pass C
// ---------------------------------------------------------------------------
struct LayC {
    static constexpr int STAGES = 6;                                // TMA ring
    static constexpr int NA = 3;                                    // A-operand ring
    static constexpr int NTM = 4;                                   // tensor-memory / denominator ring
    static constexpr int Q_OFF = 0, C_OFF = 8192, S_OFF = 12288, STAGE = 16384;
    static constexpr int A_OFF = STAGES * STAGE, A_BYTES = 16384;   // [128 rows (head, token)][q~hi | q~lo]
    static constexpr int B_OFF = A_OFF + NA * A_BYTES;              // 2 (unit parity) x [64 rows (head, c)][P hi | P lo]
    static constexpr int O_OFF = B_OFF + 2 * 8192;                  // 4 warps x 2 x [32 tok][64 B] output blocks
    static constexpr int D_OFF = O_OFF + 4 * 2 * 2048;              // denominator parts [NTM][2 h][4 f][64 r]
    static constexpr int CTRL = D_OFF + NTM * 2048;
    static constexpr int BYTES = CTRL + 512 + 1024;
    static constexpr int NTHREADS = 704;                            // epilogue 0-3, producer 4, MMA 5, prologue 6-21
    static constexpr int W_PROD = 4, W_MMA = 5, W_PRO0 = 6, NPRO = 512;
    static constexpr uint32_t TX = STAGE;
    static constexpr uint32_t IDESC = idesc_bf16(128, 64, 0, 0);
    static constexpr int TMEM_COLS = NTM * 64;
};

__global__ void __launch_bounds__(LayC::NTHREADS, 1)
pass_c_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mc,
          const __grid_constant__ CUtensorMap ms, const __grid_constant__ CUtensorMap mo,
          const LclaPlan p, const float *__restrict__ pref, const float eps,
          __nv_bfloat16 *__restrict__ out, int *__restrict__ status)
{
    using L = LayC;
    constexpr int S = L::STAGES, NA = L::NA, NTM = L::NTM;
    extern __shared__ __align__(1024) unsigned char smraw[];
    const uint32_t raw = s32(smraw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    unsigned char *sm = smraw + pad;
    const uint32_t sb = raw + pad;
    const uint32_t FULL = sb + L::CTRL, EMPTY = FULL + 8 * S, AREADY = EMPTY + 8 * S, AFREE = AREADY + 8 * NA,
                   TFULL = AFREE + 8 * NA, TFREE = TFULL + 8 * NTM, DREADY = TFREE + 8 * NTM,
                   BFREE = DREADY + 8 * NTM;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::CTRL + 8 * (2 * S + 2 * NA + 3 * NTM + 2));
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    float *dens = reinterpret_cast<float *>(sm + L::D_OFF);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const long long nunits = (long long)p.nseg * p.ngroups * p.B;

    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            bar_init(FULL + 8 * i, 1);
            bar_init(EMPTY + 8 * i, L::NPRO / 32);
        }
        for (int i = 0; i < NA; ++i) {
            bar_init(AREADY + 8 * i, L::NPRO / 32);
            bar_init(AFREE + 8 * i, 1);
        }
        for (int i = 0; i < NTM; ++i) {
            bar_init(TFULL + 8 * i, 1);
            bar_init(TFREE + 8 * i, 4);
            bar_init(DREADY + 8 * i, L::NPRO / 32);
        }
        for (int i = 0; i < 2; ++i) bar_init(BFREE + 8 * i, 1);
        *abort_flag = 0;
        bar_fence_init();
    }
    if (w == L::W_MMA) {
        tmem_alloc(s32(tslot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tslot;

    if (w == L::W_PROD) {
        // ---------------- producer (q and the tables are inputs: no wait on earlier kernels) ----------------
        if (lane == 0) {
            Ring er = {0, 1u};
            int issued = 0;
            bool ok = true;
            for (long long u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const Unit x = unit_at(p, u);
                for (int i = 0; i < x.ntile; ++i) {
                    if (!bar_wait(EMPTY + 8 * er.idx, er.phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t base = sb + er.idx * L::STAGE, fb = FULL + 8 * er.idx;
                    const int t = x.t0 + i * T;
                    bar_expect_tx(fb, L::TX);
                    tma_load3(base + L::Q_OFF, &mq, fb, 64 * x.hp, t, x.b);
                    tma_load2(base + L::C_OFF, &mc, fb, 0, t);
                    tma_load2(base + L::S_OFF, &ms, fb, 0, t);
                    ring_next<S>(er);
                    ++issued;
                }
            }
            if (!ok)
                for (int j = issued > S ? issued - S : 0; j < issued; ++j)
                    bar_wait_quiet(FULL + 8 * (j % S), (uint32_t)((j / S) & 1));
        }
    } else if (w == L::W_MMA) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            Ring ar = {0, 0u}, tr = {0, 0u};   // A-ready; TMEM slot (freed through the prologue's wait)
            const uint64_t adesc0 = desc_sw128(sb + L::A_OFF, 16, 1024);
            const uint64_t bdesc0 = desc_sw128(sb + L::B_OFF, 16, 1024);
            int ub = 0, issued = 0, last_tb = 0;
            uint32_t last_phase = 0;
            bool ok = true;
            for (long long u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const Unit x = unit_at(p, u);
                if (x.ntile == 0) continue;
                const uint64_t bd = bdesc0 + (uint64_t)((ub * 8192) >> 4);
                for (int i = 0; i < x.ntile; ++i) {
                    if (!bar_wait(AREADY + 8 * ar.idx, ar.phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_after();
                    const uint32_t d = tmem + tr.idx * 64;
                    const uint64_t ad = adesc0 + (uint64_t)((ar.idx * L::A_BYTES) >> 4);
#pragma unroll
                    for (int j = 0; j < 4; ++j)   // q~hi.P hi + q~lo.P hi  (32 B = 2 descriptor units per K step)
                        mma_bf16(d, ad + (uint64_t)(2 * j), bd + (uint64_t)(2 * (j & 1)), L::IDESC, j > 0);
#pragma unroll
                    for (int j = 0; j < 2; ++j)   // + q~hi.P lo
                        mma_bf16(d, ad + (uint64_t)(2 * j), bd + (uint64_t)(4 + 2 * j), L::IDESC, 1);
                    mma_commit(TFULL + 8 * tr.idx);
                    mma_commit(AFREE + 8 * ar.idx);
                    if (i == x.ntile - 1) mma_commit(BFREE + 8 * ub);
                    last_tb = tr.idx;
                    last_phase = tr.phase;
                    ring_next<NA>(ar);
                    ring_next<NTM>(tr);
                    ++issued;
                }
                ub ^= 1;
            }
            if (!ok && issued > 0) bar_wait_quiet(TFULL + 8 * last_tb, last_phase);
        }
    } else if (w >= L::W_PRO0) {
        // ---------------- prologue: prefix state staging, phi, denominator, rotary, hi/lo split ----------------
        const int pt = tid - 32 * L::W_PRO0;
        const int r = pt & 63, h = (pt >> 6) & 1, f = pt >> 7;   // token row, head, quarter of the row
        pdl_wait();   // the prefix states come from the previous kernel
        Ring fr = {0, 0u}, ar = {0, 1u}, tr = {0, 1u}, br = {0, 1u};   // stage-full, A-free, TMEM-free, B-free
        bool ok = true;
        for (long long u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
            const Unit x = unit_at(p, u);
            if (x.ntile == 0) continue;
            const int ub = br.idx;
            unsigned char *bop = sm + L::B_OFF + ub * 8192;
            const size_t pbase = ((size_t)x.blk * p.B + x.b) * p.H;
            // this unit's prefix state -> B operand rows (head, c) = [P hi | P lo], once its buffer is free
            bool fine = bar_wait(BFREE + 8 * br.idx, br.phase, abort_flag);
            ring_next<2>(br);
            if (vote_any(1, L::NPRO, !fine)) {
                ok = false;
                break;
            }
            {
                const int n = pt >> 3, j = pt & 7, hh = n >> 5, c = n & 31;   // 512 chunks, one per thread
                const int head = LCLA_HG * x.hp + hh;
                const float *P = pref + (pbase + (head < p.H ? head : 0)) * LCLA_SZ + c * LCLA_D + 8 * (j & 3);
                uint32_t hq[4], lq[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float y0 = head < p.H ? P[2 * m] : 0.f, y1 = head < p.H ? P[2 * m + 1] : 0.f;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
                    const float2 hf = __bfloat1622float2(h2);
                    hq[m] = bf2_bits(h2);
                    lq[m] = bf2_bits(__floats2bfloat162_rn(y0 - hf.x, y1 - hf.y));
                }
                *reinterpret_cast<uint4 *>(bop + n * 128 + ((j ^ (n & 7)) << 4)) =
                    j < 4 ? make_uint4(hq[0], hq[1], hq[2], hq[3]) : make_uint4(lq[0], lq[1], lq[2], lq[3]);
            }
            float zr[8];
            {
                const int head = LCLA_HG * x.hp + h;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    zr[j] = head < p.H ? pref[(pbase + head) * LCLA_SZ + LCLA_D * LCLA_D + 8 * f + j] : 0.f;
            }
            for (int i = 0; i < x.ntile; ++i) {
                const int st = fr.idx, ab = ar.idx, tb = tr.idx;
                fine = bar_wait(FULL + 8 * fr.idx, fr.phase, abort_flag);
                fine = bar_wait(AFREE + 8 * ar.idx, ar.phase, abort_flag) && fine;
                fine = bar_wait(TFREE + 8 * tr.idx, tr.phase, abort_flag) && fine;
                if (vote_any(1, L::NPRO, !fine)) {
                    ok = false;
                    break;
                }
                ring_next<S>(fr);
                ring_next<NA>(ar);
                ring_next<NTM>(tr);
                unsigned char *stg = sm + st * L::STAGE;
                const uint4 qq = load_quarter_row(stg + L::Q_OFF, r, h, f);
                const float4 c4 = load_quarter_table(stg + L::C_OFF, r, f);
                const float4 s4 = load_quarter_table(stg + L::S_OFF, r, f);
                uint32_t fw[4] = {qq.x, qq.y, qq.z, qq.w}, hi[4], lo[4];
                float den = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    fw[j] = relu2(fw[j]);
                    den = fmaf(bf_lo(fw[j]), zr[2 * j], den);
                    den = fmaf(bf_hi(fw[j]), zr[2 * j + 1], den);
                }
                dens[((tb * 2 + h) * 4 + f) * 64 + r] = den;
                rope_split4(fw, c4, s4, hi, lo);
                store_quarter_hi_lo(sm + L::A_OFF + ab * L::A_BYTES, 64 * h + r, f, hi, lo);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    bar_arrive(AREADY + 8 * ab);
                    bar_arrive(DREADY + 8 * tb);
                    bar_arrive(EMPTY + 8 * st);
                }
            }
        }
    } else {
        // ---------------- epilogue: tensor memory -> scaled bf16 -> TMA store ----------------
        const int q4 = w, er = ((q4 & 1) << 5) | lane, eh = q4 >> 1;
        Ring tr = {0, 0u};   // TMEM-full and denominators-ready share the ring
        int ob = 0;
        bool ok = true;
        for (long long u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
            const Unit x = unit_at(p, u);
            const int ehead = LCLA_HG * x.hp + eh;
            for (int i = 0; i < x.ntile; ++i) {
                const int tb = tr.idx;
                bool fine = bar_wait(TFULL + 8 * tr.idx, tr.phase, abort_flag);
                fine = bar_wait(DREADY + 8 * tr.idx, tr.phase, abort_flag) && fine;
                if (vote_any(2, 128, !fine)) {
                    ok = false;
                    break;
                }
                ring_next<NTM>(tr);
                tc_after();
                const int t = x.t0 + i * T, nt = min(T, x.t1 - t);
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + tb * 64 + eh * 32, v);
                const float *dp = dens + (tb * 2 + eh) * 4 * 64 + er;
                const float inv = 1.0f / (((dp[0] + dp[64]) + dp[128]) + dp[192] + eps);
                tmem_wait_ld();
                uint32_t o[16];
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    o[m] = bf2_bits(__floats2bfloat162_rn(__uint_as_float(v[2 * m]) * inv,
                                                          __uint_as_float(v[2 * m + 1]) * inv));
                tc_before();
                __syncwarp();
                if (lane == 0) bar_arrive(TFREE + 8 * tb);
                if (nt == T) {
                    unsigned char *obuf = sm + L::O_OFF + (q4 * 2 + ob) * 2048;
                    ob ^= 1;
                    if (lane == 0) bulk_wait_read1();   // this buffer's previous store has read it
                    __syncwarp();
                    const int sw = (lane >> 1) & 3;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<uint4 *>(obuf + lane * 64 + ((j ^ sw) << 4)) =
                            make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store3(&mo, s32(obuf), 64 * x.hp + 32 * eh, t + 32 * (q4 & 1), x.b);
                        bulk_commit();
                    }
                } else {
                    if (er < nt && ehead < p.H) {
                        uint4 *dst = reinterpret_cast<uint4 *>(
                            out + (((size_t)x.b * p.N + (size_t)(t + er)) * p.H + ehead) * LCLA_D);
#pragma unroll
                        for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                    }
                    if (lane == 0) bulk_commit();   // empty group: one group per tile keeps the ring accounting exact
                }
            }
        }
        if (lane == 0) bulk_wait_all();
    }

    tc_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicOr(status, 2);
    if (w == L::W_MMA) {
        tc_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace lcla
