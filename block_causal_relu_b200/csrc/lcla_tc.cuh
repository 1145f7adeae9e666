// lcla_tc.cuh -- tensor-core (tcgen05 + TMA) kernels: bf16 inputs, block mode.
//
// Same two passes as the CUDA-core path ("Implementing Block Causal Linear
// Attention for Long Video Generation with Sana", section "The Linear
// Attention Kernel": vk = v k_rotated^T, out = vk q_rotated, normaliser from
// the unrotated key sum; section "Rotary Position Embeddings": rotary on the
// ReLU features), with the d x d contractions on the 5th-generation tensor
// cores.
//
// A tcgen05.mma of M = 128, K = 16 takes the same time for any N up to 256,
// so both passes are built around N = 256 products: a work unit is
// (segment, head quad, batch entry) -- four heads of 32 -- and a tile is 64
// tokens of those four heads.  Both kernels are persistent (one CTA per SM,
// units c, c + gridDim.x, ..., quad fastest) and warp-specialised:
//   box producer    TMA loads of each tile's q, or k and v, boxes into a ring;
//   table producer  the tile's rotary rows into their own ring (pass C at
//                   d = 32: also each unit's prefix states, a unit ahead);
//   MMA warp        one thread issues tcgen05.mma and tcgen05.commit;
//   prologue warps  ReLU and rotary of k or q into the MMA operand (pass A:
//                   16 warps on each tile, bf16 hi + lo written in place over
//                   the stage's raw k; pass C: groups of 4 warps taking turns
//                   on the tiles -- three groups at d = 32, whose registers
//                   come from a setmaxnreg split -- one fp16 term into the
//                   group's own operand slot, and the normaliser);
//   drain/epilogue  tensor memory -> registers: warp w reads tensor memory
//                   lanes 32(w & 3)..+31, which belong to head w & 3 of the
//                   quad (pass A: 4 drain warps; pass C: 8 epilogue warps,
//                   two per head, one per half of the tile's tokens).
// Roles talk only through mbarriers.
//
// Pass A.  A = V^T of the quad exactly as TMA lands it (MN-major, rows
// (head, c)), B = the rotated keys split into bf16 hi + lo (k~ = hi + lo to
// 2^-16 relative), MN-major, one 64-column atom [hi 32 | lo 32] per head:
//     D[(h', c)][(h, part, e)] = sum_tok v[tok][h', c] part(k~)[tok][h, e].
// Warp q adds the diagonal block h = h' of every tile (hi + lo) into fp32
// registers; the unrotated key sum z comes from the prologue's registers.
// A stage holds one tile from its TMA load until the tile's MMAs complete.
//
// Pass C.  A = the block's prefix state of the quad, each row c scaled by a
// power of two (P~), K-major: fp16 [P~hi | P~lo] at d = 32, one fp16 term per
// key half at d = 64; B = the rotated ReLU queries q~ as one fp16 term, rows
// (head, token), K-major:
//     D[(h', c)][(h, tok)] = P~ . q~   (4 MMAs of K = 16 per tile),
// so the diagonal block h = h' is the output times the row's scale and the
// token's normaliser z . phi(q) + eps.  The raw q slot is freed once its
// prologue group has read it, the operand slot when the tile's MMAs complete.
// Epilogue warp q reads the accumulator in the 16x256b fragment (two c rows x
// two tokens per thread), multiplies by the inverse row scale and 1 / (z .
// phi(q) + eps), packs token pairs to bf16 and writes the [32 tok][32 c] box
// transposed with stmatrix into a 64-byte-swizzled buffer, stored by one TMA
// store (ragged tiles: the valid rows are copied out of the same buffer with
// plain stores).
//
// Every mbarrier wait is bounded (LCLA_TC_WAIT_NS of globaltimer) and gives
// up when another role has set the CTA's abort flag; each warp makes the
// outcome of a wait uniform across its lanes before acting on it, and no two
// warps share any other barrier, so an abort cannot deadlock.  An aborting
// CTA waits (bounded) for its own copies and MMAs in flight, frees its tensor
// memory, writes NaN partial states (pass A), sets the caller-visible status
// word and returns.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "lcla_common.cuh"
#include "lcla_plan.h"

#define LCLA_TC_WAIT_NS 1000000000ull   // 1 s: far above any legitimate wait

namespace lcla {
namespace tc {

constexpr int T = LCLA_TC_T;     // tokens per tile
constexpr int HQ = LCLA_TC_HQ;   // heads per unit
constexpr unsigned ALL = 0xffffffffu;

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
// Slow path of bar_wait: keep trying until the phase completes, the CTA's
// abort flag is set, or LCLA_TC_WAIT_NS pass (then set the flag).
__device__ __forceinline__ bool bar_wait_slow_body(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
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
// Out of line, so that the rare slow path does not grow every wait site.
__device__ __noinline__ bool bar_wait_slow(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
    return bar_wait_slow_body(bar, parity, abort_flag);
}
// Bounded wait for the phase with the given parity to complete; gives up when
// the CTA's abort flag is set.  Sets the flag itself on timeout.  INL: the slow
// path inline, for code that runs under a setmaxnreg limit (no calls there).
template <bool INL = false>
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
    if (INL) return bar_try(bar, parity) || bar_wait_slow_body(bar, parity, abort_flag);
    return bar_try(bar, parity) || bar_wait_slow(bar, parity, abort_flag);
}
// Bounded wait that ignores the abort flag (used to let in-flight work land).
template <bool INL = false>
__device__ __forceinline__ void bar_wait_quiet(uint32_t bar, uint32_t parity)
{
    volatile int never = 0;
    bar_wait<INL>(bar, parity, &never);
}
__device__ __forceinline__ void bar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// release_after_use: a warp releases a shared buffer that a TMA load will
// refill only after instructions have consumed every value it loaded from it.
// An arrive issued right after the loads themselves was observed to let the
// refill overtake them (pass A read the next tile's rotary rows, intermittently).

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

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Per-thread register limit of the executing warpgroup (every warp of it executes the same one): dec returns
// registers to the CTA's pool, inc takes them from it (and waits until they are there).
template <int N> __device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N> __device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

// Plain bulk copy of `bytes` contiguous bytes (addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"((uint64_t)src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tma_load2(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
// L2 eviction policies: streamed tensors (read or written once) go first, the
// small partial and prefix states that the next kernel reads back stay.
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void tma_load3_hint(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y, int z,
                                               uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%3, %4, %5}], [%2], %6;"
        ::"r"(dst), "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y), "r"(z), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void tma_store3_hint(const CUtensorMap *map, uint32_t src, int x, int y, int z, uint64_t pol)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group.L2::cache_hint [%0, {%2, %3, %4}], [%1], %5;"
                 ::"l"((uint64_t)map), "r"(src), "r"(x), "r"(y), "r"(z), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_v4_hint(float4 *p, float4 v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;"
                 ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_f32_hint(float *p, float v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void tma_store3(const CUtensorMap *map, uint32_t src, int x, int y, int z)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
                 ::"l"((uint64_t)map), "r"(src), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
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

// 32 lanes x 32 columns of 32 bits: thread t of the warp gets lane (quarter*32 + t).
// tcgen05.ld fills its destination registers asynchronously; only
// tcgen05.wait::ld makes them valid.  Both sit in one asm statement, so that
// the compiler cannot schedule any use of the outputs before the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t ta, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(ta)
        : "memory");
}

// 32 lanes x 16 columns, as tmem_ld32.
__device__ __forceinline__ void tmem_ld16(uint32_t ta, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(ta)
        : "memory");
}

// Two 16-lane halves of a warp's lane quarter, 32 columns each (shape 16x256b,
// four repeats): thread t gets, for half L (tensor-memory lanes ta + 16L + ...),
// r[16L + 4j + i] = lane t/4 + 8(i >> 1), column 8j + 2(t % 4) + (i & 1) --
// the accumulator fragment that stmatrix takes.  Loads and wait in one asm
// statement, as in tmem_ld32.
__device__ __forceinline__ void tmem_ld16x256_x4x2(uint32_t ta, uint32_t tb, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%32];\n"
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%33];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(ta), "r"(tb)
        : "memory");
}

// Four 8x8 b16 matrices stored transposed: matrix m's fragment (thread t holds
// row t/4, columns 2(t%4), 2(t%4)+1 in w[m]) lands with fragment column k at
// the 16-byte row whose address thread 8m + k passes.
__device__ __forceinline__ void stsm4_trans(uint32_t addr, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3)
{
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1),
                 "r"(w2), "r"(w3)
                 : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout, version 1).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Shared-memory matrix descriptor, 64-byte swizzle (sm_100 layout, version 1).
__device__ __forceinline__ uint64_t desc_sw64(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (4ull << 61);
}
// Instruction descriptor: kind::f16 with fp16 A and B (both K-major), fp32 D.
constexpr uint32_t idesc_f16(int M, int N)
{
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D.
constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }
__device__ __forceinline__ uint32_t pack_bf2(float a, float b) { return bf2_bits(__floats2bfloat162_rn(a, b)); }


// ReLU on two packed bf16 (NaN passes through).
__device__ __forceinline__ uint32_t relu2(uint32_t w)
{
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&w);
    x = __hmax2_nan(x, __floats2bfloat162_rn(0.f, 0.f));
    return bf2_bits(x);
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
        lo[p] = pack_bf2(y0 - hf.x, y1 - hf.y);
    }
}
// Packed bf16 -> fp32: the element in the low half, and the one in the high half.
__device__ __forceinline__ float bf_low(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_high(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }


// 1 / x from the hardware approximation (relative error of a few ulp; the
// products it scales carry bf16 operands, far coarser).
__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// z . phi for one quarter: za = z of the even elements (pairs 0-1, 2-3), zb = of the odd ones.
__device__ __forceinline__ float zdot4_x2(const uint32_t *fw, float2 za01, float2 za23, float2 zb01, float2 zb23)
{
    float2 d = __fmul2_rn(make_float2(bf_low(fw[0]), bf_low(fw[1])), za01);
    d = __ffma2_rn(make_float2(bf_low(fw[2]), bf_low(fw[3])), za23, d);
    d = __ffma2_rn(make_float2(bf_high(fw[0]), bf_high(fw[1])), zb01, d);
    d = __ffma2_rn(make_float2(bf_high(fw[2]), bf_high(fw[3])), zb23, d);
    return d.x + d.y;
}

// Quarter f of operand row r (128 B, 128-byte swizzle): hi -> chunk f, lo -> chunk 4+f.
__device__ __forceinline__ void store_quarter_hi_lo(unsigned char *tile, int r, int f, const uint32_t *hi,
                                                    const uint32_t *lo)
{
    unsigned char *row = tile + r * 128;
    *reinterpret_cast<uint4 *>(row + ((f ^ (r & 7)) << 4)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4 *>(row + (((4 + f) ^ (r & 7)) << 4)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}


// Operand atom a (8 KB: [64 rows][hi 32 | lo 32] of one head) holds head
// 2(a & 1) + (a >> 1): the [64 token][heads 2b, 2b+1] input box b lands where
// atom b lives, and the prologue thread that reads a row's quarter f of heads
// 2b and 2b+1 writes head 2b's hi and lo there -- exactly the two 16-byte
// chunks it has read -- and head 2b+1's into the fresh atom 2+b.
__device__ __forceinline__ int atom_of(int h) { return (h >> 1) + 2 * (h & 1); }

// Both prologues have 16 warps, a thread doing one token quarter of one
// head pair g = (lane >> 3) & 1 (heads 2g, 2g+1), quarter f = lane & 3, on one
// of four rows of the 8-row block k = pw >> 1: {0, 5, 1, 4} for even pw,
// {2, 7, 3, 6} for odd pw, picked by lane bits 2 and 4.  A 128-bit access is
// served eight lanes at a time, and each group of eight lanes here holds two
// rows whose 128-byte swizzles differ in bit 2 and whose parities differ: its
// eight chunks of the stage (128-byte swizzle) and of the rotary rows (64-byte
// swizzle) fall on eight different 16-byte bank groups.  in0 / in1: the raw
// chunks of heads 2g / 2g+1 in box g, which are also atom g's hi / lo chunks;
// out2 / out3: atom 2+g's hi / lo chunks.
struct PairOffs {
    int g, f, r, in0, in1, out2, out3, tab;
};
__device__ __forceinline__ PairOffs pair_offsets(int pw, int lane)
{
    PairOffs o;
    o.f = lane & 3;
    o.g = (lane >> 3) & 1;
    const int pr = ((lane >> 4) << 1) | ((lane >> 2) & 1);   // pair lane >> 4, member (lane >> 2) & 1
    o.r = 8 * (pw >> 1) + 2 * (pw & 1) + (pr >> 1) + (pr & 1) * (5 - 2 * (pr >> 1));
    const int sw = o.r & 7, row = o.r * 128;
    o.in0 = o.g * 8192 + row + ((o.f ^ sw) << 4);
    o.in1 = o.g * 8192 + row + (((4 + o.f) ^ sw) << 4);
    o.out2 = (2 + o.g) * 8192 + row + ((o.f ^ sw) << 4);
    o.out3 = (2 + o.g) * 8192 + row + (((4 + o.f) ^ sw) << 4);
    o.tab = o.r * 64 + ((o.f ^ ((o.r >> 1) & 3)) << 4);
    return o;
}
__device__ __forceinline__ uint4 lds128(const unsigned char *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ float4 ldsf4(const unsigned char *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void sts128(unsigned char *p, const uint32_t *w)
{
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// ---------------------------------------------------------------------------
// Work units of a persistent CTA: unit u = (segment, head quad, batch entry),
// quad fastest; CTA c takes units c, c + gridDim.x, ...  Quad fastest keeps
// the CTAs of a round on the same tokens: together they read and write whole
// token rows of the [B, N, H, d] tensors (measured: segment-fastest order
// made pass C 9 % slower at 480p).
// ---------------------------------------------------------------------------
struct Unit {
    int s, hq, b;       // segment, head quad, batch entry
    int t0, t1, blk;    // token range [t0, t1) and its block
    int ntile;          // 64-token tiles
};

// (The host keeps nseg * nquads * B below 2^31 on this path.)
__device__ __forceinline__ Unit unit_at(const LclaPlan &p, int u)
{
    Unit x;
    x.hq = u % p.nquads;
    const int rest = u / p.nquads;
    x.s = rest % p.nseg;
    x.b = rest / p.nseg;
    const LclaSeg g = lcla_segment(p, x.s);
    x.t0 = g.t0;
    x.t1 = g.t1;
    x.blk = g.blk;
    x.ntile = g.t1 > g.t0 ? (g.t1 - g.t0 + T - 1) / T : 0;
    return x;
}

constexpr int CTRL_BYTES = 512;   // control block: mbarriers (8 B each), tensor-memory slot, abort flag
constexpr int SMEM_MAX = 232448;  // dynamic shared memory a CTA may opt in to
constexpr int NPRO = 16;          // prologue warps (both passes)

// Head width DW: 32, or 64 seen as two 32-dim "virtual" heads (dims 0-31 and
// 32-63 of a head are virtual heads 2h and 2h+1 of the same [B, N, H * 64]
// row).  A table slot holds one tile's rotary rows: [cos | sin] of 4 KB each
// at DW = 32, [cos 0-15 | cos 16-31 | sin 0-15 | sin 16-31] at DW = 64, the
// second half rotating the second virtual head.
template <int DW>
struct Width {
    static_assert(DW == 32 || DW == 64, "head widths 32 and 64");
    static constexpr int VPH = DW / 32;               // virtual heads per head
    static constexpr int TAB_BYTES = 8192 * VPH;      // one table slot
    static constexpr int SZ = (DW + 1) * DW;          // floats per (S, z) state
};

// Producers.  The tile's input boxes and its rotary rows come from two
// threads of two different warps, each running ahead through its own ring:
// a producer that waited for a slot of one ring before filling the other
// would hold the deeper ring to the depth of the shallower one.
//
// Input boxes: per tile, TMA loads of the quad's boxes into the stage ring
// (NBOX boxes of [64 token][4 / NBOX heads] per tensor map, heads past H read
// as zeros).  On abort, waits (bounded) for the loads already issued.
template <int S, int STAGE, int NMAP, int NBOX, bool INL = false>
__device__ __forceinline__ void produce_boxes(const LclaPlan &p, int nunits, uint32_t sb, uint32_t FULL, uint32_t EMPTY,
                                              const CUtensorMap *const (&maps)[NMAP], const int (&offs)[NMAP],
                                              volatile int *abort_flag)
{
    Ring er = {0, 1u};
    int issued = 0;
    bool ok = true;
    const uint64_t stream_pol = policy_evict_first();
    for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        const Unit x = unit_at(p, u);
        const int x0 = HQ * LCLA_D * x.hq;
        for (int i = 0; i < x.ntile; ++i) {
            const int t = x.t0 + i * T;
            if (!bar_wait<INL>(EMPTY + 8 * er.idx, er.phase, abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t base = sb + er.idx * STAGE, fb = FULL + 8 * er.idx;
            bar_expect_tx(fb, (uint32_t)(NMAP * HQ * LCLA_D * T * 2));
#pragma unroll
            for (int m = 0; m < NMAP; ++m)
#pragma unroll
                for (int j = 0; j < NBOX; ++j)   // box j: heads [j HQ / NBOX, (j + 1) HQ / NBOX) of the quad
                    tma_load3_hint(base + offs[m] + j * (HQ * LCLA_D * T * 2 / NBOX), maps[m], fb,
                                   x0 + j * (HQ * LCLA_D / NBOX), t, x.b, stream_pol);
            ring_next<S>(er);
            ++issued;
        }
    }
    if (!ok)   // let the copies already issued land before the CTA releases its memory
        for (int j = issued > S ? issued - S : 0; j < issued; ++j)
            bar_wait_quiet<INL>(FULL + 8 * (j % S), (uint32_t)((j / S) & 1));
}

// Rotary rows: per tile, the tile's rows of the cos and sin tables into the
// table ring (DW = 64: columns 0-15 and 16-31 of each, one box per half).
// after(x, i) runs once each tile's rows are issued; false gives up.
template <int DW, int NTS, bool INL, typename After>
__device__ __forceinline__ void produce_tables(const LclaPlan &p, int nunits, uint32_t tab0, uint32_t CFULL,
                                               uint32_t CEMPTY, const CUtensorMap *mc, const CUtensorMap *ms,
                                               volatile int *abort_flag, After &&after)
{
    constexpr int TB = Width<DW>::TAB_BYTES, VPH = Width<DW>::VPH;
    Ring cr = {0, 1u};
    int issued = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        const Unit x = unit_at(p, u);
        for (int i = 0; i < x.ntile; ++i) {
            const int t = x.t0 + i * T;
            if (!bar_wait<INL>(CEMPTY + 8 * cr.idx, cr.phase, abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t tb = tab0 + cr.idx * TB, cb = CFULL + 8 * cr.idx;
            bar_expect_tx(cb, (uint32_t)TB);
#pragma unroll
            for (int hh = 0; hh < VPH; ++hh) {   // columns [16 hh, 16 hh + 16) of the [N, DW / 2] tables
                tma_load2(tb + hh * 4096, mc, cb, 16 * hh, t);
                tma_load2(tb + TB / 2 + hh * 4096, ms, cb, 16 * hh, t);
            }
            ring_next<NTS>(cr);
            ++issued;
            if (!after(x, i)) {
                ok = false;
                break;
            }
        }
    }
    if (!ok)
        for (int j = issued > NTS ? issued - NTS : 0; j < issued; ++j)
            bar_wait_quiet<INL>(CFULL + 8 * (j % NTS), (uint32_t)((j / NTS) & 1));
}

// ---------------------------------------------------------------------------
// Pass A
// ---------------------------------------------------------------------------
template <int DW>
struct LayA {
    // four stages at DW = 32; three at DW = 64, whose table slots are twice as large
    static constexpr int STAGES = DW == 32 ? 4 : 3;
    // stage: [k~ operand, 4 atoms of [64 tok][hi 32 | lo 32] (raw k lands in atoms 0-1) | v, 2 boxes]
    static constexpr int K_OFF = 0, V_OFF = 32768, STAGE = 49152;
    static constexpr int TAB_BYTES = Width<DW>::TAB_BYTES;
    static constexpr int NT = 3;                                    // rotary-table ring slots
    static constexpr int C_OFF = STAGES * STAGE;                    // rotary-table ring
    static constexpr int Z_OFF = C_OFF + NT * TAB_BYTES;            // key-sum parts [16 warps][2 g][4 f][2 heads][8]
    static constexpr int Z_BYTES = NPRO * 2 * 4 * 2 * 8 * 4;
    static constexpr int CTRL = Z_OFF + Z_BYTES;                    // mbarriers, tensor-memory slot, abort flag
    static constexpr int BYTES = CTRL + CTRL_BYTES + 1024;          // + worst-case 1024-byte alignment pad
    static constexpr int NTM = 2;                                   // tensor-memory accumulators (256 columns each)
    // tiles summed in one accumulator before the drain takes it: tensor-core
    // accumulation over whole segments (~100 K-steps) was measured to lose
    // about 1.6e-5 of max |S| against fp32 sums; 4 tiles (16 K-steps) keep the
    // state well inside 1e-5, the rest is summed in registers
    static constexpr int CHUNK = 4;
    static constexpr int NTHREADS = 736;                            // drain 0-3, producer 4, MMA 5, prologue 6-21, tables 22
    static constexpr int W_PROD = 4, W_MMA = 5, W_PRO0 = 6, W_TAB = 22;
    static constexpr uint32_t IDESC = idesc_bf16(128, 256, 1, 1);
    static constexpr int TMEM_COLS = NTM * 256;
    static constexpr int NBARS = 3 * STAGES + 2 * NT + 2 * NTM + 3;
    static_assert(BYTES <= SMEM_MAX, "pass A shared memory");
    static_assert(8 * NBARS + 8 <= CTRL_BYTES, "pass A control block");
    static_assert(W_TAB - W_PRO0 == NPRO && NTHREADS / 32 == W_TAB + 1, "pass A prologue warps: barrier counts use NPRO");
};

// Pass A over head width DW.  At DW = 64 each quad holds two heads as four
// virtual heads; the products of the quad already hold the cross blocks
// (virtual heads 2h', 2h'+1 against 2h, 2h+1) that a 64-dim head's state needs.
template <int DW>
__global__ void __launch_bounds__(LayA<DW>::NTHREADS, 1)
pass_a_tc(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
          const __grid_constant__ CUtensorMap mc, const __grid_constant__ CUtensorMap ms, const LclaPlan p,
          float *__restrict__ part, int *__restrict__ status)
{
    using L = LayA<DW>;
    constexpr int S = L::STAGES, NTM = L::NTM, VPH = Width<DW>::VPH, TB = L::TAB_BYTES, NT = L::NT;
    const int HV = p.H * VPH;   // virtual heads
    extern __shared__ __align__(1024) unsigned char smraw[];
    const uint32_t raw = s32(smraw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    unsigned char *sm = smraw + pad;
    const uint32_t sb = raw + pad;
    const uint32_t FULL = sb + L::CTRL, EMPTY = FULL + 8 * S, KREADY = EMPTY + 8 * S, CFULL = KREADY + 8 * S,
                   CEMPTY = CFULL + 8 * NT, TFULL = CEMPTY + 8 * NT, TFREE = TFULL + 8 * NTM,
                   ZREADY = TFREE + 8 * NTM, ZFREE = ZREADY + 8, MDONE = ZFREE + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::CTRL + 8 * L::NBARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    float *zbuf = reinterpret_cast<float *>(sm + L::Z_OFF);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int nunits = p.nseg * p.nquads * p.B;

    // the call's status word starts at 0: pass A is the call's first kernel (launched after everything before it
    // in the stream), and a bounded wait of this call can only give up a second after this store
    if (blockIdx.x == 0 && tid == 0) *status = 0;
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            bar_init(FULL + 8 * i, 1);
            bar_init(EMPTY + 8 * i, 1);
            bar_init(KREADY + 8 * i, NPRO);
        }
        for (int i = 0; i < NT; ++i) {
            bar_init(CFULL + 8 * i, 1);
            bar_init(CEMPTY + 8 * i, NPRO);
        }
        for (int i = 0; i < NTM; ++i) {
            bar_init(TFULL + 8 * i, 1);
            bar_init(TFREE + 8 * i, 4);
        }
        bar_init(ZREADY, NPRO);
        bar_init(ZFREE, 4);
        bar_init(MDONE, 1);
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
        // ---------------- producer: k and v boxes of each tile ----------------
        if (lane == 0) {
            const CUtensorMap *const maps[2] = {&mk, &mv};
            const int offs[2] = {L::K_OFF, L::V_OFF};
            produce_boxes<S, L::STAGE, 2, 2>(p, nunits, sb, FULL, EMPTY, maps, offs, abort_flag);
        }
    } else if (w == L::W_TAB) {
        // ---------------- producer: rotary rows of each tile ----------------
        if (lane == 0)
            produce_tables<DW, NT, false>(p, nunits, sb + L::C_OFF, CFULL, CEMPTY, &mc, &ms, abort_flag,
                                          [](const Unit &, int) { return true; });
    } else if (w == L::W_MMA) {
        // ---------------- MMA issuer: one accumulator per chunk of CHUNK tiles ----------------
        if (lane == 0) {
            Ring sr = {0, 0u}, tr = {0, 1u};   // stage (k~ ready), accumulator free
            const uint64_t vdesc0 = desc_sw128(sb + L::V_OFF, 8192, 1024);
            const uint64_t kdesc0 = desc_sw128(sb + L::K_OFF, 8192, 1024);
            int issued = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const Unit x = unit_at(p, u);
                for (int i = 0; i < x.ntile; ++i) {
                    const int ic = i % L::CHUNK;
                    if ((ic == 0 && !bar_wait(TFREE + 8 * tr.idx, tr.phase, abort_flag)) ||
                        !bar_wait(KREADY + 8 * sr.idx, sr.phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_after();
                    const uint32_t d = tmem + tr.idx * 256;
                    // descriptor start addresses advance in 16-byte units; 16 tokens = 2048 B
                    const uint64_t so = (uint64_t)((sr.idx * L::STAGE) >> 4);
#pragma unroll
                    for (int j = 0; j < T / 16; ++j)   // D (+)= v^T (x) [k~hi | k~lo]
                        mma_bf16(d, vdesc0 + so + 128 * j, kdesc0 + so + 128 * j, L::IDESC, (ic | j) != 0);
                    mma_commit(EMPTY + 8 * sr.idx);
                    ring_next<S>(sr);
                    ++issued;
                    if (ic == L::CHUNK - 1 || i == x.ntile - 1) {   // chunk complete: hand it to the drain
                        mma_commit(TFULL + 8 * tr.idx);
                        ring_next<NTM>(tr);
                    }
                }
            }
            if (!ok && issued > 0) {   // let the MMAs in flight finish before the memory is released
                mma_commit(MDONE);
                bar_wait_quiet(MDONE, 0);
            }
        }
    } else if (w >= L::W_PRO0) {
        // ---------------- prologue: phi, key sum, rotary, hi/lo split ----------------
        const int pw = w - L::W_PRO0;
        const PairOffs o = pair_offsets(pw, lane);
        Ring fr = {0, 0u}, cr = {0, 0u}, zr = {0, 1u};   // stage full, table full, key-sum buffer free (1 slot)
        bool ok = true;
        for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
            const Unit x = unit_at(p, u);
            if (x.ntile == 0) continue;
            float zacc[2][8];   // z[8f, 8f+8) of heads 2g, 2g+1 over this thread's rows
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int j = 0; j < 8; ++j) zacc[hh][j] = 0.f;
            for (int i = 0; i < x.ntile; ++i) {
                const int st = fr.idx, ct = cr.idx;
                bool fine = bar_wait(FULL + 8 * fr.idx, fr.phase, abort_flag);
                fine = bar_wait(CFULL + 8 * cr.idx, cr.phase, abort_flag) && fine;
                if (!__all_sync(ALL, fine)) {
                    ok = false;
                    break;
                }
                ring_next<S>(fr);
                ring_next<NT>(cr);
                unsigned char *stg = sm + st * L::STAGE;
                const unsigned char *tab = sm + L::C_OFF + ct * TB;
                // DW = 64: heads 2g, 2g+1 are the halves of one head and rotate with table halves 0, 1
                float4 c4[2], s4[2];
                c4[0] = ldsf4(tab + o.tab);
                s4[0] = ldsf4(tab + TB / 2 + o.tab);
                c4[1] = VPH == 2 ? ldsf4(tab + 4096 + o.tab) : c4[0];
                s4[1] = VPH == 2 ? ldsf4(tab + TB / 2 + 4096 + o.tab) : s4[0];
                const uint4 k0 = lds128(stg + L::K_OFF + o.in0);   // head 2g
                const uint4 k1 = lds128(stg + L::K_OFF + o.in1);   // head 2g+1
                const int t = x.t0 + i * T, nt = min(T, x.t1 - t);
                const bool valid = o.r < nt;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint4 kv = hh ? k1 : k0;
                    uint32_t fw[4] = {kv.x, kv.y, kv.z, kv.w}, hi[4], lo[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        fw[j] = valid ? relu2(fw[j]) : 0u;
                        zacc[hh][2 * j] += bf_lo(fw[j]);
                        zacc[hh][2 * j + 1] += bf_hi(fw[j]);
                    }
                    rope_split4(fw, c4[hh], s4[hh], hi, lo);
                    // head 2g -> atom g (over the raw chunks just read), head 2g+1 -> atom 2+g
                    sts128(stg + L::K_OFF + (hh ? o.out2 : o.in0), hi);
                    sts128(stg + L::K_OFF + (hh ? o.out3 : o.in1), lo);
                }
                if (!valid) {   // rows past the segment belong to another unit: zero this quarter of v
                    *reinterpret_cast<uint4 *>(stg + L::V_OFF + o.in0) = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(stg + L::V_OFF + o.in1) = make_uint4(0u, 0u, 0u, 0u);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    bar_arrive(KREADY + 8 * st);
                    bar_arrive(CEMPTY + 8 * ct);   // after the rows have been used: see release_after_use
                }
            }
            if (!ok) break;
            // unit done: sum this warp's four rows (lane bits 2 and 4) and hand the parts to the drain
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    zacc[hh][j] += __shfl_xor_sync(ALL, zacc[hh][j], 4);
                    zacc[hh][j] += __shfl_xor_sync(ALL, zacc[hh][j], 16);
                }
            if (!__all_sync(ALL, bar_wait(ZFREE, zr.phase, abort_flag))) {
                ok = false;
                break;
            }
            ring_next<1>(zr);
            if ((lane & 0x14) == 0) {   // lanes 0-3 (g = 0) and 8-11 (g = 1), quarter f = lane & 3
                float4 *dst = reinterpret_cast<float4 *>(zbuf + ((pw * 2 + o.g) * 4 + o.f) * 16);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    dst[2 * hh] = make_float4(zacc[hh][0], zacc[hh][1], zacc[hh][2], zacc[hh][3]);
                    dst[2 * hh + 1] = make_float4(zacc[hh][4], zacc[hh][5], zacc[hh][6], zacc[hh][7]);
                }
            }
            __syncwarp();
            if (lane == 0) bar_arrive(ZREADY);
        }
    } else {
        // ---------------- drain: chunk accumulators -> partial state of the unit ----------------
        // warp q: virtual head q of the quad, tensor-memory lanes 32q + c.  DW = 32: row c of its own S (the
        // diagonal block, hi + lo columns).  DW = 64: row 32 a + c of its head's S, a = q & 1, from the blocks
        // against both halves of the head (virtual heads q & ~1 and q | 1: columns e and 32 + e).
        const int q = w;
        const float nanv = __int_as_float(0x7fc00000);
        Ring tr = {0, 0u}, zr = {0, 0u};   // accumulator full, key sum ready (1 slot)
        bool ok = true;
        for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
            const Unit x = unit_at(p, u);
            const int vh = HQ * x.hq + q;
            const bool live = vh < HV;
            float *dst = part + (((size_t)x.s * p.B + x.b) * p.H + (live ? vh / VPH : 0)) * Width<DW>::SZ;
            float *rows = dst + (size_t)(vh % VPH) * 32 * DW;   // this warp's 32 rows of S
            float *zdst = dst + DW * DW + (vh % VPH) * 32;       // and its 32 entries of z
            if (ok && x.ntile == 0) {   // empty segment: nothing was loaded or summed
                if (live) {
                    for (int e = lane; e < 32 * DW; e += 32) rows[e] = 0.f;
                    zdst[lane] = 0.f;
                }
                continue;
            }
            if (ok) {
                float sacc[DW];   // S row (lane) over the unit's chunks
#pragma unroll
                for (int j = 0; j < DW; ++j) sacc[j] = 0.f;
                for (int i = 0; i < x.ntile; i += L::CHUNK) {
                    const int tb = tr.idx;
                    if (!__all_sync(ALL, bar_wait(TFULL + 8 * tr.idx, tr.phase, abort_flag))) {
                        ok = false;
                        break;
                    }
                    ring_next<NTM>(tr);
                    tc_after();
#pragma unroll
                    for (int hb = 0; hb < VPH; ++hb) {
                        const int atom = atom_of(VPH == 1 ? q : (q & ~1) + hb);
                        const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + tb * 256 + 64 * atom;
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {   // k~hi columns e = 0-15, 16-31, then k~lo
                            uint32_t v[16];
                            tmem_ld16(ta + 16 * c4, v);
#pragma unroll
                            for (int j = 0; j < 16; ++j) sacc[32 * hb + 16 * (c4 & 1) + j] += __uint_as_float(v[j]);
                        }
                    }
                    tc_before();
                    __syncwarp();
                    if (lane == 0) bar_arrive(TFREE + 8 * tb);
                }
                if (ok && !__all_sync(ALL, bar_wait(ZREADY, zr.phase, abort_flag))) ok = false;
                if (ok) {
                    ring_next<1>(zr);
                    // z[e], e = lane: head q = 2g + hh, quarter f = e >> 3, over the prologue warps
                    const float *zp = zbuf + ((q >> 1) * 4 + (lane >> 3)) * 16 + (q & 1) * 8 + (lane & 7);
                    float zs = 0.f;
#pragma unroll
                    for (int pw = 0; pw < NPRO; ++pw) zs += zp[pw * 2 * 4 * 16];
                    __syncwarp();
                    if (lane == 0) bar_arrive(ZFREE);
                    if (live) {   // row of S, then z; kept in L2 for the scan
                        const uint64_t keep = policy_evict_last();
                        float4 *row = reinterpret_cast<float4 *>(rows + lane * DW);
#pragma unroll
                        for (int j = 0; j < DW / 4; ++j)
                            st_v4_hint(row + j, make_float4(sacc[4 * j], sacc[4 * j + 1], sacc[4 * j + 2], sacc[4 * j + 3]),
                                       keep);
                        st_f32_hint(zdst + lane, zs, keep);
                    }
                }
            }
            if (!ok && live) {   // aborted: this and every later partial of the head reads NaN
                for (int e = lane; e < 32 * DW; e += 32) rows[e] = nanv;
                zdst[lane] = nanv;
            }
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
template <int DW>
struct LayC {
    // raw q ring: one tile's two TMA boxes [64 tok][2 heads x 32] bf16 (16 KB) per slot, released when the
    // prologue has used it; operand ring: the tile's query operand, 4 atoms of [64 rows (tok)][32 fp16]
    // (64-byte swizzle, 16 KB), held until the tile's MMAs complete.  DW = 64 has table slots twice as large.
    static constexpr int RAW = 5, RAW_BYTES = 16384;
    // prologue: groups of 4 warps that take turns on the tiles (three at DW = 32, two at DW = 64), so that one
    // group's waits, fences and load latencies overlap the others' arithmetic; one operand slot per group
    static constexpr int NGRP = DW == 32 ? 3 : 2, GW = 4, NPC = GW * NGRP, RPT = NPRO / GW;
    static constexpr int OPS = NGRP, OP_BYTES = 16384, ATOM = 4096;
    static constexpr int RAW_OFF = 0, OP_OFF = RAW * RAW_BYTES;
    static constexpr int TAB_BYTES = Width<DW>::TAB_BYTES;
    static constexpr int NT = DW == 32 ? 5 : 3;                     // rotary-table ring slots
    static constexpr int C_OFF = OP_OFF + OPS * OP_BYTES;           // rotary-table ring
    // prefix operands, each row scaled by a power of two (P~), one buffer per unit, double-buffered: DW = 32,
    // [128 rows (head, c)][P~hi | P~lo] fp16 (128-byte swizzle, 16 KB); DW = 64, the unit's two key halves
    // (e < 32, e >= 32), each [128 rows (virtual head, c)][P~] as one fp16 term (64-byte swizzle, 8 KB)
    static constexpr int P_BYTES = 16384, NPB = 2, PH_BYTES = 8192, VPH_C = Width<DW>::VPH;
    static constexpr int P_OFF = C_OFF + NT * TAB_BYTES;
    static constexpr int O_OFF = P_OFF + 2 * P_BYTES;               // output staging: 8 warps x [32 tok][32 c] bf16
    static constexpr int OBUF = 2048;
    // the normaliser 1 / (z . phi(q) + eps) of each tile, [4 virtual heads][64 tok] fp32, from the prologue to the
    // epilogue; and the inverse row scales of each prefix operand, [2][128] fp32
    static constexpr int NG = 2 * NGRP, G_BYTES = 1024;
    static constexpr int G_OFF = O_OFF + 8 * OBUF;
    static constexpr int S_OFF = G_OFF + NG * G_BYTES;
    // DW = 32: the table producer copies each unit's prefix states ahead of time, S into the prefix operand buffer
    // the unit will use (the prologue converts it in place: a row's raw fp32 and its fp16 hi | lo both take 128 B)
    // and z here, [2][4 heads][32] fp32
    static constexpr int Z_OFF = S_OFF + 2 * 128 * 4, Z_BYTES = 512;
    static constexpr int CTRL = Z_OFF + (DW == 32 ? 2 * Z_BYTES : 0);  // mbarriers, tensor-memory slot, abort flag
    static constexpr int BYTES = CTRL + CTRL_BYTES + 1024;          // + worst-case 1024-byte alignment pad
    // a prologue thread does four token rows of its group's tiles (the row sets that pair_offsets gives warps
    // 4 gw .. 4 gw + 3).  Warps: DW = 32, epilogue 0-7, prologue 8-19, producer 20, MMA 21, tables and prefix
    // states 22, 23 idle: six warpgroups launched at 80 registers a thread, the prologue's three raise their limit
    // to 96, the epilogue's two lower it to 72 and the last one to 40; DW = 64, epilogue 0-7, producer 8, MMA 9,
    // prologue 10-17, tables 18, at one register limit.
    static constexpr int NTHREADS = DW == 32 ? 768 : 608;
    static constexpr int W_PROD = DW == 32 ? 20 : 8, W_MMA = W_PROD + 1, W_PRO0 = DW == 32 ? 8 : 10,
                         W_TAB = DW == 32 ? 22 : 18, NEPI = 8;
    static constexpr int REG_LAUNCH = 80, REG_PRO = 96, REG_EPI = 72, REG_LOW = 40;   // DW = 32
    static constexpr int NTM = 2;                                   // tensor-memory ring (256 columns each)
    static constexpr uint32_t IDESC = idesc_f16(128, 256);
    static constexpr int TMEM_COLS = NTM * 256;
    static constexpr int NBARS = 2 * RAW + 2 * OPS + 2 * NT + 2 * NTM + 6 + 2 * NG + 2;
    static_assert(NPB == 2 && VPH_C * PH_BYTES <= P_BYTES, "two prefix buffers of P_BYTES");
    static_assert(BYTES <= SMEM_MAX, "pass C shared memory");
    static_assert(8 * NBARS + 12 <= CTRL_BYTES, "pass C control block: barriers, TMEM slot, abort flag");
    static_assert(W_PRO0 + NPC <= W_PROD || W_PRO0 >= W_MMA + 1, "pass C prologue warps apart from the producers");
    static_assert(DW != 32 || (NTHREADS == 768 && W_PRO0 == 8 && W_PROD == 20 && W_TAB == 22),
                  "DW = 32: warpgroups 2-4 prologue, 5 producers (the register split assumes it)");
    static_assert(DW != 32 || 128 * (REG_LAUNCH - REG_LOW) + 256 * (REG_LAUNCH - REG_EPI) >=
                                  128 * NGRP * (REG_PRO - REG_LAUNCH),
                  "the prologue warpgroups take no more registers than the others give up");
    static_assert(DW != 64 || (W_TAB - W_PRO0 == NPC && NTHREADS / 32 == W_TAB + 1), "DW = 64 warp roles");
    static_assert(NPB == 2 || DW != 32, "the prefix states are copied a unit ahead into the other prefix buffer");
    static_assert(GW * RPT == NPRO, "a group's rows cover the 16 row sets");
    static_assert(OP_OFF % 1024 == 0 && OP_BYTES % 1024 == 0 && P_OFF % 1024 == 0, "swizzled operands: 1 KB alignment");
    static_assert(O_OFF % 1024 == 0 && OBUF % 512 == 0, "64-byte-swizzled output boxes need 512-byte alignment");
};

// Chunk f (16 bytes) of row r of a [rows][64 B] operand or box with the 64-byte swizzle.
__device__ __forceinline__ int sw64(int r, int f) { return r * 64 + ((f ^ ((r >> 1) & 3)) << 4); }

// fp16 operand of one quarter (4 pairs) of a head: the ReLU features rotated in fp32, rounded once to fp16
// (RNE).  The features are O(1) (bf16 inputs through ReLU and a rotation), inside fp16's range; the normaliser
// is applied to the accumulator instead.  Returns four packed f16x2 words, pair j in word j.
__device__ __forceinline__ uint4 rope4_f16(const uint32_t *fw, float2 c01, float2 c23, float2 s01, float2 s23,
                                           float2 ns01, float2 ns23)
{
    const float2 a01 = make_float2(bf_low(fw[0]), bf_low(fw[1])), a23 = make_float2(bf_low(fw[2]), bf_low(fw[3]));
    const float2 b01 = make_float2(bf_high(fw[0]), bf_high(fw[1])), b23 = make_float2(bf_high(fw[2]), bf_high(fw[3]));
    const float2 y0_01 = __ffma2_rn(a01, c01, __fmul2_rn(b01, ns01));   // a c - b s
    const float2 y0_23 = __ffma2_rn(a23, c23, __fmul2_rn(b23, ns23));
    const float2 y1_01 = __ffma2_rn(b01, c01, __fmul2_rn(a01, s01));    // a s + b c
    const float2 y1_23 = __ffma2_rn(b23, c23, __fmul2_rn(a23, s23));
    const __half2 h0 = __floats2half2_rn(y0_01.x, y1_01.x), h1 = __floats2half2_rn(y0_01.y, y1_01.y);
    const __half2 h2 = __floats2half2_rn(y0_23.x, y1_23.x), h3 = __floats2half2_rn(y0_23.y, y1_23.y);
    return make_uint4(*reinterpret_cast<const uint32_t *>(&h0), *reinterpret_cast<const uint32_t *>(&h1),
                      *reinterpret_cast<const uint32_t *>(&h2), *reinterpret_cast<const uint32_t *>(&h3));
}

// Power-of-two scale that brings a row whose largest magnitude is m below 2^14 (fp16 holds up to 65504),
// and its inverse; zero, subnormal and non-finite maxima keep the scale 1 (NaN states stay NaN).
__device__ __forceinline__ void row_scale(float m, float &scale, float &inv)
{
    const int E = (int)((__float_as_uint(m) >> 23) & 0xffu);   // biased exponent: m < 2^(E - 126)
    if (E == 0 || E == 255) {
        scale = inv = 1.0f;
        return;
    }
    const int es = min(max(267 - E, 1), 253);                   // 2^(es - 127) = 2^(14 - (E - 126))
    scale = __uint_as_float((uint32_t)es << 23);
    inv = __uint_as_float((uint32_t)(254 - es) << 23);
}

// Pass C over head width DW.  The accumulator holds, per (virtual head, c)
// row and (head, token) column, sum_e P~[c][e] q~[e] with P~ = the prefix row
// times its power-of-two scale (fp16 hi + lo, 22 significant bits) and q~ =
// the rotated ReLU query in fp16 (one term); the epilogue multiplies by the
// inverse row scale and the token's 1 / (z . phi(q) + eps).  At DW = 64 the
// quad holds two heads as four virtual heads; the output of head R, half a, is
// sum over the key halves b of P_R[32 a + c][32 b + e] q~_{R, b}[e]: one set of
// MMAs with the first key half of P against the tile's operand, one with the
// second half against the operand two atoms on (atoms hold virtual heads
// 0, 2, 1, 3, so the window from atom 2 holds 1, 3), which lands both sums in
// column block R.
template <int DW>
__global__ void __launch_bounds__(LayC<DW>::NTHREADS, 1)
pass_c_tc(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mc,
          const __grid_constant__ CUtensorMap ms, const __grid_constant__ CUtensorMap mo, const LclaPlan p,
          const float *__restrict__ pref, const float eps, __nv_bfloat16 *__restrict__ out, int *__restrict__ status)
{
    using L = LayC<DW>;
    constexpr bool INL = DW == 32;   // the register split: no calls in the role code
    constexpr int R = L::RAW, O = L::OPS, NTM = L::NTM, VPH = Width<DW>::VPH, TB = L::TAB_BYTES, SZ = Width<DW>::SZ;
    constexpr int NT = L::NT, NG = L::NG;
    const int HV = p.H * VPH;   // virtual heads
    extern __shared__ __align__(1024) unsigned char smraw[];
    const uint32_t raw = s32(smraw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    unsigned char *sm = smraw + pad;
    const uint32_t sb = raw + pad;
    // FULL / RAWFREE: raw q slots (TMA landed / used by the tile's prologue group); OPREADY / OPFREE: operand
    // slots (written by the group / the tile's MMAs complete); CFULL / CEMPTY: rotary rows; TFULL / TFREE:
    // accumulators; PFREE / PREADY: prefix operands (the unit's MMAs complete / staged by every prologue warp);
    // SFREE: the prefix operand's inverse row scales read by every epilogue warp; GREADY / GFREE: normalisers;
    // PRAW: a unit's raw prefix states landed (DW = 32)
    const uint32_t FULL = sb + L::CTRL, RAWFREE = FULL + 8 * R, OPREADY = RAWFREE + 8 * R, OPFREE = OPREADY + 8 * O,
                   CFULL = OPFREE + 8 * O, CEMPTY = CFULL + 8 * NT, TFULL = CEMPTY + 8 * NT, TFREE = TFULL + 8 * NTM,
                   PFREE = TFREE + 8 * NTM, PREADY = PFREE + 16, SFREE = PREADY + 16, GREADY = SFREE + 16,
                   GFREE = GREADY + 8 * NG, PRAW = GFREE + 8 * NG;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + L::CTRL + 8 * L::NBARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tslot + 1);
    float *gbuf = reinterpret_cast<float *>(sm + L::G_OFF);   // [NG][4 vh][64 tok]
    float *sinv = reinterpret_cast<float *>(sm + L::S_OFF);   // [2][128 rows]

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int nunits = p.nseg * p.nquads * p.B;

    if (tid == 0) {
        for (int i = 0; i < R; ++i) {
            bar_init(FULL + 8 * i, 1);
            bar_init(RAWFREE + 8 * i, L::GW);
        }
        for (int i = 0; i < O; ++i) {
            bar_init(OPREADY + 8 * i, L::GW);
            bar_init(OPFREE + 8 * i, 1);
        }
        for (int i = 0; i < NT; ++i) {
            bar_init(CFULL + 8 * i, 1);
            bar_init(CEMPTY + 8 * i, L::GW);
        }
        for (int i = 0; i < NTM; ++i) {
            bar_init(TFULL + 8 * i, 1);
            bar_init(TFREE + 8 * i, L::NEPI);
        }
        for (int i = 0; i < 2; ++i) {
            bar_init(PFREE + 8 * i, 1);
            bar_init(PREADY + 8 * i, L::NPC);
            bar_init(SFREE + 8 * i, L::NEPI);
            bar_init(PRAW + 8 * i, 1);
        }
        for (int i = 0; i < NG; ++i) {
            bar_init(GREADY + 8 * i, L::GW);
            bar_init(GFREE + 8 * i, L::NEPI);
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

    auto run_producer = [&]() {
        // ---------------- producer (q and the tables are inputs: no wait on earlier kernels) ----------------
        if (lane == 0) {
            const CUtensorMap *const maps[1] = {&mq};
            const int offs[1] = {0};
            produce_boxes<R, L::RAW_BYTES, 1, 2, INL>(p, nunits, sb + L::RAW_OFF, FULL, RAWFREE, maps, offs, abort_flag);
        }
    };
    auto run_tables = [&]() {
        // ---------------- producer: rotary rows of each tile; DW = 32, also each unit's prefix states ----------------
        if (lane == 0) {
            if (DW == 32) {
                // the copy of unit k's states waits for its buffer (the MMAs of unit k - 2 done): it goes out with
                // unit k's first table rows, a few tiles before the prologue reaches the unit, and for the first
                // unit once the table ring is full (the states come from the previous kernel)
                Ring br = {0, 1u};
                int k = 0, copies = 0;
                auto prefix_copy = [&](const Unit &x, int i) -> bool {
                    if (i != (k == 0 ? min(NT, x.ntile) - 1 : 0)) return true;
                    if (k++ == 0) pdl_wait();
                    if (!bar_wait<INL>(PFREE + 8 * br.idx, br.phase, abort_flag)) return false;
                    // the quad's heads inside H: per head S (rows c, 128 B each) and z; the prologue reads heads past
                    // H as zeros
                    const int nh = min(HQ, HV - HQ * x.hq);
                    const uint32_t fb = PRAW + 8 * br.idx;
                    const float *src = pref + (((size_t)x.blk * p.B + x.b) * p.H + HQ * x.hq) * SZ;
                    bar_expect_tx(fb, (uint32_t)(nh * SZ * 4));
                    for (int j = 0; j < nh; ++j) {
                        bulk_load(sb + L::P_OFF + br.idx * L::P_BYTES + j * (DW * DW * 4), src + (size_t)j * SZ,
                                  DW * DW * 4, fb);
                        bulk_load(sb + L::Z_OFF + br.idx * L::Z_BYTES + j * (DW * 4), src + (size_t)j * SZ + DW * DW,
                                  DW * 4, fb);
                    }
                    ring_next<L::NPB>(br);
                    ++copies;
                    return true;
                };
                produce_tables<DW, NT, INL>(p, nunits, sb + L::C_OFF, CFULL, CEMPTY, &mc, &ms, abort_flag, prefix_copy);
                // let the copies issued land before the CTA releases its memory (at once unless a role gave up)
                for (int j = copies > L::NPB ? copies - L::NPB : 0; j < copies; ++j)
                    bar_wait_quiet<INL>(PRAW + 8 * (j % L::NPB), (uint32_t)((j / L::NPB) & 1));
            } else {
                produce_tables<DW, NT, INL>(p, nunits, sb + L::C_OFF, CFULL, CEMPTY, &mc, &ms, abort_flag,
                                       [](const Unit &, int) { return true; });
            }
        }
    };
    auto run_mma = [&]() {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            Ring sr = {0, 0u}, tr = {0, 1u};   // operand ready, TMEM free
            const uint64_t pdesc0 = DW == 32 ? desc_sw128(sb + L::P_OFF, 16, 1024) : desc_sw64(sb + L::P_OFF, 16, 512);
            const uint64_t qdesc0 = desc_sw64(sb + L::OP_OFF, 16, 512);
            int ub = 0, issued = 0, last_tb = 0;
            uint32_t last_phase = 0;
            Ring pr = {0, 0u};   // prefix operand staged
            bool ok = true;
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const Unit x = unit_at(p, u);
                if (x.ntile == 0) continue;
                if (!bar_wait<INL>(PREADY + 8 * pr.idx, pr.phase, abort_flag)) {
                    ok = false;
                    break;
                }
                ring_next<L::NPB>(pr);
                const uint64_t pd = pdesc0 + (uint64_t)((ub * L::P_BYTES) >> 4);
                for (int i = 0; i < x.ntile; ++i) {
                    if (!bar_wait<INL>(OPREADY + 8 * sr.idx, sr.phase, abort_flag) ||
                        !bar_wait<INL>(TFREE + 8 * tr.idx, tr.phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_after();
                    const uint32_t d = tmem + tr.idx * 256;
                    const uint64_t bd0 = qdesc0 + (uint64_t)((sr.idx * L::OP_BYTES) >> 4);
                    if (DW == 32) {
                        // K steps of 16 elements = 32 B = 2 descriptor units; P hi at +0, P lo at +64 B
                        mma_bf16(d, pd + 0, bd0 + 0, L::IDESC, 0);   // P~hi . q~
                        mma_bf16(d, pd + 2, bd0 + 2, L::IDESC, 1);
                        mma_bf16(d, pd + 4, bd0 + 0, L::IDESC, 1);   // P~lo . q~
                        mma_bf16(d, pd + 6, bd0 + 2, L::IDESC, 1);
                    } else {
#pragma unroll
                        for (int kh = 0; kh < VPH; ++kh) {   // key half kh of P against the operand from atom 2 kh
                            const uint64_t pk = pd + (uint64_t)((kh * L::PH_BYTES) >> 4);
                            const uint64_t bd = bd0 + (uint64_t)((kh * 2 * L::ATOM) >> 4);
                            mma_bf16(d, pk + 0, bd + 0, L::IDESC, kh);
                            mma_bf16(d, pk + 2, bd + 2, L::IDESC, 1);
                        }
                    }
                    mma_commit(TFULL + 8 * tr.idx);
                    mma_commit(OPFREE + 8 * sr.idx);
                    if (i == x.ntile - 1) mma_commit(PFREE + 8 * ub);
                    last_tb = tr.idx;
                    last_phase = tr.phase ^ 1u;   // TFULL runs one phase behind TFREE's producer-side parity
                    ring_next<O>(sr);
                    ring_next<NTM>(tr);
                    ++issued;
                }
                ub = (ub + 1) % L::NPB;
            }
            if (!ok && issued > 0) bar_wait_quiet<INL>(TFULL + 8 * last_tb, last_phase);
        }
    };
    auto run_prologue = [&]() {
        // ---------------- prologue: prefix staging, phi, normaliser, rotary, fp16 operand ----------------
        // Group grp of GW warps takes the tiles whose sequence number (over this CTA's units) is grp modulo NGRP
        // and writes operand slot grp.  Thread: RPT token rows (row sets RPT gw .. RPT gw + RPT - 1 of
        // pair_offsets), one quarter f of the 32 dims of head pair g; all its rows share g and f (lane bits).
        const int pw = w - L::W_PRO0, pt = tid - 32 * L::W_PRO0;
        const int grp = pw / L::GW, gw = pw % L::GW;
        const int f = lane & 3, g = (lane >> 3) & 1;   // as pair_offsets gives them
        pdl_wait();   // the prefix states come from the previous kernel
        // raw full, table full, prefix buffer free (DW = 64) or its raw states landed (DW = 32), scales read
        Ring fr = {0, 0u}, cr = {0, 0u}, br = {0, DW == 32 ? 0u : 1u}, sr = {0, 1u};
        uint32_t op_phase = 1u;                                         // operand slot grp free
        int tseq = 0;                                                   // tile sequence number
        bool ok = true;
        for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
            const Unit x = unit_at(p, u);
            if (x.ntile == 0) continue;
            const int ub = br.idx;
            const size_t pbase = ((size_t)x.blk * p.B + x.b) * p.H;
            bool fine = bar_wait<INL>((DW == 32 ? PRAW : PFREE) + 8 * br.idx, br.phase, abort_flag);
            fine = bar_wait<INL>(SFREE + 8 * sr.idx, sr.phase, abort_flag) && fine;
            if (!__all_sync(ALL, fine)) {
                ok = false;
                break;
            }
            ring_next<L::NPB>(br);
            ring_next<L::NPB>(sr);
#pragma unroll 1
            for (int rep = 0; 32 * L::NPC * rep < 512; ++rep) {
                // the quad's prefix -> A operand rows m = (virtual head, c): [P~hi | P~lo] fp16, P~ = P times the
                // row's power-of-two scale; thread (m, quarter qq of the 32 keys of each key half kh), the row's
                // four threads in lanes qq = 0..3; DW = 64: row 32 (vh % 2) + c of head vh / 2, one operand per kh
                const int ptt = pt + 32 * L::NPC * rep;
                if (ptt >= 512) break;   // whole warps
                const int m = ptt >> 2, qq = ptt & 3, vh = HQ * x.hq + (m >> 5);
                float y[VPH][8];
                float mx = 0.f;
#pragma unroll
                for (int kh = 0; kh < VPH; ++kh) {
                    float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f), b4 = a4;
                    if (vh < HV) {
                        if (DW == 32) {   // the raw row in place: head m / 32, row c = m % 32, 128 B
                            const unsigned char *rowp = sm + L::P_OFF + ub * L::P_BYTES + m * 128 + qq * 32;
                            a4 = ldsf4(rowp);
                            b4 = ldsf4(rowp + 16);
                        } else {
                            const float4 *src = reinterpret_cast<const float4 *>(
                                pref + (pbase + vh / VPH) * SZ + (size_t)(32 * (vh % VPH) + (m & 31)) * DW + 32 * kh +
                                8 * qq);
                            a4 = src[0];
                            b4 = src[1];
                        }
                    }
                    y[kh][0] = a4.x; y[kh][1] = a4.y; y[kh][2] = a4.z; y[kh][3] = a4.w;
                    y[kh][4] = b4.x; y[kh][5] = b4.y; y[kh][6] = b4.z; y[kh][7] = b4.w;
#pragma unroll
                    for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(y[kh][j]));   // NaN: fmaxf keeps the other
                }
                mx = fmaxf(mx, __shfl_xor_sync(ALL, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(ALL, mx, 2));
                if (DW == 32) __syncwarp();   // the row's four lanes have read it before any of them overwrites it
                float scale, inv;
                row_scale(mx, scale, inv);
#pragma unroll
                for (int kh = 0; kh < VPH; ++kh) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float a = y[kh][2 * j] * scale, b = y[kh][2 * j + 1] * scale;   // exact
                        const __half2 h2 = __floats2half2_rn(a, b);
                        hw[j] = *reinterpret_cast<const uint32_t *>(&h2);
                        if (DW == 32) {
                            const float2 hf = __half22float2(h2);
                            const __half2 l2 = __floats2half2_rn(a - hf.x, b - hf.y);
                            lw[j] = *reinterpret_cast<const uint32_t *>(&l2);
                        }
                    }
                    if (DW == 32)
                        store_quarter_hi_lo(sm + L::P_OFF + ub * L::P_BYTES, m, qq, hw, lw);
                    else   // DW = 64: one fp16 term, key half kh: [128 rows][32 fp16], 64-byte swizzle
                        *reinterpret_cast<uint4 *>(sm + L::P_OFF + ub * L::P_BYTES + kh * L::PH_BYTES + sw64(m, qq)) =
                            make_uint4(hw[0], hw[1], hw[2], hw[3]);
                }
                if (qq == 0) sinv[ub * 128 + m] = inv;
            }
            // z[8f, 8f+8) of virtual heads 2g, 2g+1, as (even, odd) element vectors over pairs 0-1 and 2-3; read
            // before the arrival on PREADY (DW = 32: the unit's MMAs completing frees the buffer for the next copy)
            float2 za01[2], za23[2], zb01[2], zb23[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int vh = HQ * x.hq + 2 * g + hh;
                float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f), b4 = a4;
                if (vh < HV) {
                    if (DW == 32) {
                        const unsigned char *zp = sm + L::Z_OFF + ub * L::Z_BYTES + (2 * g + hh) * 128 + 32 * f;
                        a4 = ldsf4(zp);
                        b4 = ldsf4(zp + 16);
                    } else {
                        const float4 *src = reinterpret_cast<const float4 *>(pref + (pbase + vh / VPH) * SZ + DW * DW +
                                                                             32 * (vh % VPH) + 8 * f);
                        a4 = src[0];
                        b4 = src[1];
                    }
                }
                za01[hh] = make_float2(a4.x, a4.z);
                zb01[hh] = make_float2(a4.y, a4.w);
                za23[hh] = make_float2(b4.x, b4.z);
                zb23[hh] = make_float2(b4.y, b4.w);
            }
            fence_async_smem();   // the MMAs read the prefix operand
            __syncwarp();
            if (lane == 0) bar_arrive(PREADY + 8 * ub);
            for (int i = 0; i < x.ntile; ++i) {
                const int rt = fr.idx, ct = cr.idx, gt = tseq % NG;
                const uint32_t rph = fr.phase, cph = cr.phase, gph = (uint32_t)(((tseq / NG) & 1) ^ 1);
                ring_next<R>(fr);
                ring_next<NT>(cr);
                if ((tseq++) % L::NGRP != grp) continue;   // another group's tile
                bool fine = bar_wait<INL>(FULL + 8 * rt, rph, abort_flag);
                fine = bar_wait<INL>(CFULL + 8 * ct, cph, abort_flag) && fine;
                fine = bar_wait<INL>(GFREE + 8 * gt, gph, abort_flag) && fine;
                if (!__all_sync(ALL, fine)) {
                    ok = false;
                    break;
                }
                const unsigned char *rq = sm + L::RAW_OFF + rt * L::RAW_BYTES;
                const unsigned char *tab = sm + L::C_OFF + ct * TB;
                unsigned char *op = sm + L::OP_OFF + grp * L::OP_BYTES;
                float *gt_buf = gbuf + gt * (L::G_BYTES / 4);
                // rows [0, RPT / 2) are computed before the wait for the operand slot (free once the MMAs of
                // this group's previous tile are done), so that their arithmetic overlaps those MMAs
                uint4 hq[L::RPT / 2][2];
                bool slot_ok = true;
#pragma unroll
                for (int k = 0; k < L::RPT; ++k) {
                    if (k == L::RPT / 2) {
                        slot_ok = __all_sync(ALL, bar_wait<INL>(OPFREE + 8 * grp, op_phase, abort_flag));
                        if (!slot_ok) break;
                        op_phase ^= 1u;
#pragma unroll
                        for (int k2 = 0; k2 < L::RPT / 2; ++k2) {
                            const int r2 = pair_offsets(L::RPT * gw + k2, lane).r;
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh)   // virtual head 2g + hh -> atom atom_of(2g + hh)
                                *reinterpret_cast<uint4 *>(op + atom_of(2 * g + hh) * L::ATOM + sw64(r2, f)) = hq[k2][hh];
                        }
                    }
                    const PairOffs o = pair_offsets(L::RPT * gw + k, lane);
                    // the raw features of heads 2g, 2g+1 of this row, phi applied
                    uint32_t fw[2][4];   // [head of the pair][pair j]
                    const uint4 q0 = lds128(rq + o.in0);   // head 2g
                    const uint4 q1 = lds128(rq + o.in1);   // head 2g+1
                    fw[0][0] = relu2(q0.x); fw[0][1] = relu2(q0.y); fw[0][2] = relu2(q0.z); fw[0][3] = relu2(q0.w);
                    fw[1][0] = relu2(q1.x); fw[1][1] = relu2(q1.y); fw[1][2] = relu2(q1.z); fw[1][3] = relu2(q1.w);
                    // rotary rows (DW = 64: virtual heads 2g, 2g+1 are the halves of one head and rotate with
                    // table halves 0, 1)
                    float4 c4[2], s4[2];
                    c4[0] = ldsf4(tab + o.tab);
                    s4[0] = ldsf4(tab + TB / 2 + o.tab);
                    c4[1] = VPH == 2 ? ldsf4(tab + 4096 + o.tab) : c4[0];
                    s4[1] = VPH == 2 ? ldsf4(tab + TB / 2 + 4096 + o.tab) : s4[0];
                    // z . phi(q) over the token's four quarters (lanes f, f ^ 1, f ^ 2, f ^ 3), then the factor
                    // 1 / (z . phi(q) + eps) for the epilogue
                    const float d0 = zdot4_x2(fw[0], za01[0], za23[0], zb01[0], zb23[0]);
                    const float d1 = zdot4_x2(fw[1], za01[1], za23[1], zb01[1], zb23[1]);
                    if (VPH == 2) {   // one 64-dim head: the two halves' sums add
                        float dd = d0 + d1;
                        dd += __shfl_xor_sync(ALL, dd, 1);
                        dd += __shfl_xor_sync(ALL, dd, 2);
                        if (f < 2) gt_buf[(2 * g + f) * 64 + o.r] = rcp_approx(dd + eps);
                    } else {
                        // lanes with odd f finish head 2g+1, even f head 2g: each first adds its partner's (lane ^ 1)
                        // share of the head it finishes, then the other pair of quarters (lane ^ 2)
                        const bool odd = f & 1;
                        float keep = odd ? d1 : d0;
                        keep += __shfl_xor_sync(ALL, odd ? d0 : d1, 1);
                        keep += __shfl_xor_sync(ALL, keep, 2);
                        if (f < 2) gt_buf[(2 * g + f) * 64 + o.r] = rcp_approx(keep + eps);
                    }
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const float4 cc = c4[hh], ss = s4[hh];
                        const uint4 h = rope4_f16(fw[hh], make_float2(cc.x, cc.y), make_float2(cc.z, cc.w),
                                              make_float2(ss.x, ss.y), make_float2(ss.z, ss.w),
                                              make_float2(-ss.x, -ss.y), make_float2(-ss.z, -ss.w));
                        if (k < L::RPT / 2)
                            hq[k % (L::RPT / 2)][hh] = h;
                        else   // virtual head 2g + hh -> atom atom_of(2g + hh): [64 tok][32 fp16], chunk f of row r
                            *reinterpret_cast<uint4 *>(op + atom_of(2 * g + hh) * L::ATOM + sw64(o.r, f)) = h;
                    }
                }
                if (!slot_ok) {
                    ok = false;
                    break;
                }
                // the stores above used every value this warp loaded from the raw and table slots: release both
                // with the operand and the normalisers
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    bar_arrive(OPREADY + 8 * grp);
                    bar_arrive(GREADY + 8 * gt);
                    bar_arrive(RAWFREE + 8 * rt);
                    bar_arrive(CEMPTY + 8 * ct);
                }
            }
        }
    };
    auto run_epilogue = [&]() {
        // ---------------- epilogue: tensor memory -> scaled -> bf16 -> transposed into a TMA store box ----------------
        // warp e: virtual head q = e & 3 of the quad (tensor-memory lanes 32q + c), tokens [32 hf, 32 hf + 32) of
        // the tile, hf = e >> 2.  out = accumulator x (inverse row scale of c) x (1 / (z . phi(q) + eps) of the
        // token).
        const int q = w & 3, hf = w >> 2;
        const size_t tstride = (size_t)p.H * DW;   // elements per token
        // the accumulator block of this warp's rows: its own head's (DW = 32), or column block R of head R's
        // two virtual heads (DW = 64)
        const int ocol = 64 * (VPH == 1 ? atom_of(q) : (q >> 1));
        const uint32_t obs = sb + L::O_OFF + w * L::OBUF;
        const unsigned char *obp = sm + L::O_OFF + w * L::OBUF;
        // stmatrix row of this lane: c group m = lane >> 3 (c in [8m, 8m + 8)), token 8j + k, k = lane & 7;
        // the box is [32 tok][32 c] bf16 with the 64-byte swizzle (16-byte chunk m of row r at m ^ ((r >> 1) & 3))
        const int smm = lane >> 3, smk = lane & 7;
        const uint64_t stream_pol = policy_evict_first();
        Ring tr = {0, 0u}, pr = {0, 0u}, gr = {0, 0u};   // TMEM full, prefix staged, normalisers ready
        bool ok = true;
        for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
            const Unit x = unit_at(p, u);
            if (x.ntile == 0) continue;
            const int head = HQ * x.hq + q;
            // this lane's accumulator rows c = lane / 4 + 8 k: their inverse scales
            const int sb_idx = pr.idx;
            if (!__all_sync(ALL, bar_wait<INL>(PREADY + 8 * pr.idx, pr.phase, abort_flag))) {
                ok = false;
                break;
            }
            ring_next<L::NPB>(pr);
            float rinv[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) rinv[k] = sinv[sb_idx * 128 + 32 * q + (lane >> 2) + 8 * k];
            __syncwarp();
            if (lane == 0) bar_arrive(SFREE + 8 * sb_idx);
            for (int i = 0; i < x.ntile; ++i) {
                const int tb = tr.idx, gt = gr.idx;
                bool fine = bar_wait<INL>(TFULL + 8 * tr.idx, tr.phase, abort_flag);
                fine = bar_wait<INL>(GREADY + 8 * gr.idx, gr.phase, abort_flag) && fine;
                if (!__all_sync(ALL, fine)) {
                    ok = false;
                    break;
                }
                ring_next<NTM>(tr);
                ring_next<NG>(gr);
                tc_after();
                const int t = x.t0 + i * T, nt = min(T, x.t1 - t);
                // the normalisers of this lane's token pairs (8 j + 2 (lane % 4), + 1) of the half
                float2 gn[4];
                const float *gq = gbuf + gt * (L::G_BYTES / 4) + q * 64 + 32 * hf + 2 * (lane & 3);
#pragma unroll
                for (int j = 0; j < 4; ++j) gn[j] = *reinterpret_cast<const float2 *>(gq + 8 * j);
                uint32_t v[32];
                const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + tb * 256 + ocol + 32 * hf;
                tmem_ld16x256_x4x2(ta, ta + (16u << 16), v);
                tc_before();
                __syncwarp();
                if (lane == 0) {   // the accumulator and the normalisers are in registers: free both slots
                    bar_arrive(TFREE + 8 * tb);
                    bar_arrive(GFREE + 8 * gt);
                    bulk_wait_read0();   // this warp's previous store has read its box
                }
                __syncwarp();
                // v[16 L + 4 j + i] = D[c = 16 L + lane / 4 + 8 (i >> 1)][tok = 8 j + 2 (lane % 4) + (i & 1)];
                // row c's inverse scale is rinv[2 L + (i >> 1)]
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t pk[4];
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {   // rr = 2 L + (i >> 1)
                        const int base = 16 * (rr >> 1) + 4 * j + 2 * (rr & 1);
                        const float2 o2 = __fmul2_rn(make_float2(__uint_as_float(v[base]), __uint_as_float(v[base + 1])),
                                                     __fmul2_rn(gn[j], make_float2(rinv[rr], rinv[rr])));
                        pk[rr] = pack_bf2(o2.x, o2.y);
                    }
                    const int tok = 8 * j + smk;
                    stsm4_trans(obs + tok * 64 + ((smm ^ ((tok >> 1) & 3)) << 4), pk[0], pk[1], pk[2], pk[3]);
                }
                if (nt == T) {
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0 && head < HV) tma_store3_hint(&mo, obs, LCLA_D * head, t + 32 * hf, x.b, stream_pol);
                } else {   // ragged tile: lane = token, its 64-byte row back from the box to global memory
                    __syncwarp();
                    const int tok = lane;
                    if (head < HV && 32 * hf + tok < nt) {
                        const unsigned char *row = obp + tok * 64;
                        uint4 *gp = reinterpret_cast<uint4 *>(out + ((size_t)x.b * p.N + t + 32 * hf + tok) * tstride +
                                                              (size_t)head * LCLA_D);
#pragma unroll
                        for (int m = 0; m < 4; ++m) gp[m] = lds128(row + ((m ^ ((tok >> 1) & 3)) << 4));
                    }
                    __syncwarp();
                }
                if (lane == 0) bulk_commit();
            }
        }
        if (lane == 0) bulk_wait_all();
    };
    // DW = 32: each warpgroup first sets its register limit (the host checks that the kernel launches at
    // REG_LAUNCH): the last one (producer, MMA, tables, one idle warp) lowers it, the epilogue's two lower it a
    // little, the prologue's three raise it by what the others gave up
    if (DW == 32) {
        if (w >= L::W_PROD) {
            setmaxnreg_dec<L::REG_LOW>();
            if (w == L::W_PROD)
                run_producer();
            else if (w == L::W_MMA)
                run_mma();
            else if (w == L::W_TAB)
                run_tables();
        } else if (w >= L::W_PRO0) {
            setmaxnreg_inc<L::REG_PRO>();
            run_prologue();
        } else {
            setmaxnreg_dec<L::REG_EPI>();
            run_epilogue();
        }
    } else {
        if (w == L::W_PROD)
            run_producer();
        else if (w == L::W_TAB)
            run_tables();
        else if (w == L::W_MMA)
            run_mma();
        else if (w >= L::W_PRO0)
            run_prologue();
        else
            run_epilogue();
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
