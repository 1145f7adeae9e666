// lcla_api.cu -- the C ABI declared in include/lcla.h.
//
// Validates every argument on the host before anything is enqueued, builds
// the work plan, and launches pass A (segment partial states), the scan
// (prefix states, carried state in/out) and pass C (outputs) on the caller's
// stream -- all three for a forward or a step, pass A and the scan for the
// first half of a sharded forward, the carry-in, the scan and pass C for the
// second.  Kernels: tensor cores for bf16 at d = 32 in block mode, the tiled
// CUDA-core kernels otherwise at d = 32, the generic CUDA-core kernels at
// d = 64.  Allocates nothing.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "lcla.h"
#include "lcla_ffma.cuh"
#include "lcla_scan.cuh"
#include "lcla_gen.cuh"
#include "lcla_plan.h"
#include "lcla_selftest.cuh"
#include "lcla_shard.cuh"
#include "lcla_tc.cuh"

namespace {

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Shape checks shared by both entry points and the workspace queries.
int check_shape(int B, int H, int N, int d, int L, int dtype)
{
    if (B < 1 || H < 1 || N < 0 || d < 1 || L < 1) return LCLA_ERR_INVALID_ARG;
    if (dtype != LCLA_BF16 && dtype != LCLA_F32) return LCLA_ERR_INVALID_ARG;
    if (d & 1) return LCLA_ERR_INVALID_ARG;
    if (d != LCLA_D && d != LCLA_D_WIDE) return LCLA_ERR_UNSUPPORTED;
    if (d == LCLA_D_WIDE && H > 65535) return LCLA_ERR_UNSUPPORTED;   // grid y of the d = 64 kernels
    if (N > (1 << 30)) return LCLA_ERR_UNSUPPORTED;
    if (B > 65535) return LCLA_ERR_UNSUPPORTED;
    if ((long long)B * H > 0x7fffffffLL) return LCLA_ERR_UNSUPPORTED;
    return LCLA_OK;
}

// Cut the problem into segments (see lcla_plan.h) and lay out the workspace:
// [status word, 256 B][part: nseg x B x H x (d+1) x d fp32][pref: npref x B x H x (d+1) x d fp32]
// [chunk totals of the scan, when it runs in chunks].  nblocks > 0: that many explicit blocks (their
// offsets are read on the device), always in block mode, sized by their mean length.
LclaPlan make_plan(int B, int H, int N, int L, int dtype, int nblocks = 0, int d = LCLA_D)
{
    LclaPlan p;
    memset(&p, 0, sizeof p);
    if (nblocks > 0 && N > 0) L = (int)(((long long)N + nblocks - 1) / nblocks);
    p.B = B; p.H = H; p.N = N; p.L = L; p.dtype = dtype;
    p.d = d; p.sz = (d + 1) * d;
    p.ngroups = (H + LCLA_HG - 1) / LCLA_HG;
    // tensor-core work units hold four 32-dim (virtual) heads: four heads at d = 32, two at d = 64
    p.nquads = (int)(((long long)H * (d / LCLA_D) + LCLA_TC_HQ - 1) / LCLA_TC_HQ);
    if (N == 0) return p;
    p.nb = nblocks > 0 ? nblocks : (int)(((long long)N + L - 1) / L);
    // CUDA-core CTAs per segment: head pairs at d = 32, single heads at d = 64
    const long long units = (long long)(d == LCLA_D ? p.ngroups : H) * B;
    // d = 64 runs in block mode for every block length (its kernels have no chunk mode)
    if (nblocks > 0 || L >= LCLA_T || d != LCLA_D) {
        p.chunk = 0;
        p.tc = dtype == LCLA_BF16;
        p.T = p.tc ? LCLA_TC_T : LCLA_T;
        const long long tpb = ((long long)(L < N ? L : N) + p.T - 1) / p.T;   // tiles per full block
        long long nsb;
        if (p.tc) {
            // Persistent CTAs take units (segment, head quad, batch entry)
            // round-robin.  Pick the split that minimises (1 + partial-state
            // overhead) / balance, where balance is the busy fraction of the
            // CTAs over the rounds of units and the overhead is a segment's
            // partial state per head (4224 B, written and read back) relative
            // to the head's q, k, v, out bytes.
            const long long base = (long long)p.nquads * B * p.nb;
            const long long Lb = L < N ? L : N;
            long long best = 1;
            double best_cost = 1e30;
            for (nsb = 1; nsb <= tpb && nsb <= 64; ++nsb) {
                const long long n = base * nsb;
                const long long ctas = n < LCLA_TC_CTAS ? n : LCLA_TC_CTAS;
                const long long rounds = (n + ctas - 1) / ctas;
                const double balance = (double)n / (double)(rounds * LCLA_TC_CTAS);
                const double overhead = (4.0 * 4.0 * p.sz * nsb) / (8.0 * d * (double)Lb);
                const double cost = (1.0 + overhead) / balance;
                if (cost < best_cost - 1e-9) { best_cost = cost; best = nsb; }
            }
            nsb = best;
        } else if (d != LCLA_D) {
            // fp32 at d = 64: one CTA per (segment, head, batch entry) and pass; pick the split that fills whole waves of
            // both passes' resident CTAs best, against a segment's partial state (written and read back)
            // relative to its q, k, v, out bytes
            const long long Lb = L < N ? L : N;
            const double io = 4.0 * d * (dtype == LCLA_BF16 ? 2 : 4);   // bytes per token and head
            long long best = 1;
            double best_cost = 1e30;
            for (nsb = 1; nsb <= tpb && nsb <= 64; ++nsb) {
                const long long n = units * p.nb * nsb;
                double bal = 0.0;
                for (int res : {lcla::gen::RES_A, lcla::gen::RES_C}) {
                    const long long cap = (long long)LCLA_SMS * res;
                    bal += 0.5 * (double)n / (double)(((n + cap - 1) / cap) * cap);
                }
                const double overhead = (2.0 * 4.0 * p.sz * nsb) / (io * (double)Lb);
                const double cost = (1.0 + overhead) / bal;
                if (cost < best_cost - 1e-9) { best_cost = cost; best = nsb; }
            }
            nsb = best;
        } else {
            nsb = (LCLA_TARGET_CTAS + units * p.nb - 1) / (units * p.nb);
        }
        if (nsb > tpb) nsb = tpb;
        if (nsb < 1) nsb = 1;
        p.nsb = (int)nsb;
        p.nseg = p.nb * p.nsb;
        p.npref = p.nb;
        // the tensor-core kernels index work units with 32-bit integers
        if ((long long)p.nseg * p.nquads * B > 0x7fffffffLL) p.tc = 0;
    } else {
        p.chunk = 1;
        p.T = (LCLA_T / L) * L;
        const long long ntiles = ((long long)N + p.T - 1) / p.T;
        long long tps = (ntiles * units + LCLA_TARGET_CTAS - 1) / LCLA_TARGET_CTAS;
        if (tps < 1) tps = 1;
        if (tps > ntiles) tps = ntiles;
        p.tps = (int)tps;
        p.nseg = (int)((ntiles + tps - 1) / tps);
        p.npref = p.nseg;
    }
    // the scan runs in one pass for up to SCANG_MAX_GROUPS groups (blocks, or segments in chunk mode);
    // beyond that in chunks of SCAN_CHUNK_GROUPS whole groups, whose totals it keeps in the workspace
    const int scan_groups = p.chunk ? p.nseg : p.nb;
    if (scan_groups > lcla::SCANG_MAX_GROUPS) {
        p.scs = lcla::SCAN_CHUNK_GROUPS * (p.chunk ? 1 : p.nsb);
        p.nch = (p.nseg + p.scs - 1) / p.scs;
    }
    const size_t slice = (size_t)B * H * p.sz * sizeof(float);
    p.part_off = kAlign;
    p.pref_off = p.part_off + round_up((size_t)p.nseg * slice);
    p.ctot_off = p.pref_off + round_up((size_t)p.npref * slice);
    p.ws_bytes = p.ctot_off + (p.nch ? round_up((size_t)(p.nch + 1) * slice) : 0);
    return p;
}

// What one call runs: the whole forward, or one of the two halves that a
// sequence-sharded forward splits it into (lcla_shard_begin: pass A and the
// shard's total state; lcla_shard_end: the scan from the carried-in state and
// pass C, reading the partials that the begin call left in the workspace).
enum Phase { PH_ALL, PH_BEGIN, PH_END };

// The launch grid flattens (segment, head group) into blockIdx.x.
bool grid_fits(const LclaPlan &p)
{
    return (long long)p.nseg * (p.d == LCLA_D ? p.ngroups : 1) <= 0x7fffffffLL;
}

bool misaligned(const void *ptr) { return ((uintptr_t)ptr & 15u) != 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    if (!a || !b || !na || !nb) return false;
    const uintptr_t a0 = (uintptr_t)a, a1 = a0 + na, b0 = (uintptr_t)b, b1 = b0 + nb;
    return a0 < b1 && b0 < a1;
}

// Launch with programmatic dependent launch: the kernel may start while the
// previous kernel of the stream finishes; it calls griddepcontrol.wait before
// reading anything that kernel wrote.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

unsigned scan_blocks(const LclaPlan &p)
{
    const size_t n = (size_t)p.B * p.H * (p.sz / lcla::SCAN_VEC);
    return (unsigned)((n + lcla::SCAN_THREADS - 1) / lcla::SCAN_THREADS);
}

// Partials -> prefixes: the grouped two-phase scan when its group sums fit in
// shared memory, else the one-thread-per-column serial scan.
void launch_scan(const LclaPlan &p, const float *part, float *pref, const float *state_in, float *state_out,
                 unsigned char *ws, cudaStream_t st)
{
    if (p.nch == 0) {
        const int ngroups = p.chunk ? p.nseg : p.nb;
        const size_t n4 = (size_t)p.B * p.H * (p.sz / lcla::SCAN_VEC);
        const int smem = ngroups * 32 * 16;
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(lcla::scan_states_grouped, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        launch_pdl(lcla::scan_states_grouped, dim3((unsigned)((n4 + 31) / 32)), dim3(32 * lcla::SCANG_WARPS),
                   (size_t)smem, st, p, part, pref, state_in, state_out);
    } else {
        float *ctot = reinterpret_cast<float *>(ws + p.ctot_off);
        const dim3 grid(scan_blocks(p), (unsigned)p.nch);
        launch_pdl(lcla::scan_chunk_totals, grid, dim3(lcla::SCAN_THREADS), 0, st, p, part, state_in, ctot);
        launch_pdl(lcla::scan_chunk_prefix, grid, dim3(lcla::SCAN_THREADS), 0, st, p, part, (const float *)ctot,
                   pref, state_out);
    }
}

template <typename F>
void set_smem(F *kernel, int bytes)
{
    // Idempotent; cheap compared with the launches it precedes.
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// Encoded tensor maps of recent calls, keyed by what the map encodes (kind, base address, shape): a streaming
// caller that reuses its buffers skips the host-side encode.  A map holds an address and a shape only, so a hit
// is exact even when a buffer was freed and another allocated at the same address.
class MapCache {
  public:
    bool get(int kind, const void *base, int a, int b, int c, CUtensorMap *m)
    {
        std::lock_guard<std::mutex> lock(mu_);
        for (Entry &e : e_)
            if (e.used && e.kind == kind && e.base == base && e.a == a && e.b == b && e.c == c) {
                *m = e.map;
                e.tick = ++tick_;
                return true;
            }
        return false;
    }
    void put(int kind, const void *base, int a, int b, int c, const CUtensorMap &m)
    {
        std::lock_guard<std::mutex> lock(mu_);
        Entry *v = &e_[0];
        for (Entry &e : e_) {
            if (!e.used) {
                v = &e;
                break;
            }
            if (e.tick < v->tick) v = &e;   // least recently used
        }
        *v = Entry{true, kind, base, a, b, c, ++tick_, m};
    }

  private:
    struct Entry {
        bool used;
        int kind;
        const void *base;
        int a, b, c;
        unsigned long long tick;
        CUtensorMap map;
    };
    std::mutex mu_;
    Entry e_[64] = {};
    unsigned long long tick_ = 0;
};
MapCache &map_cache()
{
    static MapCache c;
    return c;
}

// [B, N, H*d] bf16 viewed as a 3-D tensor; box = 2 heads x 64 tokens, 128-byte swizzle.
bool map_tokens(CUtensorMap *m, const void *base, int B, int N, int H)
{
    if (map_cache().get(0, base, B, N, H, m)) return true;
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)H * LCLA_D, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)H * LCLA_D * 2, (cuuint64_t)N * H * LCLA_D * 2};
    cuuint32_t box[3] = {2 * LCLA_D, LCLA_TC_T, 1};   // 128 B of a token row: 2 heads
    cuuint32_t es[3] = {1, 1, 1};
    if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    map_cache().put(0, base, B, N, H, *m);
    return true;
}

// [B, N, H*d] bf16 output blocks of one head x 32 tokens, 64-byte swizzle (TMA stores).
bool map_out_blocks(CUtensorMap *m, const void *base, int B, int N, int H)
{
    if (map_cache().get(1, base, B, N, H, m)) return true;
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)H * LCLA_D, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)H * LCLA_D * 2, (cuuint64_t)N * H * LCLA_D * 2};
    cuuint32_t box[3] = {LCLA_D, LCLA_TC_T / 2, 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    map_cache().put(1, base, B, N, H, *m);
    return true;
}

// [N, d/2] fp32 rotary table; box = 16 columns of one tile of tokens, 64-byte swizzle (d = 64: two boxes).
bool map_table(CUtensorMap *m, const float *base, int N, int d)
{
    if (map_cache().get(2, base, N, d, 0, m)) return true;
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d / 2, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)(d / 2) * 4};
    cuuint32_t box[2] = {LCLA_D / 2, LCLA_TC_T};
    cuuint32_t es[2] = {1, 1};
    if (fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    map_cache().put(2, base, N, d, 0, *m);
    return true;
}

// Pass C at d = 32 splits its registers between warpgroups (setmaxnreg): the
// split adds up only if the kernel launches at exactly LayC<32>::REG_LAUNCH
// registers a thread, so it is not launched otherwise.
bool pass_c_launch_limit_ok()
{
    static const bool ok = [] {
        cudaFuncAttributes a;
        return cudaFuncGetAttributes(&a, lcla::tc::pass_c_tc<LCLA_D>) == cudaSuccess &&
               a.numRegs == lcla::tc::LayC<LCLA_D>::REG_LAUNCH &&
               a.maxThreadsPerBlock >= lcla::tc::LayC<LCLA_D>::NTHREADS;
    }();
    return ok;
}

// Tensor-core path: returns false (nothing enqueued) when a tensor map cannot
// be encoded, so that the caller can run the CUDA-core kernels instead.  At
// d = 64 the tensors are mapped as 2H virtual heads of 32 dims.
template <int DW>
bool launch_tc(const void *q, const void *k, const void *v, const float *rc, const float *rs,
               const LclaPlan &p, float eps, void *out, const float *state_in, float *state_out,
               unsigned char *ws, cudaStream_t st, cudaEvent_t const *ev, int *rc_out, Phase ph = PH_ALL)
{
    CUtensorMap mq, mk, mv, mo, mc, ms;
    const bool a = ph != PH_END, c = ph != PH_BEGIN;
    const int HV = p.H * (DW / LCLA_D);
    if ((a && (!map_tokens(&mk, k, p.B, p.N, HV) || !map_tokens(&mv, v, p.B, p.N, HV))) ||
        (c && (!map_tokens(&mq, q, p.B, p.N, HV) || !map_out_blocks(&mo, out, p.B, p.N, HV))) ||
        !map_table(&mc, rc, p.N, DW) || !map_table(&ms, rs, p.N, DW))
        return false;
    using LA = lcla::tc::LayA<DW>;
    using LC = lcla::tc::LayC<DW>;
    if (DW == LCLA_D && c && !pass_c_launch_limit_ok()) {   // nothing enqueued
        *rc_out = LCLA_ERR_CUDA;
        return true;
    }
    float *part = reinterpret_cast<float *>(ws + p.part_off);
    float *pref = reinterpret_cast<float *>(ws + p.pref_off);
    int *status = reinterpret_cast<int *>(ws);
    const long long units = (long long)p.nseg * p.nquads * p.B;
    const dim3 grid((unsigned)(units < LCLA_TC_CTAS ? units : LCLA_TC_CTAS));
    if (a) {
        set_smem(lcla::tc::pass_a_tc<DW>, LA::BYTES);   // pass A zeroes the status word itself
        if (ev) cudaEventRecord(ev[0], st);
        lcla::tc::pass_a_tc<DW><<<grid, LA::NTHREADS, LA::BYTES, st>>>(mk, mv, mc, ms, p, part, status);
        if (ev) cudaEventRecord(ev[1], st);
    }
    launch_scan(p, part, pref, state_in, state_out, ws, st);
    if (c) {
        set_smem(lcla::tc::pass_c_tc<DW>, LC::BYTES);
        if (ev) cudaEventRecord(ev[2], st);
        launch_pdl(lcla::tc::pass_c_tc<DW>, grid, dim3(LC::NTHREADS), LC::BYTES, st, mq, mc, ms, mo, p,
                   (const float *)pref, eps, (__nv_bfloat16 *)out, status);
        if (ev) cudaEventRecord(ev[3], st);
    }
    *rc_out = cudaGetLastError() == cudaSuccess ? LCLA_OK : LCLA_ERR_CUDA;
    return true;
}

template <typename Tin>
int launch_all(const Tin *q, const Tin *k, const Tin *v, const float *rc, const float *rs,
               const LclaPlan &p, float eps, Tin *out, const float *state_in, float *state_out,
               unsigned char *ws, cudaStream_t st, cudaEvent_t const *ev, Phase ph)
{
    using G = lcla::Geo<Tin>;
    float *part = reinterpret_cast<float *>(ws + p.part_off);
    float *pref = reinterpret_cast<float *>(ws + p.pref_off);
    const dim3 grid(p.nseg * p.ngroups, p.B);
    if (ph != PH_END) {
        cudaMemsetAsync(ws, 0, sizeof(int), st);   // status word (no CUDA-core kernel sets it)
        const int smem_a = 2 * (2 * G::TILE_IN + 2 * G::TILE_TAB) + G::TILE_F;
        set_smem(lcla::pass_a_ffma<Tin>, smem_a);
        if (ev) cudaEventRecord(ev[0], st);
        lcla::pass_a_ffma<Tin><<<grid, 256, smem_a, st>>>(k, v, rc, rs, p, part);
        if (ev) cudaEventRecord(ev[1], st);
    }
    launch_scan(p, part, pref, state_in, state_out, ws, st);
    if (ph == PH_BEGIN) return cudaGetLastError() == cudaSuccess ? LCLA_OK : LCLA_ERR_CUDA;
    if (ev) cudaEventRecord(ev[2], st);

    if (!p.chunk) {
        const int smem_c = 2 * (G::TILE_IN + 2 * G::TILE_TAB) + G::TILE_F +
                           (LCLA_HG * LCLA_D * LCLA_D + LCLA_HG * LCLA_D + LCLA_T * LCLA_HG) * 4;
        set_smem(lcla::pass_c_ffma<Tin>, smem_c);
        launch_pdl(lcla::pass_c_ffma<Tin>, grid, dim3(256), smem_c, st, q, rc, rs, p, (const float *)pref, eps, out);
    } else {
        const int smem_c = 3 * G::TILE_IN + 2 * G::TILE_TAB + 4 * G::TILE_F +
                           (LCLA_HG * LCLA_T * LCLA_T + LCLA_HG * LCLA_D * LCLA_D + LCLA_HG * LCLA_D) * 4 +
                           lcla::chunk_smem_extra<Tin>();
        set_smem(lcla::pass_c_chunk_ffma<Tin>, smem_c);
        launch_pdl(lcla::pass_c_chunk_ffma<Tin>, grid, dim3(lcla::CHUNK_THREADS), smem_c, st, q, k, v, rc, rs, p,
                   (const float *)pref, eps, out);
    }
    if (ev) cudaEventRecord(ev[3], st);
    return cudaGetLastError() == cudaSuccess ? LCLA_OK : LCLA_ERR_CUDA;
}

// Head dim 64: the generic CUDA-core passes (block mode), one CTA per (segment, head, batch entry).
template <typename Tin>
int launch_gen(const Tin *q, const Tin *k, const Tin *v, const float *rc, const float *rs, const LclaPlan &p,
               float eps, Tin *out, const float *state_in, float *state_out, unsigned char *ws, cudaStream_t st,
               cudaEvent_t const *ev, Phase ph)
{
    float *part = reinterpret_cast<float *>(ws + p.part_off);
    float *pref = reinterpret_cast<float *>(ws + p.pref_off);
    const dim3 grid(p.nseg, p.H, p.B);
    if (ph != PH_END) {
        cudaMemsetAsync(ws, 0, sizeof(int), st);   // status word (no CUDA-core kernel sets it)
        if (ev) cudaEventRecord(ev[0], st);
        lcla::gen::pass_a_gen<Tin, LCLA_D_WIDE><<<grid, lcla::gen::THREADS, 0, st>>>(k, v, rc, rs, p, part);
        if (ev) cudaEventRecord(ev[1], st);
    }
    launch_scan(p, part, pref, state_in, state_out, ws, st);
    if (ph != PH_BEGIN) {
        if (ev) cudaEventRecord(ev[2], st);
        launch_pdl(lcla::gen::pass_c_gen<Tin, LCLA_D_WIDE>, grid, dim3(lcla::gen::THREADS), 0, st, q, rc, rs, p,
                   (const float *)pref, eps, out);
        if (ev) cudaEventRecord(ev[3], st);
    }
    return cudaGetLastError() == cudaSuccess ? LCLA_OK : LCLA_ERR_CUDA;
}

// Shared body of every entry point once the arguments are checked.
int run(const void *q, const void *k, const void *v, const float *rc, const float *rs,
        const LclaPlan &p, float eps, void *out, const float *state_in, float *state_out,
        void *ws, cudaStream_t st, cudaEvent_t const *ev = nullptr, Phase ph = PH_ALL)
{
    if (p.tc) {
        int status = LCLA_OK;
        const bool launched =
            p.d == LCLA_D
                ? launch_tc<LCLA_D>(q, k, v, rc, rs, p, eps, out, state_in, state_out, (unsigned char *)ws, st, ev,
                                    &status, ph)
                : launch_tc<LCLA_D_WIDE>(q, k, v, rc, rs, p, eps, out, state_in, state_out, (unsigned char *)ws, st,
                                         ev, &status, ph);
        if (launched) return status;
    }
    if (p.d != LCLA_D) {
        if (p.dtype == LCLA_BF16)
            return launch_gen<__nv_bfloat16>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                             (const __nv_bfloat16 *)v, rc, rs, p, eps, (__nv_bfloat16 *)out,
                                             state_in, state_out, (unsigned char *)ws, st, ev, ph);
        return launch_gen<float>((const float *)q, (const float *)k, (const float *)v, rc, rs, p, eps,
                                 (float *)out, state_in, state_out, (unsigned char *)ws, st, ev, ph);
    }
    if (p.dtype == LCLA_BF16)
        return launch_all<__nv_bfloat16>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                         (const __nv_bfloat16 *)v, rc, rs, p, eps,
                                         (__nv_bfloat16 *)out, state_in, state_out,
                                         (unsigned char *)ws, st, ev, ph);
    return launch_all<float>((const float *)q, (const float *)k, (const float *)v, rc, rs, p, eps,
                             (float *)out, state_in, state_out, (unsigned char *)ws, st, ev, ph);
}

// Pointer, alignment, overlap and workspace checks for one call.
int check_buffers(const void *q, const void *k, const void *v, const float *rc, const float *rs,
                  const void *out, const float *state, bool state_required, int B, int H, int N,
                  int d, int dtype, float eps, const void *ws, size_t ws_bytes, size_t need)
{
    if (!(eps >= 0.f) || !isfinite(eps)) return LCLA_ERR_INVALID_ARG;
    if (state_required && !state) return LCLA_ERR_INVALID_ARG;
    if (N == 0) {
        if (state && misaligned(state)) return LCLA_ERR_MISALIGNED;
        return LCLA_OK;
    }
    if (!q || !k || !v || !rc || !rs || !out) return LCLA_ERR_INVALID_ARG;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(rc) || misaligned(rs) ||
        misaligned(out) || (state && misaligned(state)) || (ws && misaligned(ws)))
        return LCLA_ERR_MISALIGNED;
    const size_t esz = dtype == LCLA_BF16 ? 2 : 4;
    const size_t nio = (size_t)B * N * H * d * esz;
    const size_t ntab = (size_t)N * (d / 2) * sizeof(float);
    const size_t nst = (size_t)B * H * (d + 1) * d * sizeof(float);
    if (overlaps(out, nio, q, nio) || overlaps(out, nio, k, nio) || overlaps(out, nio, v, nio) ||
        overlaps(out, nio, rc, ntab) || overlaps(out, nio, rs, ntab) ||
        overlaps(out, nio, state, nst) || overlaps(out, nio, ws, ws_bytes))
        return LCLA_ERR_INVALID_ARG;
    if (need > 0) {
        if (!ws || ws_bytes < need) return LCLA_ERR_WORKSPACE;
        if (overlaps(ws, need, q, nio) || overlaps(ws, need, k, nio) || overlaps(ws, need, v, nio) ||
            overlaps(ws, need, rc, ntab) || overlaps(ws, need, rs, ntab) || overlaps(ws, need, state, nst))
            return LCLA_ERR_INVALID_ARG;
    }
    if (state && (overlaps(state, nst, q, nio) || overlaps(state, nst, k, nio) ||
                  overlaps(state, nst, v, nio) || overlaps(state, nst, rc, ntab) ||
                  overlaps(state, nst, rs, ntab)))
        return LCLA_ERR_INVALID_ARG;
    return LCLA_OK;
}

// Sequence sharding keeps the forward's workspace and, after it, the rank's
// carried-in state (one [B, H, d+1, d] fp32 slice).
size_t shard_ws_bytes(const LclaPlan &p)
{
    return p.N == 0 ? 0 : p.ws_bytes + round_up((size_t)p.B * p.H * p.sz * sizeof(float));
}

void launch_combine(const float *totals, int nranks, int rank, const float *state_in, float *carry,
                    float *state_final, int B, int H, int d, cudaStream_t st)
{
    const size_t n4 = (size_t)B * H * ((d + 1) * d / lcla::SCAN_VEC);
    lcla::combine_rank_totals<<<(unsigned)((n4 + lcla::SCAN_THREADS - 1) / lcla::SCAN_THREADS), lcla::SCAN_THREADS,
                                0, st>>>(totals, nranks, rank, n4, state_in, carry, state_final);
}

}  // namespace

extern "C" {

size_t lcla_forward_workspace_bytes(int B, int H, int N, int d, int block_len, int dtype)
{
    if (check_shape(B, H, N, d, block_len, dtype) != LCLA_OK) return 0;
    const LclaPlan p = make_plan(B, H, N, block_len, dtype, 0, d);
    return grid_fits(p) ? p.ws_bytes : 0;
}

size_t lcla_step_workspace_bytes(int B, int H, int L, int d, int dtype)
{
    if (check_shape(B, H, L, d, L < 1 ? 1 : L, dtype) != LCLA_OK) return 0;
    const LclaPlan p = make_plan(B, H, L, L < 1 ? 1 : L, dtype, 0, d);
    return grid_fits(p) ? p.ws_bytes : 0;
}

int lcla_forward_timed(const void *q, const void *k, const void *v, const float *rope_cos,
                       const float *rope_sin, int B, int H, int N, int d, int block_len, float eps,
                       void *out, float *state_out, int dtype, void *workspace,
                       size_t workspace_bytes, void *stream, void *const *events)
{
    int rc = check_shape(B, H, N, d, block_len, dtype);
    if (rc != LCLA_OK) return rc;
    const LclaPlan p = make_plan(B, H, N, block_len, dtype, 0, d);
    if (!grid_fits(p)) return LCLA_ERR_UNSUPPORTED;
    rc = check_buffers(q, k, v, rope_cos, rope_sin, out, state_out, false, B, H, N, d, dtype, eps,
                       workspace, workspace_bytes, p.ws_bytes);
    if (rc != LCLA_OK) return rc;
    if (events && (!events[0] || !events[1] || !events[2] || !events[3])) return LCLA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaEvent_t const *ev = reinterpret_cast<cudaEvent_t const *>(events);
    if (N == 0) {
        if (ev) cudaEventRecord(ev[0], st);
        if (state_out && cudaMemsetAsync(state_out, 0, (size_t)B * H * (d + 1) * d * sizeof(float), st) != cudaSuccess)
            return LCLA_ERR_CUDA;
        if (ev) { cudaEventRecord(ev[1], st); cudaEventRecord(ev[2], st); cudaEventRecord(ev[3], st); }
        return LCLA_OK;
    }
    return run(q, k, v, rope_cos, rope_sin, p, eps, out, nullptr, state_out, workspace, st, ev);
}

int lcla_forward(const void *q, const void *k, const void *v, const float *rope_cos,
                 const float *rope_sin, int B, int H, int N, int d, int block_len, float eps,
                 void *out, float *state_out, int dtype, void *workspace, size_t workspace_bytes,
                 void *stream)
{
    return lcla_forward_timed(q, k, v, rope_cos, rope_sin, B, H, N, d, block_len, eps, out,
                              state_out, dtype, workspace, workspace_bytes, stream, nullptr);
}

size_t lcla_forward_blocks_workspace_bytes(int B, int H, int N, int d, int nblocks, int dtype)
{
    if (check_shape(B, H, N, d, 1, dtype) != LCLA_OK) return 0;
    if (N > 0 && (nblocks < 1 || nblocks > N)) return 0;
    const LclaPlan p = make_plan(B, H, N, 1, dtype, nblocks, d);
    return grid_fits(p) ? p.ws_bytes : 0;
}

int lcla_forward_blocks(const void *q, const void *k, const void *v, const float *rope_cos,
                        const float *rope_sin, int B, int H, int N, int d, const int *block_offsets,
                        int nblocks, float eps, void *out, float *state_out, int dtype, void *workspace,
                        size_t workspace_bytes, void *stream)
{
    int rc = check_shape(B, H, N, d, 1, dtype);
    if (rc != LCLA_OK) return rc;
    if (N > 0 && (nblocks < 1 || nblocks > N || !block_offsets)) return LCLA_ERR_INVALID_ARG;
    if (N > 0 && ((uintptr_t)block_offsets & 3u)) return LCLA_ERR_MISALIGNED;
    LclaPlan p = make_plan(B, H, N, 1, dtype, nblocks, d);
    if (!grid_fits(p)) return LCLA_ERR_UNSUPPORTED;
    rc = check_buffers(q, k, v, rope_cos, rope_sin, out, state_out, false, B, H, N, d, dtype, eps, workspace,
                       workspace_bytes, p.ws_bytes);
    if (rc != LCLA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        if (state_out && cudaMemsetAsync(state_out, 0, (size_t)B * H * (d + 1) * d * sizeof(float), st) != cudaSuccess)
            return LCLA_ERR_CUDA;
        return LCLA_OK;
    }
    p.boff = block_offsets;
    return run(q, k, v, rope_cos, rope_sin, p, eps, out, nullptr, state_out, workspace, st, nullptr);
}

size_t lcla_shard_workspace_bytes(int B, int H, int N, int d, int block_len, int dtype)
{
    if (check_shape(B, H, N, d, block_len, dtype) != LCLA_OK) return 0;
    const LclaPlan p = make_plan(B, H, N, block_len, dtype, 0, d);
    return grid_fits(p) ? shard_ws_bytes(p) : 0;
}

int lcla_shard_begin(const void *k, const void *v, const float *rope_cos, const float *rope_sin, int B, int H,
                     int N, int d, int block_len, float *total_out, int dtype, void *workspace,
                     size_t workspace_bytes, void *stream)
{
    int rc = check_shape(B, H, N, d, block_len, dtype);
    if (rc != LCLA_OK) return rc;
    const LclaPlan p = make_plan(B, H, N, block_len, dtype, 0, d);
    if (!grid_fits(p)) return LCLA_ERR_UNSUPPORTED;
    if (!total_out) return LCLA_ERR_INVALID_ARG;
    if (misaligned(total_out)) return LCLA_ERR_MISALIGNED;
    const size_t nst = (size_t)B * H * (d + 1) * d * sizeof(float);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) return cudaMemsetAsync(total_out, 0, nst, st) == cudaSuccess ? LCLA_OK : LCLA_ERR_CUDA;
    if (!k || !v || !rope_cos || !rope_sin) return LCLA_ERR_INVALID_ARG;
    if (misaligned(k) || misaligned(v) || misaligned(rope_cos) || misaligned(rope_sin) ||
        (workspace && misaligned(workspace)))
        return LCLA_ERR_MISALIGNED;
    const size_t need = shard_ws_bytes(p);
    if (!workspace || workspace_bytes < need) return LCLA_ERR_WORKSPACE;
    const size_t nio = (size_t)B * N * H * d * (dtype == LCLA_BF16 ? 2 : 4);
    const size_t ntab = (size_t)N * (d / 2) * sizeof(float);
    const void *reads[4] = {k, v, rope_cos, rope_sin};
    const size_t rlen[4] = {nio, nio, ntab, ntab};
    for (int i = 0; i < 4; ++i)
        if (overlaps(total_out, nst, reads[i], rlen[i]) || overlaps(workspace, need, reads[i], rlen[i]))
            return LCLA_ERR_INVALID_ARG;
    if (overlaps(total_out, nst, workspace, need)) return LCLA_ERR_INVALID_ARG;
    return run(nullptr, k, v, rope_cos, rope_sin, p, 0.f, nullptr, nullptr, total_out, workspace, st, nullptr,
               PH_BEGIN);
}

int lcla_shard_end(const void *q, const void *k, const void *v, const float *rope_cos, const float *rope_sin,
                   int B, int H, int N, int d, int block_len, float eps, const float *totals, int nranks, int rank,
                   const float *state_in, void *out, float *state_out, int dtype, void *workspace,
                   size_t workspace_bytes, void *stream)
{
    int rc = check_shape(B, H, N, d, block_len, dtype);
    if (rc != LCLA_OK) return rc;
    const LclaPlan p = make_plan(B, H, N, block_len, dtype, 0, d);
    if (!grid_fits(p)) return LCLA_ERR_UNSUPPORTED;
    if (nranks < 1 || rank < 0 || rank >= nranks || !totals) return LCLA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !isfinite(eps)) return LCLA_ERR_INVALID_ARG;
    if (misaligned(totals) || (state_in && misaligned(state_in)) || (state_out && misaligned(state_out)))
        return LCLA_ERR_MISALIGNED;
    const size_t nst = (size_t)B * H * (d + 1) * d * sizeof(float);
    const size_t ntot = nst * (size_t)nranks;
    // state_out may be state_in itself, but no other overlap with the states it is summed from
    if (overlaps(state_out, nst, totals, ntot) || (state_in != state_out && overlaps(state_out, nst, state_in, nst)))
        return LCLA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        if (state_out) launch_combine(totals, nranks, rank, state_in, nullptr, state_out, B, H, d, st);
        return cudaGetLastError() == cudaSuccess ? LCLA_OK : LCLA_ERR_CUDA;
    }
    const size_t need = shard_ws_bytes(p);
    rc = check_buffers(q, k, v, rope_cos, rope_sin, out, state_out, false, B, H, N, d, dtype, eps, workspace,
                       workspace_bytes, need);
    if (rc != LCLA_OK) return rc;
    const size_t nio = (size_t)B * N * H * d * (dtype == LCLA_BF16 ? 2 : 4);
    if (overlaps(out, nio, totals, ntot) || overlaps(workspace, need, totals, ntot) ||
        overlaps(out, nio, state_in, nst) || overlaps(workspace, need, state_in, nst))
        return LCLA_ERR_INVALID_ARG;
    float *carry = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + p.ws_bytes);
    launch_combine(totals, nranks, rank, state_in, carry, state_out, B, H, d, st);
    return run(q, k, v, rope_cos, rope_sin, p, eps, out, carry, nullptr, workspace, st, nullptr, PH_END);
}

int lcla_step(const void *q_blk, const void *k_blk, const void *v_blk, const float *cos_blk,
              const float *sin_blk, int B, int H, int L, int d, float eps, float *state, int save,
              void *out, int dtype, void *workspace, size_t workspace_bytes, void *stream)
{
    int rc = check_shape(B, H, L, d, L < 1 ? 1 : L, dtype);
    if (rc != LCLA_OK) return rc;
    const LclaPlan p = make_plan(B, H, L, L < 1 ? 1 : L, dtype, 0, d);
    if (!grid_fits(p)) return LCLA_ERR_UNSUPPORTED;
    rc = check_buffers(q_blk, k_blk, v_blk, cos_blk, sin_blk, out, state, true, B, H, L, d, dtype, eps,
                       workspace, workspace_bytes, p.ws_bytes);
    if (rc != LCLA_OK) return rc;
    if (L == 0) return LCLA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return run(q_blk, k_blk, v_blk, cos_blk, sin_blk, p, eps, out, state, save ? state : nullptr,
               workspace, st);
}

int lcla_forward_plan_info(int B, int H, int N, int d, int block_len, int dtype, int *info)
{
    const int rc = check_shape(B, H, N, d, block_len, dtype);
    if (rc != LCLA_OK) return rc;
    if (!info) return LCLA_ERR_INVALID_ARG;
    const LclaPlan p = make_plan(B, H, N, block_len, dtype, 0, d);
    if (!grid_fits(p)) return LCLA_ERR_UNSUPPORTED;
    info[0] = p.chunk;
    info[1] = p.nseg;
    info[2] = p.npref;
    info[3] = p.T;
    info[4] = p.tc;
    return LCLA_OK;
}

int lcla_forward_plan_segments(int B, int H, int N, int d, int block_len, int dtype, int *seg_t0, int *seg_t1,
                               int *seg_blk, int capacity)
{
    const int rc = check_shape(B, H, N, d, block_len, dtype);
    if (rc != LCLA_OK) return rc;
    if (!seg_t0 || !seg_t1 || !seg_blk) return LCLA_ERR_INVALID_ARG;
    const LclaPlan p = make_plan(B, H, N, block_len, dtype, 0, d);
    if (!grid_fits(p)) return LCLA_ERR_UNSUPPORTED;
    if (capacity < p.nseg) return LCLA_ERR_INVALID_ARG;
    for (int s = 0; s < p.nseg; ++s) {   // the segment map the kernels evaluate, here on the host
        const LclaSeg g = lcla_segment(p, s);
        seg_t0[s] = g.t0;
        seg_t1[s] = g.t1;
        seg_blk[s] = g.blk;
    }
    return LCLA_OK;
}

const char *lcla_status_string(int status)
{
    switch (status) {
    case LCLA_OK: return "ok";
    case LCLA_ERR_INVALID_ARG: return "invalid argument";
    case LCLA_ERR_UNSUPPORTED: return "unsupported problem (the library serves d = 32 and 64, N <= 2^30)";
    case LCLA_ERR_MISALIGNED: return "array pointer not 16-byte aligned";
    case LCLA_ERR_WORKSPACE: return "workspace missing or too small";
    case LCLA_ERR_CUDA: return "CUDA launch failed";
    case LCLA_ERR_TOO_LARGE: return "problem needs more scratch than the built-in array holds";
    default: return "unknown status";
    }
}

int lcla_version(void) { return 100; }

}  // extern "C"
