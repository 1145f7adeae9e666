/*
 * lcla.h -- block-causal ReLU linear attention with a carried fp32 state,
 * for NVIDIA B200 (sm_100a).  C ABI: plain pointers and sizes only.
 *
 * The operation ("Implementing Block Causal Linear Attention for Long Video
 * Generation with Sana": sections "The Linear Attention Kernel", "Rotary
 * Position Embeddings", "Chunk-Wise Causality"; "Block Causal Linear
 * Attention" note: "What SANA-Video Actually Uses"; "[feat] LongSANA" PR:
 * causal linear attention KV cache).  Per batch entry b and head h, with
 * phi = ReLU, R_n the rotary embedding at token n (interleaved pairs (2p,2p+1),
 * (x,y) -> (x c - y s, x s + y c), c = rope_cos[n][p], s = rope_sin[n][p]) and
 * blk(n) = n / block_len:
 *
 *   out_i = sum_{j: blk(j) <= blk(i)} v_j (R_j phi(k_j) . R_i phi(q_i))
 *           / ( sum_{same j} phi(k_j) . phi(q_i) + eps )
 *
 * i.e. a token attends to every token of its own block (both directions) and
 * of all earlier blocks.  The carried state of one (b, h) is
 *   S[c][e] = sum_j v_j[c] (R_j phi(k_j))[e]      (d x d, row = value dim)
 *   z[e]    = sum_j phi(k_j)[e]                     (d, unrotated key sum)
 * stored as float32 [d+1][d]: rows 0..d-1 hold S, row d holds z.
 *
 * Layouts (row-major, C order):
 *   q, k, v, out        [B, N, H, d], element type `dtype` (out has q's type)
 *   rope_cos, rope_sin  [N, d/2] float32, shared by every b and h
 *   state               [B, H, d+1, d] float32
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     allocates nothing, keeps no per-call state between calls, and never
 *     frees caller memory.  The one exception is lcla_forward_noalloc, which
 *     uses a scratch array compiled into the library (see its comment).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.  Results are valid
 *     once the stream has reached the work.
 *   - Arguments are validated before anything is enqueued; on any error code
 *     other than LCLA_ERR_CUDA nothing was enqueued and no memory was touched.
 *   - Every array pointer must be 16-byte aligned (LCLA_ERR_MISALIGNED).
 *   - d must be 32 or 64 (the pages set linear_head_dim to 32 or 64: "Implementing
 *     Block Causal Linear Attention ...", section "Integration into Sana's
 *     Video Backbone"); other head dims: LCLA_ERR_UNSUPPORTED.  bf16 runs on
 *     tensor cores at both head dims (at d = 32 for block_len >= 64; shorter
 *     blocks take a CUDA-core kernel whose tiles hold whole blocks).  float32
 *     runs on CUDA cores; at d = 64 with one thread block per (segment, head,
 *     batch entry), so H <= 65535 at d = 64.
 *   - `out` must not overlap q, k, v, the tables, the state or the workspace
 *     (LCLA_ERR_INVALID_ARG).
 *   - eps must be finite and >= 0.
 *   - The results do not depend on the stream or on run-to-run timing: the
 *     kernels use no floating-point atomics, so identical calls give
 *     bit-identical outputs.
 */
#ifndef LCLA_H
#define LCLA_H

#include <stddef.h>

#if defined(__GNUC__)
#define LCLA_API __attribute__((visibility("default")))
#else
#define LCLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LCLA_OK = 0,
    LCLA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad dtype, overlap, bad eps */
    LCLA_ERR_UNSUPPORTED = 2,   /* valid request the library does not serve (d not 32 or 64, N > 2^30) */
    LCLA_ERR_MISALIGNED = 3,    /* an array pointer is not 16-byte aligned */
    LCLA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than the query says */
    LCLA_ERR_CUDA = 5,          /* a CUDA launch failed; see cudaGetLastError */
    LCLA_ERR_TOO_LARGE = 6      /* lcla_forward_noalloc: problem needs more scratch than built in */
} lcla_status;

typedef enum {
    LCLA_BF16 = 0,              /* q, k, v, out are bfloat16 */
    LCLA_F32 = 1                /* q, k, v, out are float32 */
} lcla_dtype;

/*
 * Workspace bytes lcla_forward needs for this problem (0 when the arguments
 * are invalid).  Depends only on the arguments, never on the device.
 */
LCLA_API size_t lcla_forward_workspace_bytes(int B, int H, int N, int d, int block_len, int dtype);

/*
 * Whole-sequence forward.
 *   q, k, v     [B, N, H, d] device, dtype.  Read only.
 *   rope_cos/sin [N, d/2] float32 device.  Read only.
 *   B, H >= 1; N >= 0 (N = 0: no outputs, state_out set to zero);
 *   block_len >= 1 (the last block holds the N mod block_len leftover tokens).
 *   eps         added to every denominator.
 *   out         [B, N, H, d] device, dtype.  Written.
 *   state_out   [B, H, d+1, d] float32 device, or NULL.  Written with the
 *               state after the last block (S and z summed over all tokens).
 *   workspace   device scratch of at least lcla_forward_workspace_bytes(...)
 *               bytes, 16-byte aligned (may be NULL when that is 0).  Its
 *               contents on entry are ignored; it must not be shared with
 *               another call that is in flight at the same time.
 * Returns an lcla_status.
 */
LCLA_API int lcla_forward(const void *q, const void *k, const void *v,
                 const float *rope_cos, const float *rope_sin,
                 int B, int H, int N, int d, int block_len, float eps,
                 void *out, float *state_out, int dtype,
                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * lcla_forward plus pass timing: `events` points to 4 cudaEvent_t handles
 * created by the caller (cudaEventDefault flags); they are recorded on
 * `stream` before pass A (partial states), before the scan, before pass C
 * (outputs) and after pass C, so cudaEventElapsedTime gives each pass's
 * device time.  events == NULL behaves exactly like lcla_forward.  Same
 * arguments, ownership and errors as lcla_forward.
 */
LCLA_API int lcla_forward_timed(const void *q, const void *k, const void *v,
                 const float *rope_cos, const float *rope_sin,
                 int B, int H, int N, int d, int block_len, float eps,
                 void *out, float *state_out, int dtype,
                 void *workspace, size_t workspace_bytes, void *stream,
                 void *const *events);

/*
 * Workspace bytes lcla_forward_blocks needs for `nblocks` explicit blocks
 * (0 when the arguments are invalid).  Depends only on the arguments.
 */
LCLA_API size_t lcla_forward_blocks_workspace_bytes(int B, int H, int N, int d, int nblocks, int dtype);

/*
 * Whole-sequence forward with explicit block boundaries instead of uniform
 * blocks: block b holds tokens [block_offsets[b], block_offsets[b+1]), and a
 * token attends to its own block and every earlier block, as in lcla_forward.
 * The pages name a non-uniform partition as the one a released model
 * configuration uses ("Add SANA-WM camera-controlled image-to-video
 * pipeline", the review reply on uniform-only chunking: `first_chunk_plus_one`
 * is the live configuration, e.g. a first block one latent frame longer).
 *   block_offsets  int32 device array of nblocks + 1 offsets, 4-byte aligned,
 *                  0 = o[0] < o[1] < ... < o[nblocks] = N.  Read only, on the
 *                  device: the host cannot check it.  Offsets outside [0, N]
 *                  are clamped and an inverted pair is an empty block, so a
 *                  malformed array never reads or writes out of bounds, but
 *                  the outputs of tokens it misses or covers twice are then
 *                  undefined.
 *   nblocks        1 <= nblocks <= N when N > 0.
 * Every other argument, ownership and error as lcla_forward; the workspace is
 * sized by lcla_forward_blocks_workspace_bytes.  Blocks of any length run on
 * the whole-block path (tensor cores for bf16), with ragged tiles at block
 * ends.
 */
LCLA_API int lcla_forward_blocks(const void *q, const void *k, const void *v,
                 const float *rope_cos, const float *rope_sin,
                 int B, int H, int N, int d, const int *block_offsets, int nblocks, float eps,
                 void *out, float *state_out, int dtype,
                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * Causal temporal convolution of the Mix-FFN with a cached last frame, the
 * step after attention in a block.  The pages say the causal Mix-FFN keeps
 * the previous block's last frame for its temporal convolution ("Block Causal
 * Linear Attention", section "What SANA-Video Actually Uses"; "[feat]
 * LongSANA": causal computation for the Mix-FFN, the convolution in the MLP)
 * and give no kernel size; one retained frame is read as a depthwise causal
 * convolution of size 2 over latent frames:
 *   y[b, f, s, c] = weight[0][c] x[b, f, s, c] + weight[1][c] x[b, f-1, s, c]
 *                   + bias[c]
 * where x[b, -1, s, c] is cache[b, s, c] (zeros when cache is NULL).
 *   x, y     [B, F * S, C] device, dtype (token f * S + s of frame f); F >= 0
 *            frames of S >= 1 tokens; C >= 8, a multiple of 8.  y must not
 *            overlap x, the cache, weight or bias.
 *   weight   [2][C] float32 device; bias [C] float32 device or NULL.
 *   cache    [B, S, C] device, dtype, or NULL (no earlier frame).  Read; with
 *            save = 1 it is overwritten with the last frame x[b, F-1] (the
 *            next block's history); save = 0 leaves it bit-unchanged (several
 *            denoising steps per block).  It must not overlap x.
 * Every pointer 16-byte aligned.  Computed in fp32, y rounded to dtype.
 * Returns an lcla_status (F = 0: LCLA_OK, nothing enqueued).
 */
LCLA_API int lcla_temporal_conv(const void *x, int B, int F, int S, int C,
                 const float *weight, const float *bias, void *cache, int save,
                 void *y, int dtype, void *stream);

/*
 * Sequence-sharded forward, in two calls per rank with one exchange between
 * them.  The pages carry one fixed-size cumulative state from earlier blocks
 * to later ones ("Block Causal Linear Attention", introduction and section
 * "What SANA-Video Actually Uses": a block needs only the cumulative
 * attention state and key summary of the blocks before it), so a sequence
 * cut into runs of whole blocks, one per rank, needs from the ranks before
 * it only the sum of their states.  Rank r of R holds tokens
 * [t_r, t_{r+1}) with t_r a multiple of block_len (the last rank may end in
 * a ragged block), the tables' rows at those absolute positions, and N =
 * t_{r+1} - t_r >= 0 (a rank may hold no tokens).
 *
 *   1. lcla_shard_begin: the state total (S, z summed over the rank's tokens,
 *      [B, H, d+1, d] fp32) into total_out.
 *   2. The caller gathers the R totals in rank order into one device array
 *      [R][B, H, d+1, d] (one all-gather of B*H*(d+1)*d*4 bytes per rank).
 *   3. lcla_shard_end: the rank's outputs, each block using state_in plus the
 *      totals of ranks 0..r-1 plus its own blocks; and, if state_out is not
 *      NULL, the state after the whole sequence, state_in plus all R totals,
 *      summed in rank order so that every rank writes the same bits.
 *
 * The outputs equal those of lcla_forward on the whole sequence with
 * state_in added to every block's state, up to the order of fp32 additions.
 * Both calls take the same B, H, N, d, block_len, dtype and the same
 * workspace, whose contents lcla_shard_end reads (pass A's partial states):
 * nothing else may use it in between.  A mismatch is not detected and gives
 * wrong outputs.
 */
LCLA_API size_t lcla_shard_workspace_bytes(int B, int H, int N, int d, int block_len, int dtype);

/*
 *   k, v         [B, N, H, d] device, dtype: the rank's tokens.  Read only.
 *   rope_cos/sin [N, d/2] float32 device, rows at the tokens' absolute
 *                positions.  Read only.
 *   total_out    [B, H, d+1, d] float32 device.  Written (zeros when N = 0).
 *   workspace    at least lcla_shard_workspace_bytes(...) bytes, 16-byte
 *                aligned; it must not overlap the other arrays.
 * Returns an lcla_status.
 */
LCLA_API int lcla_shard_begin(const void *k, const void *v,
                 const float *rope_cos, const float *rope_sin,
                 int B, int H, int N, int d, int block_len,
                 float *total_out, int dtype,
                 void *workspace, size_t workspace_bytes, void *stream);

/*
 *   q, k, v      [B, N, H, d] device, dtype: the rank's tokens (k and v as
 *                given to lcla_shard_begin; they are read again only when
 *                block_len < 64).  Read only.
 *   rope_cos/sin as for lcla_shard_begin.
 *   totals       [nranks][B, H, d+1, d] float32 device: every rank's
 *                total_out, in rank order.  Read only.
 *   nranks >= 1, 0 <= rank < nranks.
 *   state_in     [B, H, d+1, d] float32 device, or NULL (zero): the state
 *                before the whole sequence.  Read only.
 *   out          [B, N, H, d] device, dtype.  Written.
 *   state_out    [B, H, d+1, d] float32 device, or NULL.  Written with the
 *                state after the whole sequence; may be state_in itself, but
 *                must not otherwise overlap it or totals.
 *   workspace    the one lcla_shard_begin used, unchanged since.
 * With N = 0 only state_out is written.  Returns an lcla_status.
 */
LCLA_API int lcla_shard_end(const void *q, const void *k, const void *v,
                 const float *rope_cos, const float *rope_sin,
                 int B, int H, int N, int d, int block_len, float eps,
                 const float *totals, int nranks, int rank, const float *state_in,
                 void *out, float *state_out, int dtype,
                 void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes lcla_step needs (0 when the arguments are invalid). */
LCLA_API size_t lcla_step_workspace_bytes(int B, int H, int L, int d, int dtype);

/*
 * Streaming step: one block of L tokens against the carried state
 * ("[feat] LongSANA" PR: multi-step denoising per chunk against the cache,
 * and the cache's enable_save switch).
 *   q, k, v     [B, L, H, d] device, dtype: the block's tokens.
 *   cos/sin     [L, d/2] float32 device: table rows at the block's absolute
 *               positions.
 *   L >= 0 (L = 0: nothing is done).
 *   state       [B, H, d+1, d] float32 device, in/out.  P = state + (S, z)
 *               of this block; every output uses P.  save != 0: state
 *               becomes P.  save == 0: state is not written (bit-unchanged),
 *               so the same block can be evaluated again, e.g. once per
 *               denoising step, before a final call with save = 1.
 *   out         [B, L, H, d] device, dtype.  Written.
 *   workspace   as for lcla_forward, sized by lcla_step_workspace_bytes.
 * Returns an lcla_status.
 */
LCLA_API int lcla_step(const void *q_blk, const void *k_blk, const void *v_blk,
              const float *cos_blk, const float *sin_blk,
              int B, int H, int L, int d, float eps,
              float *state, int save, void *out, int dtype,
              void *workspace, size_t workspace_bytes, void *stream);

/*
 * How lcla_forward cuts this problem, for benchmarks and tests: writes
 * info[0] = 1 when tiles hold whole blocks (d = 32 and block_len < 64), else 0;
 * info[1] = segments (partial states written by the first pass);
 * info[2] = prefix states (blocks, or segments when info[0] = 1);
 * info[3] = tokens per tile; info[4] = 1 when the tensor-core kernels run
 * (bf16 in block mode: d = 32 with block_len >= 64, or d = 64 at any block
 * length), else 0.  `info` holds 5 ints.  Returns an lcla_status; touches no
 * device.
 */
LCLA_API int lcla_forward_plan_info(int B, int H, int N, int d, int block_len, int dtype,
                                    int *info);

/*
 * The segments lcla_forward cuts this problem into (uniform blocks), from the
 * same segment map the kernels evaluate: segment s covers tokens
 * [seg_t0[s], seg_t1[s]) (possibly empty) and, in block mode, lies in block
 * seg_blk[s] (-1 in chunk mode).  The three int arrays are HOST memory of at
 * least `capacity` entries; capacity must be >= info[1] of
 * lcla_forward_plan_info.  Returns an lcla_status; touches no device.
 */
LCLA_API int lcla_forward_plan_segments(int B, int H, int N, int d, int block_len, int dtype,
                                        int *seg_t0, int *seg_t1, int *seg_blk, int capacity);

/*
 * lcla_forward for callers that cannot allocate device memory.  (The paper
 * has no counterpart: this is a packaging choice of this library.)
 *
 * Some callers have no way to obtain scratch memory: a plugin running inside
 * a host application whose device memory is owned by that application's own
 * pool, or a real-time loop that must not enter the driver's allocator
 * (cudaMalloc and cudaFree can block and synchronise the device).  This entry
 * point takes the same arguments as lcla_forward minus the workspace, and
 * uses instead a fixed scratch array of LCLA_NOALLOC_SCRATCH_BYTES compiled
 * into the library.  Every GPU that loads the library holds that array until
 * the process exits.  It allocates nothing.
 *
 *   - Returns LCLA_ERR_TOO_LARGE, with nothing enqueued, when the problem
 *     needs more scratch than the array holds, i.e. when
 *     lcla_forward_workspace_bytes(B, H, N, d, block_len, dtype) >
 *     LCLA_NOALLOC_SCRATCH_BYTES.  Other errors are those of lcla_forward.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress)
 *     in the context current on the calling thread, so it follows the device
 *     that is current, a context the caller created and made current, and a
 *     device reset.  The first call in a context loads the library's device
 *     code into it; make that first call before any stream capture.
 *     `stream` must belong to the current context.
 *   - The workspace's device status word (LCLA_DEVICE_STATUS_*) lives in the
 *     library's array, which the caller cannot read: on this entry point a
 *     bounded wait that gives up shows only as NaN outputs and state.
 *   - All calls on a device share the one array, and it keeps the previous
 *     call's contents (each call re-initialises what it reads).  Calls whose
 *     GPU work overlaps -- on different streams, or from different host
 *     threads -- race on the array and give wrong results: serialise them.
 */
#define LCLA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
LCLA_API int lcla_forward_noalloc(const void *q, const void *k, const void *v,
                 const float *rope_cos, const float *rope_sin,
                 int B, int H, int N, int d, int block_len, float eps,
                 void *out, float *state_out, int dtype, void *stream);

/*
 * Device status of a call.  The first 4 bytes of the workspace of
 * lcla_forward, lcla_forward_blocks, lcla_step and the shard calls hold an int
 * that the call zeroes first -- on the tensor-core path its first kernel does,
 * before any of its waits can give up (lcla_shard_end keeps
 * lcla_shard_begin's) -- and
 * that its tensor-core kernels OR bits into when one of their bounded waits
 * (1 s) gives up: bit 0 pass A, bit 1 pass C.  A CTA that gives up lets its
 * copies and MMAs in flight land, frees its tensor memory, writes NaN partial
 * states and returns, so the outputs are NaN instead of the GPU hanging; the
 * status is read once the stream has reached the call.
 */
#define LCLA_DEVICE_STATUS_PASS_A 1
#define LCLA_DEVICE_STATUS_PASS_C 2

/*
 * Self-test of that bounded wait: one thread waits on an mbarrier phase with
 * the kernels' wait.  arrive_first != 0: the phase is completed first and the
 * wait must return at once; 0: nothing arrives and the wait must give up after
 * its limit (about 1 s).  Writes result[0] = 1 if the wait gave up (else 0),
 * result[1] = nanoseconds spent waiting, result[2] = the abort flag it left.
 *   result   3 x uint64 device array, 8-byte aligned.
 * Returns an lcla_status; the kernel runs on `stream`.
 */
LCLA_API int lcla_selftest_bounded_wait(int arrive_first, unsigned long long *result, void *stream);

/* Static, human-readable name of a status code. */
LCLA_API const char *lcla_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
LCLA_API int lcla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LCLA_H */
