// lcla_shard.cuh -- the one kernel of a sequence-sharded forward that the
// unsharded forward does not have (lcla_shard_end in include/lcla.h).
#pragma once

#include "lcla_scan.cuh"

namespace lcla {

// Sequence sharding: each rank holds whole blocks of one sequence.  Rank r
// starts from state_in plus the state totals of ranks 0..r-1; the state after
// the whole sequence is state_in plus all the totals.  Both sums run in rank
// order, so every rank writes the same final state bit for bit.  state_final
// may alias state_in (each thread reads its element before writing it).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(SCAN_THREADS)
combine_rank_totals(const float *__restrict__ totals, int nranks, int rank, size_t n4, const float *state_in,
                    float *carry, float *state_final)
{
    const size_t x = (size_t)blockIdx.x * SCAN_THREADS + threadIdx.x;
    if (x >= n4) return;
    const float4 *t4 = reinterpret_cast<const float4 *>(totals);
    float4 acc = state_in ? reinterpret_cast<const float4 *>(state_in)[x] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < nranks; ++r) {
        if (r == rank && carry) reinterpret_cast<float4 *>(carry)[x] = acc;
        add4(acc, __ldg(t4 + (size_t)r * n4 + x));
    }
    if (state_final) reinterpret_cast<float4 *>(state_final)[x] = acc;
}

}  // namespace lcla
