// lcla_selftest.cuh -- self-test of the bounded mbarrier wait that every
// tensor-core kernel uses (lcla_selftest_bounded_wait in include/lcla.h);
// compiled into lcla_api.cu, the one translation unit that holds the kernels.
//
// One thread initialises an mbarrier and waits on its first phase with the
// same bar_wait as the passes.  With arrive_first the phase is completed
// before the wait, which must return at once; without it nothing ever
// arrives, and the wait must give up after its limit, raise the CTA's abort
// flag and report failure -- the path that turns a lost TMA load or MMA into
// a status bit and NaN partial states instead of a hung GPU.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "lcla.h"
#include "lcla_tc.cuh"

namespace lcla_selftest {

__global__ void bounded_wait_probe(int arrive_first, unsigned long long *result)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    const uint32_t b = lcla::tc::s32(&bar);
    abort_flag = 0;
    lcla::tc::bar_init(b, 1);
    lcla::tc::bar_fence_init();
    if (arrive_first) lcla::tc::bar_arrive(b);
    const uint64_t t0 = lcla::tc::gtimer();
    const bool done = lcla::tc::bar_wait(b, 0u, &abort_flag);
    const uint64_t t1 = lcla::tc::gtimer();
    result[0] = done ? 0ull : 1ull;
    result[1] = (unsigned long long)(t1 - t0);
    result[2] = (unsigned long long)abort_flag;
}

}  // namespace lcla_selftest

extern "C" int lcla_selftest_bounded_wait(int arrive_first, unsigned long long *result, void *stream)
{
    if (!result) return LCLA_ERR_INVALID_ARG;
    if ((uintptr_t)result & 7u) return LCLA_ERR_MISALIGNED;
    lcla_selftest::bounded_wait_probe<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(arrive_first, result);
    return cudaGetLastError() == cudaSuccess ? LCLA_OK : LCLA_ERR_CUDA;
}
