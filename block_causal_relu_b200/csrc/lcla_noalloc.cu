// lcla_noalloc.cu -- lcla_forward with scratch compiled into the library.
//
// For callers that cannot allocate device memory (see lcla_forward_noalloc in
// include/lcla.h).  The scratch is a file-scope device array; host code only
// knows a host-side stand-in for it under that name, so every call looks up
// its device address in the current context, and that address is what the
// kernels receive.  The lookup is not cached: a cached address would go stale
// after a device reset, or belong to another context's copy of the module when
// the caller switches contexts.
#include <cuda_runtime.h>

#include "lcla.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[LCLA_NOALLOC_SCRATCH_BYTES];

// Device address of g_scratch in the context current on this thread.
int scratch_in_current_context(void **ptr)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return LCLA_ERR_CUDA;
    *ptr = p;
    return LCLA_OK;
}

}  // namespace

extern "C" int lcla_forward_noalloc(const void *q, const void *k, const void *v, const float *rope_cos,
                                    const float *rope_sin, int B, int H, int N, int d, int block_len,
                                    float eps, void *out, float *state_out, int dtype, void *stream)
{
    const size_t need = lcla_forward_workspace_bytes(B, H, N, d, block_len, dtype);
    if (need > LCLA_NOALLOC_SCRATCH_BYTES) return LCLA_ERR_TOO_LARGE;
    void *scratch = nullptr;
    if (need > 0) {
        const int rc = scratch_in_current_context(&scratch);
        if (rc != LCLA_OK) return rc;
    }
    return lcla_forward(q, k, v, rope_cos, rope_sin, B, H, N, d, block_len, eps, out, state_out, dtype,
                        scratch, LCLA_NOALLOC_SCRATCH_BYTES, stream);
}
