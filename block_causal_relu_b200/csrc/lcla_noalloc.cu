// lcla_noalloc.cu -- lcla_forward with scratch compiled into the library.
//
// For callers that cannot allocate device memory (see lcla_forward_noalloc in
// include/lcla.h).  The scratch is a file-scope device array; host code only
// knows a host-side stand-in for it under that name, so its device address is
// looked up once per device, with that device current, and that address is
// what the kernels receive.
#include <cuda_runtime.h>

#include <mutex>

#include "lcla.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[LCLA_NOALLOC_SCRATCH_BYTES];

std::mutex g_lock;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up on first use).
int scratch_on_current_device(void **ptr)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LCLA_ERR_CUDA;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return LCLA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *ptr = g_scratch_ptr[dev];
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
        const int rc = scratch_on_current_device(&scratch);
        if (rc != LCLA_OK) return rc;
    }
    return lcla_forward(q, k, v, rope_cos, rope_sin, B, H, N, d, block_len, eps, out, state_out, dtype,
                        scratch, LCLA_NOALLOC_SCRATCH_BYTES, stream);
}
