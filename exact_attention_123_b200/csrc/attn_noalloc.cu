// attn_noalloc.cu -- the backward entry point for callers that cannot allocate
// device memory: the backward's scratch is a fixed array owned by the library.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/libattn.h"

namespace {

// Backward scratch for attn_bwd_noalloc.  One copy exists on every GPU that loads
// the library and stays allocated until the process exits.  In host code this name
// is only a handle for the runtime, not a device address: the address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct ScratchAddress {
    std::once_flag once;
    void *ptr = nullptr;
    cudaError_t err = cudaSuccess;
};
ScratchAddress g_scratch[kMaxDevices];

// Device address of the current device's copy, looked up once per device (with
// that device current) the first time it is needed.
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
    ScratchAddress &s = g_scratch[dev];
    std::call_once(s.once, [&] { s.err = cudaGetSymbolAddress(&s.ptr, g_noalloc_scratch); });
    if (s.err != cudaSuccess || s.ptr == nullptr) return ATTN_ERR_CUDA;
    *out = s.ptr;
    return ATTN_OK;
}

}  // namespace

extern "C" int attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const float *lse,
                                const void *dout, void *dq, void *dk, void *dv, int B, int H, int N, int d,
                                float scale, int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep,
                                void *stream) {
    const size_t need = attn_bwd_deterministic_workspace_bytes(B, H, N, d);
    if (need == 0)  // invalid sizes: let the backward report the argument error
        return attn_bwd_deterministic(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, is_causal, cu_seqlens,
                                      key_keep, nullptr, 0, stream);
    if (need > ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    void *ws = nullptr;
    const int rc = scratch_address(&ws);
    if (rc != ATTN_OK) return rc;
    return attn_bwd_deterministic(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, is_causal, cu_seqlens,
                                  key_keep, ws, ATTN_NOALLOC_SCRATCH_BYTES, stream);
}
