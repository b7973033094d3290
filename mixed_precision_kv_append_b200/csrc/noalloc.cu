// noalloc.cu -- loopkv_append_noalloc: the append entry point for callers that cannot
// allocate device memory (an engine whose arena already holds all of it, or a decode loop
// that cannot afford the device-wide synchronisation an allocation may cause).
//
// The append kernel reads the request ids of its batch from device memory.  Here they are
// staged in a fixed array that the library image carries, so the call allocates nothing and
// touches no staging words of the cache.  Host code may not use the array's name as an
// address (it names a host-side stand-in): the device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
#include <cuda_runtime.h>

#include <mutex>

#include "lkv_internal.h"

// Request-id staging of loopkv_append_noalloc, shared by every call on a device; each call
// writes the ids it reads before its kernel runs.
static __device__ __align__(256) int32_t g_noalloc_req_ids[LOOPKV_NOALLOC_MAX_IDS];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t *g_ids_dev[kMaxDevices]; // device address of g_noalloc_req_ids, per device (null: not yet)

// Device address of the staging array on the current device (looked up on first use).
int staging_address(int32_t **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return LOOPKV_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ids_dev[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_req_ids) != cudaSuccess || !p) {
            cudaGetLastError();
            return LOOPKV_ERR_CUDA;
        }
        g_ids_dev[dev] = static_cast<int32_t *>(p);
    }
    *out = g_ids_dev[dev];
    return LOOPKV_OK;
}

}  // namespace

extern "C" int loopkv_append_noalloc(loopkv_cache *cache, int loop, int layer, const void *k, const void *v,
                                     const int32_t *req_ids, int B, void *stream)
{
    lkv::CacheInfo ci;
    if (!cache || !k || !v || B < 0)
        return LOOPKV_ERR_INVALID_ARG;
    int rc = lkv::cache_info(cache, &ci);
    if (rc)
        return rc;
    if (loop < 0 || loop >= ci.n_loops || layer < 0 || layer >= ci.n_layers)
        return LOOPKV_ERR_INVALID_ARG;
    if (B > ci.max_batch || B > LOOPKV_NOALLOC_MAX_IDS)
        return LOOPKV_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int32_t *ids = nullptr;
    if (req_ids) {
        for (int i = 0; i < B; ++i)
            if (req_ids[i] < 0 || req_ids[i] >= ci.max_batch)
                return LOOPKV_ERR_INVALID_ARG;
        int32_t *dst = nullptr;
        rc = staging_address(&dst);
        if (rc)
            return rc;
        if (B > 0 && cudaMemcpyAsync(dst, req_ids, sizeof(int32_t) * (size_t)B, cudaMemcpyHostToDevice, s) !=
                         cudaSuccess)
            return LOOPKV_ERR_CUDA;
        ids = dst;
    }
    return lkv::launch_append(ci.st, loop * ci.n_layers + layer, ci.n_heads, ci.head_dim, ci.in_dtype,
                              ci.max_batch, k, v, ids, B, s);
}
