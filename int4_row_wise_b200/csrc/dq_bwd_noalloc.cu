// dq_bwd_noalloc.cu -- dq_embbag_int4_bwd_sgd for callers that cannot allocate
// device memory: a plugin running inside a host program that owns the allocator, a
// process under a fixed memory budget, or code that must not grow the device heap
// once it is serving. Its scratch is one file-scope device array of
// DQ_BWD_STATIC_SCRATCH_BYTES, which every GPU that loads the library holds until
// the process exits.
//
// In host code the array's name only stands in for the symbol; its device address
// comes from cudaGetSymbolAddress, taken once per device (with that device
// current) on the first call there. That first call should therefore come before
// any stream capture. The address is cached per device ordinal until the process
// exits; a cudaDeviceReset recreates the device's context and module, after which
// the cached address is stale (the header documents that such a device must not be
// used with this entry point again). All calls share the array and it keeps the previous call's
// contents: the backward clears the only part that must start at zero (its
// 256-byte header) at the start of every call, and writes everything else before
// reading it. Calls whose work overlaps on the GPU (other streams, other host
// threads) race on the array.
#include <cstdio>
#include <mutex>

#include "dq_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_bwd_scratch[DQ_BWD_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device (set up once per device).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_bwd_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

} // namespace

extern "C" {

dq_status dq_embbag_int4_bwd_sgd_noalloc(const dq_master_table *tables, int32_t n_tables, int32_t d,
                                         const int32_t *indices, const int32_t *offsets, int32_t batch,
                                         int64_t n_indices, const float *grad_out, float lr, int32_t mode,
                                         uint32_t *d_flags, void *cuda_stream)
{
    const size_t need = dq_embbag_int4_bwd_workspace_bytes(d, n_indices);
    if (need > (size_t)DQ_BWD_STATIC_SCRATCH_BYTES) {
        char buf[256];
        snprintf(buf, sizeof buf,
                 "d = %d and n_indices = %lld need %zu bytes of scratch, above the static %u bytes; "
                 "use dq_embbag_int4_bwd_sgd with a workspace",
                 d, (long long)n_indices, need, (unsigned)DQ_BWD_STATIC_SCRATCH_BYTES);
        dq::set_last_error(buf);
        return DQ_ERR_INVALID_ARG;
    }
    void *scratch = nullptr;
    if (n_indices > 0 && need > 0) {
        const cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess) {
            char buf[256];
            snprintf(buf, sizeof buf, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
            dq::set_last_error(buf);
            return DQ_ERR_CUDA;
        }
    }
    return dq_embbag_int4_bwd_sgd(tables, n_tables, d, indices, offsets, batch, n_indices, grad_out, lr, mode,
                                  scratch, DQ_BWD_STATIC_SCRATCH_BYTES, d_flags, cuda_stream);
}

} // extern "C"
