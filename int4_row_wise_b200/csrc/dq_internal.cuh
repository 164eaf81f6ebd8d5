// dq_internal.cuh -- launcher declarations and small device helpers shared by
// libdq's own translation units (never by anything outside csrc/).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dq.h"

namespace dq {

struct QuantArgs {
    const float *x;
    int64_t n, ld;
    int d;
    uint8_t *codes;
    int64_t codes_ld;
    uint16_t *scale_bias;
    float *row_loss;
    uint8_t *best_ij;
    uint32_t *flags;
};

struct DequantArgs {
    const uint8_t *codes;
    int64_t codes_ld;
    const uint16_t *scale_bias;
    int64_t n;
    int d;
    float *out;
    int64_t out_ld;
};

// Kernel parameter block for the bag: up to DQ_MAX_TABLES tables passed by value
// (2 KB of the 4 KB parameter space), so the launch needs no device allocation.
struct BagTables {
    const uint8_t *codes[DQ_MAX_TABLES];
    const uint16_t *scale_bias[DQ_MAX_TABLES];
    int64_t n_rows[DQ_MAX_TABLES];
    int64_t codes_ld[DQ_MAX_TABLES];
};

struct L2Args {
    const float *x;
    int64_t n, ld;
    int d;
    const uint8_t *codes;
    int64_t codes_ld;
    const uint16_t *scale_bias;
    double *row_err;
    double *err_sum;
};

struct BagArgs {
    int T, d, batch;
    const int32_t *indices;
    const int32_t *offsets;
    float *out;
    uint32_t *flags;
};

cudaError_t launch_quantize(const QuantArgs &a, int mode, int num_sms, cudaStream_t stream);
cudaError_t launch_dequantize(const DequantArgs &a, int num_sms, cudaStream_t stream);
cudaError_t launch_embbag(const BagTables &tabs, const BagArgs &a, int num_sms, cudaStream_t stream);
cudaError_t launch_row_l2(const L2Args &a, int num_sms, cudaStream_t stream);

__device__ __forceinline__ void raise_flag(uint32_t *flags, uint32_t bit)
{
    if (flags)
        atomicOr(flags, bit);
}

__device__ __forceinline__ bool aligned(const void *p, unsigned bytes)
{
    return (reinterpret_cast<uintptr_t>(p) & (bytes - 1)) == 0;
}

} // namespace dq
