// dq_internal.cuh -- launcher declarations and small device helpers shared by
// libdq's own translation units (never by anything outside csrc/).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

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
    int32_t slot[DQ_MAX_TABLES];   // the table's column block in the output rows
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

// Division of 32-bit unsigned n by the invariant batch (T. Granlund, P. Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994, Fig. 4.1):
// t = umulhi(m, n), n / batch = (t + ((n - t) >> sh1)) >> sh2.
struct BatchDiv {
    uint32_t m, sh1, sh2;
};

struct BagArgs {
    int T, d, batch;
    const int32_t *indices;
    const int32_t *offsets;
    float *out;
    uint32_t *flags;
    BatchDiv div;
};

// Where bag (t, b) is stored: with n == 0, out[b][t*d ..]; otherwise the row of sample
// b % bl in ptr[b / bl], column block slot[t] of t_out. A kernel parameter of its own:
// folded into BagArgs it made the 64-register lookup kernels spill.
struct BagDest {
    int n, bl, t_out;
    BatchDiv div;
    float *ptr[DQ_MAX_DEST];
};

// Master and packed tables of the bag backward, passed by value (about 2.8 KB of
// parameter space). Row id of table t has the global key key_base[t] + id;
// key_base[n_tables] is the total row count and marks invalid entries.
struct RequantTables {
    float *master[DQ_MAX_TABLES];
    int64_t master_ld[DQ_MAX_TABLES];
    uint8_t *codes[DQ_MAX_TABLES];
    int64_t codes_ld[DQ_MAX_TABLES];
    uint16_t *scale_bias[DQ_MAX_TABLES];
    uint32_t key_base[DQ_MAX_TABLES + 1];
};

// Re-quantization of the rows listed by the bag backward, with the SGD step.
struct RequantArgs {
    RequantTables tabs;
    int n_tables, d;
    const uint32_t *list;      // global keys of the listed rows
    const uint32_t *count;     // number of listed rows (device)
    const uint32_t *bad;       // nonzero: the offsets were rejected, nothing to do
    const float *grad_rows;    // G of listed row i at grad_rows + i * grad_ld
    int64_t grad_ld;
    float lr;
    uint32_t *flags;
};

// The bag backward's sort and reduction. The workspace pointers are carved from
// the caller's buffer (bwd_layout).
struct BwdArgs {
    int T, d, batch;
    int64_t n;                 // number of indices = entries
    const int32_t *indices;
    const int32_t *offsets;
    const float *grad;         // [batch][T * d]
    uint32_t key_base[DQ_MAX_TABLES + 1];
    BatchDiv div;
    uint32_t *hdr;             // [0] offsets rejected, [1] rows listed
    uint32_t *keys[2];
    int32_t *bags[2];
    uint32_t *hist;            // [256][tiles]
    uint32_t *totals;          // [256]
    double *partials;          // [windows][2][d]
    uint32_t *span_slot;       // [windows] list slot of the spanning row ending there
    uint32_t *list;            // [entries]
    float *grad_rows;          // [entries][grad_ld]
    int64_t grad_ld;
    uint32_t *flags;
};

// Codebook (per-row k-means) quantizer, dequantization and bag.
struct KmeansArgs {
    const float *x;
    int64_t n, ld;
    int d, iters;
    uint8_t *codes;
    int64_t codes_ld;
    uint16_t *codebook;        // [n][16] binary16
    float *row_loss;
    int32_t *row_iters;        // [n], nullable: Lloyd iterations run for the row
    uint32_t *flags;
};

struct KmeansDequantArgs {
    const uint8_t *codes;
    int64_t codes_ld;
    const uint16_t *codebook;
    int64_t n;
    int d;
    float *out;
    int64_t out_ld;
};

struct KmeansBagTables {
    const uint8_t *codes[DQ_MAX_TABLES];
    const uint16_t *codebook[DQ_MAX_TABLES];
    int64_t n_rows[DQ_MAX_TABLES];
    int64_t codes_ld[DQ_MAX_TABLES];
};

struct KmeansBagArgs {
    int T, d, batch;
    const int32_t *indices;
    const int32_t *offsets;
    float *out;
    uint32_t *flags;
    BatchDiv div;
};

// Byte offsets of the pieces of the backward's workspace (each 256-byte aligned).
struct BwdLayout {
    size_t hdr, keys0, keys1, bags0, bags1, hist, totals, partials, span_slot, list, grad_rows, total;
    int64_t tiles, windows, grad_ld;
};
BwdLayout bwd_layout(int64_t n, int d);

inline BatchDiv make_batch_div(uint32_t dvs)
{
    uint32_t l = 0;
    while ((1ull << l) < dvs)
        ++l;
    BatchDiv r;
    r.m = (uint32_t)(((1ull << 32) * ((1ull << l) - dvs)) / dvs + 1);
    r.sh1 = l < 1 ? l : 1;
    r.sh2 = l > 1 ? l - 1 : 0;
    return r;
}

__device__ __forceinline__ uint32_t div_batch(uint32_t n, const BatchDiv &v)
{
    const uint32_t t = __umulhi(v.m, n);
    return (t + ((n - t) >> v.sh1)) >> v.sh2;
}

// The output row of bag (t, b) of a lookup (see BagArgs).
// The plain lookup's kernels take this in place of BagDest (rows go to out).
struct NoDest {
    int n;
};

template <class D>
__device__ __forceinline__ float *bag_row(const BagTables &tabs, const BagArgs &a, const D &dst, int t, int b)
{
    if constexpr (std::is_same<D, BagDest>::value) {
        if (dst.n > 0) {
            const uint32_t r = div_batch((uint32_t)b, dst.div);
            const int64_t s = (int64_t)b - (int64_t)r * dst.bl;
            return dst.ptr[r] + (s * dst.t_out + tabs.slot[t]) * a.d;
        }
    }
    return a.out + ((int64_t)b * a.T + t) * a.d;
}

cudaError_t launch_quantize(const QuantArgs &a, int mode, int num_sms, cudaStream_t stream);
cudaError_t launch_dequantize(const DequantArgs &a, int num_sms, cudaStream_t stream);
cudaError_t launch_embbag(const BagTables &tabs, const BagArgs &a, const BagDest &dst, int num_sms,
                          cudaStream_t stream);
cudaError_t launch_row_l2(const L2Args &a, int num_sms, cudaStream_t stream);
cudaError_t launch_bwd_sort_reduce(BwdArgs &a, int num_sms, cudaStream_t stream);
cudaError_t launch_kmeans(const KmeansArgs &a, cudaStream_t stream);
cudaError_t launch_kmeans_dequantize(const KmeansDequantArgs &a, int num_sms, cudaStream_t stream);
cudaError_t launch_kmeans_bag(const KmeansBagTables &tabs, const KmeansBagArgs &a, int num_sms, cudaStream_t stream);
cudaError_t launch_requant(const RequantArgs &a, int64_t max_rows, int mode, int num_sms, cudaStream_t stream);

// Sets the calling thread's dq_last_error() text (for entry points outside dq_api.cu).
void set_last_error(const char *msg);

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
