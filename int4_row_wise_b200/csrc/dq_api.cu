// dq_api.cu -- the C ABI of libdq (declared in include/dq.h): host-side argument
// validation, device checks and kernel dispatch. Every argument is checked before
// anything is enqueued; the library allocates no memory.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "dq_internal.cuh"

namespace {

thread_local std::string g_last_error;

dq_status fail(dq_status s, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

dq_status ok()
{
    g_last_error.clear();
    return DQ_OK;
}

// Test hook: DQ_FAULT_INJECT=launch makes every entry point that would launch a
// kernel return DQ_ERR_CUDA instead, with nothing enqueued.
bool fault_injected()
{
    const char *v = getenv("DQ_FAULT_INJECT");
    return v && strcmp(v, "launch") == 0;
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];  // 0 = unknown, -1 = unsupported, else the SM count

// Checks that the current device is an sm_100-class part; returns its SM count.
dq_status current_device(int *num_sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return fail(DQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return fail(DQ_ERR_UNSUPPORTED, "device ordinal %d beyond the library's table", dev);
    int sms = g_sms[dev].load(std::memory_order_relaxed);
    if (sms == 0) {
        int major = 0, count = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return fail(DQ_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        sms = major == 10 ? count : -1;
        g_sms[dev].store(sms, std::memory_order_relaxed);
    }
    if (sms < 0)
        return fail(DQ_ERR_UNSUPPORTED, "device %d is not an sm_100 (B200-class) GPU", dev);
    *num_sms = sms;
    return DQ_OK;
}

dq_status launched(cudaError_t e, const char *what)
{
    if (e != cudaSuccess)
        return fail(DQ_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
    return ok();
}

} // namespace

namespace dq {
void set_last_error(const char *msg)
{
    g_last_error = msg;
}
} // namespace dq

extern "C" {

dq_status dq_quantize_rows_int4(const float *x, int64_t n_rows, int32_t d, int64_t x_ld, uint8_t *codes,
                                int64_t codes_ld, uint16_t *scale_bias, float *row_loss, uint8_t *best_ij,
                                int32_t mode, uint32_t *d_flags, void *cuda_stream)
{
    if (n_rows < 0)
        return fail(DQ_ERR_INVALID_ARG, "n_rows = %lld < 0", (long long)n_rows);
    if (d < 1 || d > DQ_MAX_D)
        return fail(DQ_ERR_INVALID_ARG, "d = %d outside [1, %d]", d, DQ_MAX_D);
    if (x_ld < d)
        return fail(DQ_ERR_INVALID_ARG, "x_ld = %lld < d = %d", (long long)x_ld, d);
    if (codes_ld < (d + 1) / 2)
        return fail(DQ_ERR_INVALID_ARG, "codes_ld = %lld < (d+1)/2 = %d", (long long)codes_ld, (d + 1) / 2);
    if (mode != DQ_MODE_GREEDY && mode != DQ_MODE_MINMAX)
        return fail(DQ_ERR_INVALID_ARG, "mode = %d is neither DQ_MODE_GREEDY nor DQ_MODE_MINMAX", mode);
    if (n_rows > 0 && (!x || !codes || !scale_bias))
        return fail(DQ_ERR_INVALID_ARG, "x, codes and scale_bias must be non-NULL when n_rows > 0");
    if (n_rows > 0 && ((reinterpret_cast<uintptr_t>(x) & 3) || (reinterpret_cast<uintptr_t>(scale_bias) & 1) ||
                       (reinterpret_cast<uintptr_t>(row_loss) & 3)))
        return fail(DQ_ERR_INVALID_ARG, "x and row_loss must be 4-byte and scale_bias 2-byte aligned");
    if (n_rows > ((int64_t)1 << 40))
        return fail(DQ_ERR_INVALID_ARG, "n_rows = %lld beyond 2^40", (long long)n_rows);
    if (n_rows == 0)
        return ok();
    int sms = 0;
    dq_status st = current_device(&sms);
    if (st != DQ_OK)
        return st;
    if (fault_injected())
        return fail(DQ_ERR_CUDA, "launch failure injected by DQ_FAULT_INJECT=launch");
    dq::QuantArgs a{x, n_rows, x_ld, d, codes, codes_ld, scale_bias, row_loss, best_ij, d_flags};
    return launched(dq::launch_quantize(a, mode, sms, (cudaStream_t)cuda_stream), "quantize");
}

dq_status dq_dequantize_rows(const uint8_t *codes, int64_t codes_ld, const uint16_t *scale_bias,
                             int64_t n_rows, int32_t d, float *out, int64_t out_ld, void *cuda_stream)
{
    if (n_rows < 0)
        return fail(DQ_ERR_INVALID_ARG, "n_rows = %lld < 0", (long long)n_rows);
    if (d < 1 || d > DQ_MAX_D)
        return fail(DQ_ERR_INVALID_ARG, "d = %d outside [1, %d]", d, DQ_MAX_D);
    if (codes_ld < (d + 1) / 2)
        return fail(DQ_ERR_INVALID_ARG, "codes_ld = %lld < (d+1)/2 = %d", (long long)codes_ld, (d + 1) / 2);
    if (out_ld < d)
        return fail(DQ_ERR_INVALID_ARG, "out_ld = %lld < d = %d", (long long)out_ld, d);
    if (n_rows > 0 && (!codes || !scale_bias || !out))
        return fail(DQ_ERR_INVALID_ARG, "codes, scale_bias and out must be non-NULL when n_rows > 0");
    if (n_rows > 0 && ((reinterpret_cast<uintptr_t>(scale_bias) & 1) || (reinterpret_cast<uintptr_t>(out) & 3)))
        return fail(DQ_ERR_INVALID_ARG, "scale_bias must be 2-byte and out 4-byte aligned");
    if (n_rows == 0)
        return ok();
    int sms = 0;
    dq_status st = current_device(&sms);
    if (st != DQ_OK)
        return st;
    if (fault_injected())
        return fail(DQ_ERR_CUDA, "launch failure injected by DQ_FAULT_INJECT=launch");
    dq::DequantArgs a{codes, codes_ld, scale_bias, n_rows, d, out, out_ld};
    return launched(dq::launch_dequantize(a, sms, (cudaStream_t)cuda_stream), "dequantize");
}

namespace {

// Element alignment of a typed array (a misaligned one would fault in the kernels).
bool misaligned(const void *p, uintptr_t bytes) { return (reinterpret_cast<uintptr_t>(p) & (bytes - 1)) != 0; }

// Checks and copies the lookup's tables (column block t of each output row by default).
dq_status bag_tables(const dq_table *tables, int32_t n_tables, int32_t d, int32_t batch, dq::BagTables &tabs)
{
    if (n_tables < 1 || n_tables > DQ_MAX_TABLES)
        return fail(DQ_ERR_INVALID_ARG, "n_tables = %d outside [1, %d]", n_tables, DQ_MAX_TABLES);
    if (!tables)
        return fail(DQ_ERR_INVALID_ARG, "tables must be non-NULL");
    if (d < 1 || d > DQ_MAX_D)
        return fail(DQ_ERR_INVALID_ARG, "d = %d outside [1, %d]", d, DQ_MAX_D);
    if (batch < 0)
        return fail(DQ_ERR_INVALID_ARG, "batch = %d < 0", batch);
    if ((int64_t)n_tables * batch + 1 > INT32_MAX)
        return fail(DQ_ERR_INVALID_ARG, "n_tables * batch + 1 offsets exceed int32 indexing");
    memset(&tabs, 0, sizeof tabs);
    for (int t = 0; t < n_tables; ++t) {
        const dq_table &tb = tables[t];
        if (tb.n_rows < 0)
            return fail(DQ_ERR_INVALID_ARG, "tables[%d].n_rows = %lld < 0", t, (long long)tb.n_rows);
        if (tb.codes_ld < (d + 1) / 2 || tb.codes_ld > INT32_MAX)
            return fail(DQ_ERR_INVALID_ARG, "tables[%d].codes_ld = %lld outside [(d+1)/2 = %d, 2^31)", t,
                        (long long)tb.codes_ld, (d + 1) / 2);
        if (tb.n_rows > 0 && (!tb.codes || !tb.scale_bias))
            return fail(DQ_ERR_INVALID_ARG, "tables[%d]: codes and scale_bias must be non-NULL", t);
        if (tb.n_rows > 0 && misaligned(tb.scale_bias, 2))
            return fail(DQ_ERR_INVALID_ARG, "tables[%d]: scale_bias must be 2-byte aligned", t);
        tabs.codes[t] = tb.codes;
        tabs.scale_bias[t] = tb.scale_bias;
        tabs.n_rows[t] = tb.n_rows;
        tabs.codes_ld[t] = tb.codes_ld;
        tabs.slot[t] = t;
    }
    return DQ_OK;
}

dq_status bag_launch(const dq::BagTables &tabs, const dq::BagArgs &a, const dq::BagDest &dst, void *cuda_stream)
{
    int sms = 0;
    dq_status st = current_device(&sms);
    if (st != DQ_OK)
        return st;
    if (fault_injected())
        return fail(DQ_ERR_CUDA, "launch failure injected by DQ_FAULT_INJECT=launch");
    return launched(dq::launch_embbag(tabs, a, dst, sms, (cudaStream_t)cuda_stream), "embbag");
}

} // namespace

dq_status dq_embbag_int4_fwd(const dq_table *tables, int32_t n_tables, int32_t d, const int32_t *indices,
                             const int32_t *offsets, int32_t batch, float *out, uint32_t *d_flags,
                             void *cuda_stream)
{
    dq::BagTables tabs;
    dq_status st = bag_tables(tables, n_tables, d, batch, tabs);
    if (st != DQ_OK)
        return st;
    if (batch > 0 && (!indices || !offsets || !out))
        return fail(DQ_ERR_INVALID_ARG, "indices, offsets and out must be non-NULL when batch > 0");
    if (batch > 0 && (misaligned(indices, 4) || misaligned(offsets, 4) || misaligned(out, 4)))
        return fail(DQ_ERR_INVALID_ARG, "indices, offsets and out must be 4-byte aligned");
    if (batch == 0)
        return ok();
    dq::BagArgs a{};
    a.T = n_tables;
    a.d = d;
    a.batch = batch;
    a.indices = indices;
    a.offsets = offsets;
    a.out = out;
    a.flags = d_flags;
    a.div = dq::make_batch_div((uint32_t)batch);
    dq::BagDest dst{};   // n = 0: rows into out
    return bag_launch(tabs, a, dst, cuda_stream);
}

dq_status dq_embbag_int4_fwd_to_owners(const dq_table *tables, int32_t n_tables, int32_t d,
                                       const int32_t *indices, const int32_t *offsets, int32_t batch,
                                       const int32_t *table_slot, int32_t t_out, float *const *dest,
                                       int32_t n_dest, uint32_t *d_flags, void *cuda_stream)
{
    dq::BagTables tabs;
    dq_status st = bag_tables(tables, n_tables, d, batch, tabs);
    if (st != DQ_OK)
        return st;
    if (n_dest < 1 || n_dest > DQ_MAX_DEST)
        return fail(DQ_ERR_INVALID_ARG, "n_dest = %d outside [1, %d]", n_dest, DQ_MAX_DEST);
    if (batch % n_dest != 0)
        return fail(DQ_ERR_INVALID_ARG, "batch = %d is not a multiple of n_dest = %d", batch, n_dest);
    if (t_out < n_tables || (int64_t)t_out > (int64_t)DQ_MAX_TABLES * DQ_MAX_DEST)
        return fail(DQ_ERR_INVALID_ARG, "t_out = %d outside [n_tables = %d, %d]", t_out, n_tables,
                    DQ_MAX_TABLES * DQ_MAX_DEST);
    if (!table_slot || !dest)
        return fail(DQ_ERR_INVALID_ARG, "table_slot and dest must be non-NULL");
    for (int t = 0; t < n_tables; ++t) {
        if (table_slot[t] < 0 || table_slot[t] >= t_out)
            return fail(DQ_ERR_INVALID_ARG, "table_slot[%d] = %d outside [0, %d)", t, table_slot[t], t_out);
        for (int u = 0; u < t; ++u)
            if (table_slot[u] == table_slot[t])
                return fail(DQ_ERR_INVALID_ARG, "table_slot[%d] and table_slot[%d] are both %d", u, t,
                            table_slot[t]);
        tabs.slot[t] = table_slot[t];
    }
    if ((int64_t)(batch / n_dest) * t_out * d > ((int64_t)1 << 40))
        return fail(DQ_ERR_INVALID_ARG, "the destination buffers exceed 2^40 elements");
    if (batch > 0 && (!indices || !offsets))
        return fail(DQ_ERR_INVALID_ARG, "indices and offsets must be non-NULL when batch > 0");
    if (batch > 0 && (misaligned(indices, 4) || misaligned(offsets, 4)))
        return fail(DQ_ERR_INVALID_ARG, "indices and offsets must be 4-byte aligned");
    dq::BagDest dst{};
    for (int r = 0; r < n_dest; ++r) {
        if (batch > 0 && !dest[r])
            return fail(DQ_ERR_INVALID_ARG, "dest[%d] must be non-NULL", r);
        if (batch > 0 && misaligned(dest[r], 4))
            return fail(DQ_ERR_INVALID_ARG, "dest[%d] must be 4-byte aligned", r);
        dst.ptr[r] = dest[r];
    }
    if (batch == 0)
        return ok();
    dq::BagArgs a{};
    a.T = n_tables;
    a.d = d;
    a.batch = batch;
    a.indices = indices;
    a.offsets = offsets;
    a.out = dest[0];   // not written: every row goes through dst
    a.flags = d_flags;
    a.div = dq::make_batch_div((uint32_t)batch);
    dst.n = n_dest;
    dst.bl = batch / n_dest;
    dst.t_out = t_out;
    dst.div = dq::make_batch_div((uint32_t)dst.bl);
    return bag_launch(tabs, a, dst, cuda_stream);
}

dq_status dq_row_l2_error(const float *x, int64_t n_rows, int32_t d, int64_t x_ld, const uint8_t *codes,
                          int64_t codes_ld, const uint16_t *scale_bias, double *row_err, double *err_sum,
                          void *cuda_stream)
{
    if (n_rows < 0)
        return fail(DQ_ERR_INVALID_ARG, "n_rows = %lld < 0", (long long)n_rows);
    if (d < 1 || d > DQ_MAX_D)
        return fail(DQ_ERR_INVALID_ARG, "d = %d outside [1, %d]", d, DQ_MAX_D);
    if (x_ld < d)
        return fail(DQ_ERR_INVALID_ARG, "x_ld = %lld < d = %d", (long long)x_ld, d);
    if (codes_ld < (d + 1) / 2)
        return fail(DQ_ERR_INVALID_ARG, "codes_ld = %lld < (d+1)/2 = %d", (long long)codes_ld, (d + 1) / 2);
    if (n_rows > 0 && (!x || !codes || !scale_bias))
        return fail(DQ_ERR_INVALID_ARG, "x, codes and scale_bias must be non-NULL when n_rows > 0");
    if (n_rows > 0 && (reinterpret_cast<uintptr_t>(scale_bias) & 3) != 0)
        return fail(DQ_ERR_INVALID_ARG, "scale_bias must be 4-byte aligned");
    if (n_rows == 0)
        return ok();
    int sms = 0;
    dq_status st = current_device(&sms);
    if (st != DQ_OK)
        return st;
    if (fault_injected())
        return fail(DQ_ERR_CUDA, "launch failure injected by DQ_FAULT_INJECT=launch");
    dq::L2Args a{x, n_rows, x_ld, d, codes, codes_ld, scale_bias, row_err, err_sum};
    return launched(dq::launch_row_l2(a, sms, (cudaStream_t)cuda_stream), "row_l2_error");
}

dq_status dq_quantize_rows_kmeans4(const float *x, int64_t n_rows, int32_t d, int64_t x_ld, uint8_t *codes,
                                   int64_t codes_ld, uint16_t *codebook, float *row_loss, int32_t *row_iters,
                                   int32_t iters, uint32_t *d_flags, void *cuda_stream)
{
    if (n_rows < 0)
        return fail(DQ_ERR_INVALID_ARG, "n_rows = %lld < 0", (long long)n_rows);
    if (d < 1 || d > DQ_MAX_D)
        return fail(DQ_ERR_INVALID_ARG, "d = %d outside [1, %d]", d, DQ_MAX_D);
    if (x_ld < d)
        return fail(DQ_ERR_INVALID_ARG, "x_ld = %lld < d = %d", (long long)x_ld, d);
    if (codes_ld < (d + 1) / 2)
        return fail(DQ_ERR_INVALID_ARG, "codes_ld = %lld < (d+1)/2 = %d", (long long)codes_ld, (d + 1) / 2);
    if (iters < 0 || iters > DQ_KMEANS_MAX_ITERS)
        return fail(DQ_ERR_INVALID_ARG, "iters = %d outside [0, %d]", iters, DQ_KMEANS_MAX_ITERS);
    if (n_rows > 0 && (!x || !codes || !codebook))
        return fail(DQ_ERR_INVALID_ARG, "x, codes and codebook must be non-NULL when n_rows > 0");
    if (n_rows > 0 && ((reinterpret_cast<uintptr_t>(x) & 3) || (reinterpret_cast<uintptr_t>(codebook) & 1) ||
                       (reinterpret_cast<uintptr_t>(row_loss) & 3) || (reinterpret_cast<uintptr_t>(row_iters) & 3)))
        return fail(DQ_ERR_INVALID_ARG, "x, row_loss and row_iters must be 4-byte and codebook 2-byte aligned");
    if (n_rows == 0)
        return ok();
    int sms = 0;
    dq_status st = current_device(&sms);
    if (st != DQ_OK)
        return st;
    if (fault_injected())
        return fail(DQ_ERR_CUDA, "launch failure injected by DQ_FAULT_INJECT=launch");
    dq::KmeansArgs a{x, n_rows, x_ld, d, iters, codes, codes_ld, codebook, row_loss, row_iters, d_flags};
    return launched(dq::launch_kmeans(a, (cudaStream_t)cuda_stream), "quantize_rows_kmeans4");
}

dq_status dq_dequantize_rows_kmeans4(const uint8_t *codes, int64_t codes_ld, const uint16_t *codebook,
                                     int64_t n_rows, int32_t d, float *out, int64_t out_ld, void *cuda_stream)
{
    if (n_rows < 0)
        return fail(DQ_ERR_INVALID_ARG, "n_rows = %lld < 0", (long long)n_rows);
    if (d < 1 || d > DQ_MAX_D)
        return fail(DQ_ERR_INVALID_ARG, "d = %d outside [1, %d]", d, DQ_MAX_D);
    if (codes_ld < (d + 1) / 2)
        return fail(DQ_ERR_INVALID_ARG, "codes_ld = %lld < (d+1)/2 = %d", (long long)codes_ld, (d + 1) / 2);
    if (out_ld < d)
        return fail(DQ_ERR_INVALID_ARG, "out_ld = %lld < d = %d", (long long)out_ld, d);
    if (n_rows > 0 && (!codes || !codebook || !out))
        return fail(DQ_ERR_INVALID_ARG, "codes, codebook and out must be non-NULL when n_rows > 0");
    if (n_rows > 0 && ((reinterpret_cast<uintptr_t>(codebook) & 1) || (reinterpret_cast<uintptr_t>(out) & 3)))
        return fail(DQ_ERR_INVALID_ARG, "codebook must be 2-byte and out 4-byte aligned");
    if (n_rows == 0)
        return ok();
    int sms = 0;
    dq_status st = current_device(&sms);
    if (st != DQ_OK)
        return st;
    if (fault_injected())
        return fail(DQ_ERR_CUDA, "launch failure injected by DQ_FAULT_INJECT=launch");
    dq::KmeansDequantArgs a{codes, codes_ld, codebook, n_rows, d, out, out_ld};
    return launched(dq::launch_kmeans_dequantize(a, sms, (cudaStream_t)cuda_stream), "dequantize_rows_kmeans4");
}

dq_status dq_embbag_kmeans4_fwd(const dq_kmeans_table *tables, int32_t n_tables, int32_t d, const int32_t *indices,
                                const int32_t *offsets, int32_t batch, float *out, uint32_t *d_flags,
                                void *cuda_stream)
{
    if (n_tables < 1 || n_tables > DQ_MAX_TABLES)
        return fail(DQ_ERR_INVALID_ARG, "n_tables = %d outside [1, %d]", n_tables, DQ_MAX_TABLES);
    if (!tables)
        return fail(DQ_ERR_INVALID_ARG, "tables must be non-NULL");
    if (d < 1 || d > DQ_MAX_D)
        return fail(DQ_ERR_INVALID_ARG, "d = %d outside [1, %d]", d, DQ_MAX_D);
    if (batch < 0)
        return fail(DQ_ERR_INVALID_ARG, "batch = %d < 0", batch);
    if ((int64_t)n_tables * batch + 1 > INT32_MAX)
        return fail(DQ_ERR_INVALID_ARG, "n_tables * batch + 1 offsets exceed int32 indexing");
    dq::KmeansBagTables tabs;
    memset(&tabs, 0, sizeof tabs);
    for (int t = 0; t < n_tables; ++t) {
        const dq_kmeans_table &tb = tables[t];
        if (tb.n_rows < 0)
            return fail(DQ_ERR_INVALID_ARG, "tables[%d].n_rows = %lld < 0", t, (long long)tb.n_rows);
        if (tb.codes_ld < (d + 1) / 2)
            return fail(DQ_ERR_INVALID_ARG, "tables[%d].codes_ld = %lld < (d+1)/2 = %d", t,
                        (long long)tb.codes_ld, (d + 1) / 2);
        if (tb.n_rows > 0 && (!tb.codes || !tb.codebook))
            return fail(DQ_ERR_INVALID_ARG, "tables[%d]: codes and codebook must be non-NULL", t);
        if (tb.n_rows > 0 && misaligned(tb.codebook, 2))
            return fail(DQ_ERR_INVALID_ARG, "tables[%d]: codebook must be 2-byte aligned", t);
        tabs.codes[t] = tb.codes;
        tabs.codebook[t] = tb.codebook;
        tabs.n_rows[t] = tb.n_rows;
        tabs.codes_ld[t] = tb.codes_ld;
    }
    if (batch > 0 && (!indices || !offsets || !out))
        return fail(DQ_ERR_INVALID_ARG, "indices, offsets and out must be non-NULL when batch > 0");
    if (batch > 0 && (misaligned(indices, 4) || misaligned(offsets, 4) || misaligned(out, 4)))
        return fail(DQ_ERR_INVALID_ARG, "indices, offsets and out must be 4-byte aligned");
    if (batch == 0)
        return ok();
    int sms = 0;
    dq_status st = current_device(&sms);
    if (st != DQ_OK)
        return st;
    if (fault_injected())
        return fail(DQ_ERR_CUDA, "launch failure injected by DQ_FAULT_INJECT=launch");
    dq::KmeansBagArgs a{n_tables, d, batch, indices, offsets, out, d_flags, dq::make_batch_div((uint32_t)batch)};
    return launched(dq::launch_kmeans_bag(tabs, a, sms, (cudaStream_t)cuda_stream), "embbag_kmeans4");
}

size_t dq_embbag_int4_bwd_workspace_bytes(int32_t d, int64_t n_indices)
{
    if (d < 1 || d > DQ_MAX_D || n_indices < 0 || n_indices > INT32_MAX)
        return 0;
    return dq::bwd_layout(n_indices, d).total;
}

dq_status dq_embbag_int4_bwd_sgd(const dq_master_table *tables, int32_t n_tables, int32_t d,
                                 const int32_t *indices, const int32_t *offsets, int32_t batch, int64_t n_indices,
                                 const float *grad_out, float lr, int32_t mode, void *workspace,
                                 size_t workspace_bytes, uint32_t *d_flags, void *cuda_stream)
{
    if (n_tables < 1 || n_tables > DQ_MAX_TABLES)
        return fail(DQ_ERR_INVALID_ARG, "n_tables = %d outside [1, %d]", n_tables, DQ_MAX_TABLES);
    if (!tables)
        return fail(DQ_ERR_INVALID_ARG, "tables must be non-NULL");
    if (d < 1 || d > DQ_MAX_D)
        return fail(DQ_ERR_INVALID_ARG, "d = %d outside [1, %d]", d, DQ_MAX_D);
    if (batch < 0)
        return fail(DQ_ERR_INVALID_ARG, "batch = %d < 0", batch);
    if ((int64_t)n_tables * batch + 1 > INT32_MAX)
        return fail(DQ_ERR_INVALID_ARG, "n_tables * batch + 1 offsets exceed int32 indexing");
    if (n_indices < 0 || n_indices > INT32_MAX)
        return fail(DQ_ERR_INVALID_ARG, "n_indices = %lld outside [0, 2^31)", (long long)n_indices);
    if (batch == 0 && n_indices != 0)
        return fail(DQ_ERR_INVALID_ARG, "n_indices = %lld with batch = 0", (long long)n_indices);
    if (mode != DQ_MODE_GREEDY && mode != DQ_MODE_MINMAX)
        return fail(DQ_ERR_INVALID_ARG, "mode = %d is neither DQ_MODE_GREEDY nor DQ_MODE_MINMAX", mode);
    if (!(lr - lr == 0.0f))
        return fail(DQ_ERR_INVALID_ARG, "lr is not finite");
    dq::RequantArgs r;
    memset(&r, 0, sizeof r);
    int64_t total = 0;
    for (int t = 0; t < n_tables; ++t) {
        const dq_master_table &tb = tables[t];
        if (tb.n_rows < 0)
            return fail(DQ_ERR_INVALID_ARG, "tables[%d].n_rows = %lld < 0", t, (long long)tb.n_rows);
        if (tb.master_ld < d)
            return fail(DQ_ERR_INVALID_ARG, "tables[%d].master_ld = %lld < d = %d", t, (long long)tb.master_ld, d);
        if (tb.codes_ld < (d + 1) / 2)
            return fail(DQ_ERR_INVALID_ARG, "tables[%d].codes_ld = %lld < (d+1)/2 = %d", t,
                        (long long)tb.codes_ld, (d + 1) / 2);
        if (tb.n_rows > 0 && (!tb.master || !tb.codes || !tb.scale_bias))
            return fail(DQ_ERR_INVALID_ARG, "tables[%d]: master, codes and scale_bias must be non-NULL", t);
        if ((reinterpret_cast<uintptr_t>(tb.master) & 3) || (reinterpret_cast<uintptr_t>(tb.scale_bias) & 1))
            return fail(DQ_ERR_INVALID_ARG, "tables[%d]: master must be 4-byte and scale_bias 2-byte aligned", t);
        r.tabs.master[t] = tb.master;
        r.tabs.master_ld[t] = tb.master_ld;
        r.tabs.codes[t] = tb.codes;
        r.tabs.codes_ld[t] = tb.codes_ld;
        r.tabs.scale_bias[t] = tb.scale_bias;
        r.tabs.key_base[t] = (uint32_t)total;
        total += tb.n_rows;
        if (total > (int64_t)UINT32_MAX - 1)
            return fail(DQ_ERR_INVALID_ARG, "the tables hold more than 2^32 - 2 rows in all");
    }
    r.tabs.key_base[n_tables] = (uint32_t)total;
    if (n_indices == 0)
        return ok();
    if (!indices || !offsets || !grad_out)
        return fail(DQ_ERR_INVALID_ARG, "indices, offsets and grad_out must be non-NULL when n_indices > 0");
    if (reinterpret_cast<uintptr_t>(grad_out) & 3)
        return fail(DQ_ERR_INVALID_ARG, "grad_out must be 4-byte aligned");
    const dq::BwdLayout L = dq::bwd_layout(n_indices, d);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(DQ_ERR_INVALID_ARG, "workspace must be a non-NULL, 256-byte aligned device buffer");
    if (workspace_bytes < L.total)
        return fail(DQ_ERR_INVALID_ARG, "workspace_bytes = %zu < %zu needed (dq_embbag_int4_bwd_workspace_bytes)",
                    workspace_bytes, L.total);
    int sms = 0;
    dq_status st = current_device(&sms);
    if (st != DQ_OK)
        return st;
    if (fault_injected())
        return fail(DQ_ERR_CUDA, "launch failure injected by DQ_FAULT_INJECT=launch");
    char *ws = static_cast<char *>(workspace);
    dq::BwdArgs a;
    memset(&a, 0, sizeof a);
    a.T = n_tables;
    a.d = d;
    a.batch = batch;
    a.n = n_indices;
    a.indices = indices;
    a.offsets = offsets;
    a.grad = grad_out;
    memcpy(a.key_base, r.tabs.key_base, sizeof a.key_base);
    a.div = dq::make_batch_div((uint32_t)batch);
    a.hdr = reinterpret_cast<uint32_t *>(ws + L.hdr);
    a.keys[0] = reinterpret_cast<uint32_t *>(ws + L.keys0);
    a.keys[1] = reinterpret_cast<uint32_t *>(ws + L.keys1);
    a.bags[0] = reinterpret_cast<int32_t *>(ws + L.bags0);
    a.bags[1] = reinterpret_cast<int32_t *>(ws + L.bags1);
    a.hist = reinterpret_cast<uint32_t *>(ws + L.hist);
    a.totals = reinterpret_cast<uint32_t *>(ws + L.totals);
    a.partials = reinterpret_cast<double *>(ws + L.partials);
    a.span_slot = reinterpret_cast<uint32_t *>(ws + L.span_slot);
    a.list = reinterpret_cast<uint32_t *>(ws + L.list);
    a.grad_rows = reinterpret_cast<float *>(ws + L.grad_rows);
    a.grad_ld = L.grad_ld;
    a.flags = d_flags;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    cudaError_t e = cudaMemsetAsync(a.hdr, 0, 256, stream);
    if (e != cudaSuccess)
        return fail(DQ_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    e = dq::launch_bwd_sort_reduce(a, sms, stream);
    if (e != cudaSuccess)
        return launched(e, "embbag backward");
    r.n_tables = n_tables;
    r.d = d;
    r.list = a.list;
    r.count = a.hdr + 1;
    r.bad = a.hdr;
    r.grad_rows = a.grad_rows;
    r.grad_ld = a.grad_ld;
    r.lr = lr;
    r.flags = d_flags;
    const int64_t max_rows = n_indices < total ? n_indices : total;
    return launched(dq::launch_requant(r, max_rows, mode, sms, stream), "embbag backward re-quantization");
}

const char *dq_status_string(dq_status s)
{
    switch (s) {
    case DQ_OK: return "DQ_OK";
    case DQ_ERR_INVALID_ARG: return "DQ_ERR_INVALID_ARG: invalid argument";
    case DQ_ERR_UNSUPPORTED: return "DQ_ERR_UNSUPPORTED: unsupported device or request";
    case DQ_ERR_CUDA: return "DQ_ERR_CUDA: CUDA error";
    }
    return "unknown dq_status";
}

const char *dq_last_error(void)
{
    return g_last_error.c_str();
}

int32_t dq_version(void)
{
    return 10000;
}

} // extern "C"
