/*
 * dq.h -- C ABI of libdq: row-wise INT4 quantization of embedding tables and the
 * sum-pooled INT4 embedding bag, as hand-written CUDA kernels for sm_100a (B200).
 *
 * The method: "Post-Training 4-bit Quantization on Embedding Tables" (Guan et al.,
 * 2019), review page, section 提出的方法 (proposed method): each embedding row gets
 * its own uniform 4-bit quantizer (bullet 1), with the clipping thresholds chosen
 * by a greedy search that walks toward a local minimum of the squared error, and
 * the scale and bias stored as FP16 (bullet 2; section 主要发现 / main findings,
 * bullet 4: 13.28% of the FP32 size at d=128). The lookup: "Deep Learning
 * Recommendation Model for Personalization and Recommendation Systems", section
 * 提出的方法 (proposed method), bullet 1 (sparse ids mapped to dense vectors by
 * embedding tables), summed over each bag of ids.
 *
 * Packed row format (shared by all entry points):
 *   codes       d 4-bit codes, two per byte: byte m = q[2m] | q[2m+1] << 4; for odd d
 *               the last byte's high nibble is 0. Row r starts at codes + r*codes_ld.
 *   scale_bias  [n_rows][2] binary16 bit patterns {scale, bias}; element k of row r
 *               decodes as fma(q_k, scale, bias) in binary32 (one rounding).
 *
 * Quantization of one row x[0..d-1] (binary32 throughout, round to nearest even):
 *   xmin, xmax, R = xmax - xmin, step = R / 200; grid points lo(i) = fma(i, step, xmin),
 *   hi(j) = fma(-j, step, xmax). L(lo, hi) is the squared reconstruction error with
 *   s = (hi - lo) / 15, q = clamp(rint((x - lo) / s), 0, 15), xhat = fma(q, s, lo),
 *   summed pairwise (recursive halving, padded with zeros to a power of two).
 *   Starting from (0, 0), each of 168 moves (while the width exceeds 0.16 * R) tries
 *   (i+1, j) and (i, j+1), moves to the lower loss (to (i+1, j) on a tie), and keeps
 *   the first lowest loss seen. Then scale = fp16((hi* - lo*) / 15), bias = fp16(lo*),
 *   q = clamp(rint((x - bias) / scale), 0, 15) with IEEE division (q = 0 when scale
 *   is 0). DQ_MODE_MINMAX skips the moves (the plain min/max quantizer).
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers (except `tables`, a host array). The
 *     caller owns every buffer; the library allocates no memory and keeps no
 *     state besides cached device attributes (and, for
 *     dq_embbag_int4_bwd_sgd_noalloc, its static device scratch array).
 *   - Calls are asynchronous and stream-ordered on `cuda_stream` (a cudaStream_t;
 *     NULL = the legacy default stream). Outputs are valid after the stream is
 *     synchronized. Calls may be made from several host threads.
 *   - Arguments are validated on the host before anything is enqueued:
 *     DQ_ERR_INVALID_ARG, nothing launched. A failed launch returns DQ_ERR_CUDA.
 *     dq_last_error() gives the calling thread's last detailed message.
 *   - Typed arrays must be aligned to their element size: binary16 arrays
 *     (scale_bias, codebook) to 2 bytes, int32 and binary32 arrays (indices,
 *     offsets, x, out, dest, grad_out, row_loss) to 4 bytes; a misaligned one is
 *     rejected with DQ_ERR_INVALID_ARG. Byte arrays (codes) have no rule; aligned
 *     code rows (16-byte rows and codes_ld) take the vectorised kernels.
 *   - n_rows == 0 or batch == 0 is a no-op returning DQ_OK.
 *   - Data errors are preconditions and are never trapped on the device. When
 *     `d_flags` (a device uint32) is non-NULL the kernels OR DQ_FLAG_* bits into
 *     it; read it after synchronizing. Out-of-range ids and decreasing offsets
 *     are always skipped (contribute nothing), flagged or not.
 */
#ifndef DQ_H
#define DQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dq_status {
    DQ_OK = 0,
    DQ_ERR_INVALID_ARG = 1,  /* bad pointer, size, stride, mode or limit; nothing launched */
    DQ_ERR_UNSUPPORTED = 2,  /* no sm_100-class device or no kernel for the request */
    DQ_ERR_CUDA = 3          /* a CUDA runtime call or launch failed; see dq_last_error() */
} dq_status;

enum { DQ_MODE_GREEDY = 0, DQ_MODE_MINMAX = 1 };

enum {
    DQ_FLAG_BAD_INDEX = 1u,      /* an id < 0 or >= the table's n_rows was skipped */
    DQ_FLAG_BAD_OFFSETS = 2u,    /* a bag with offsets[g+1] < offsets[g] was treated as empty */
    DQ_FLAG_NONFINITE = 4u,      /* an input row held a NaN or an infinity */
    DQ_FLAG_FP16_OVERFLOW = 8u   /* a row's scale or bias overflowed binary16 */
};

#define DQ_MAX_D 1024
#define DQ_MAX_TABLES 64
#define DQ_MAX_DEST 64

/* One packed table for the embedding bag. codes and scale_bias are device
 * pointers in the packed row format above. */
typedef struct dq_table {
    const uint8_t *codes;
    const uint16_t *scale_bias;
    int64_t n_rows;
    int64_t codes_ld;   /* bytes between rows, in [(d + 1) / 2, 2^31) */
} dq_table;

/*
 * dq_quantize_rows_int4 -- greedy (or min/max) row-wise INT4 quantization.
 * ("Post-Training 4-bit Quantization on Embedding Tables", 提出的方法 / proposed
 * method, bullets 1-2.)
 *
 *   x           [n_rows][x_ld] binary32, row-major; the first d of each row are used
 *   n_rows      >= 0
 *   d           1..DQ_MAX_D
 *   x_ld        >= d, in elements
 *   codes       [n_rows][codes_ld] bytes (output); only the first (d+1)/2 of a row are written
 *   codes_ld    >= (d + 1) / 2, in bytes
 *   scale_bias  [n_rows][2] binary16 bit patterns (output)
 *   row_loss    [n_rows] binary32 (output, nullable): the search loss L at the chosen pair
 *   best_ij     [n_rows][2] uint8 (output, nullable): the chosen grid indices (i*, j*)
 *   mode        DQ_MODE_GREEDY or DQ_MODE_MINMAX
 *   d_flags     device uint32 (nullable): DQ_FLAG_NONFINITE, DQ_FLAG_FP16_OVERFLOW
 *   cuda_stream cudaStream_t
 *
 * Rows with non-finite values or with a scale/bias beyond binary16's range give
 * unspecified (but memory-safe) results.
 */
dq_status dq_quantize_rows_int4(const float *x, int64_t n_rows, int32_t d, int64_t x_ld,
                                uint8_t *codes, int64_t codes_ld, uint16_t *scale_bias,
                                float *row_loss, uint8_t *best_ij, int32_t mode,
                                uint32_t *d_flags, void *cuda_stream);

/*
 * dq_dequantize_rows -- out[r][k] = fma(q_k, scale, bias) in binary32.
 * ("Post-Training 4-bit Quantization on Embedding Tables", 提出的方法 / proposed
 * method, bullet 2: the FP16 scale and bias decode each row.)
 *
 *   codes, codes_ld, scale_bias   packed rows as above (inputs)
 *   n_rows >= 0, d in 1..DQ_MAX_D
 *   out         [n_rows][out_ld] binary32 (output), out_ld >= d elements
 */
dq_status dq_dequantize_rows(const uint8_t *codes, int64_t codes_ld, const uint16_t *scale_bias,
                             int64_t n_rows, int32_t d, float *out, int64_t out_ld,
                             void *cuda_stream);

/*
 * dq_embbag_int4_fwd -- sum-pooled lookup over n_tables packed tables sharing d.
 * ("Deep Learning Recommendation Model for Personalization and Recommendation
 * Systems", 提出的方法 / proposed method, bullet 1.)
 *
 *   tables      HOST array of n_tables dq_table (1..DQ_MAX_TABLES); its contents are
 *               copied at the call, the array may be reused on return
 *   d           1..DQ_MAX_D
 *   indices     int32 ids, table-relative
 *   offsets     int32 [n_tables*batch + 1], table-major: bag (t, b) is
 *               indices[offsets[t*batch + b] .. offsets[t*batch + b + 1]); indices
 *               holds offsets[n_tables*batch] ids. A bag whose offsets decrease or
 *               leave [0, offsets[n_tables*batch]] is clamped into that range (empty
 *               if they decrease) and flagged DQ_FLAG_BAD_OFFSETS
 *   batch       >= 0
 *   out         [batch][n_tables*d] binary32 (output): out[b][t*d + k] is the binary32
 *               sum over the bag of fma(q_k, scale, bias); an empty bag gives +0
 *   d_flags     device uint32 (nullable): DQ_FLAG_BAD_INDEX, DQ_FLAG_BAD_OFFSETS
 *
 * The sum is accumulated in binary32, and a bag of one id returns that row's
 * dequantized values exactly. The order of the additions is not specified: when the
 * bags average 4 ids or more, interleaved partial sums over the bag's ids are added
 * together at the end. Each output element stays within a few binary32 roundings per
 * id of the exact sum.
 */
dq_status dq_embbag_int4_fwd(const dq_table *tables, int32_t n_tables, int32_t d,
                             const int32_t *indices, const int32_t *offsets, int32_t batch,
                             float *out, uint32_t *d_flags, void *cuda_stream);

/*
 * dq_embbag_int4_fwd_to_owners -- the same lookup, each pooled row stored straight into
 * the buffer of the rank that owns its sample, at its place among all ranks' tables:
 * the lookup and the exchange of table-wise sharding in one kernel ("Deep Learning
 * Recommendation Model for Personalization and Recommendation Systems", 提出的方法 /
 * proposed method: embedding tables model-parallel, the pooled embeddings sent to the
 * data-parallel ranks; there the exchange is an all-to-all, here each rank writes its
 * rows into the owners' memory).
 *
 *   tables ... batch, d_flags   as dq_embbag_int4_fwd (batch: the global batch)
 *   table_slot  HOST int32 [n_tables]: the column block of each local table among the
 *               t_out tables of the output rows; distinct, in [0, t_out)
 *   t_out       tables in an output row (all ranks' tables), n_tables..DQ_MAX_TABLES*DQ_MAX_DEST
 *   dest        HOST array of n_dest device pointers (1..DQ_MAX_DEST, copied at the call):
 *               dest[r] is rank r's buffer [batch / n_dest][t_out*d] binary32, which may be
 *               another GPU's memory mapped into this process (peer access enabled)
 *   n_dest      ranks; batch must be a multiple of n_dest
 *
 * Bag (t, b) is stored at dest[b / bl][(b % bl) * t_out * d + table_slot[t] * d + k],
 * bl = batch / n_dest, with the values dq_embbag_int4_fwd would give. Nothing else is
 * written; the caller orders the ranks' calls against the reads of their buffers
 * (a barrier after the calls, and one before the next call writes again).
 * Errors: DQ_ERR_INVALID_ARG for the argument checks above (nothing launched).
 */
dq_status dq_embbag_int4_fwd_to_owners(const dq_table *tables, int32_t n_tables, int32_t d,
                                       const int32_t *indices, const int32_t *offsets, int32_t batch,
                                       const int32_t *table_slot, int32_t t_out, float *const *dest,
                                       int32_t n_dest, uint32_t *d_flags, void *cuda_stream);

/*
 * dq_row_l2_error -- normalized l2 error of packed rows against their binary32
 * originals: row_err[r] = sqrt(sum_k (x[r][k] - xhat_k)^2) / sqrt(sum_k x[r][k]^2),
 * xhat_k = fma(q_k, scale, bias), both sums in binary64 (a row with sum x^2 = 0 gives
 * 0 if reconstructed exactly, else +inf). ("Post-Training 4-bit Quantization on
 * Embedding Tables", 提出的方法 / proposed method, bullet 5: quantization error as
 * normalized l2 loss; 主要发现 / main findings, bullet 2.)
 *
 *   x, n_rows, d, x_ld            the binary32 rows, as for dq_quantize_rows_int4
 *   codes, codes_ld, scale_bias   their packed form (scale_bias 4-byte aligned)
 *   row_err     [n_rows] binary64 (output, nullable)
 *   err_sum     device binary64 scalar (nullable): the sum of the row errors is ADDED
 *               to it (atomically, in no fixed order); zero it before the call
 */
dq_status dq_row_l2_error(const float *x, int64_t n_rows, int32_t d, int64_t x_ld,
                          const uint8_t *codes, int64_t codes_ld, const uint16_t *scale_bias,
                          double *row_err, double *err_sum, void *cuda_stream);

/*
 * Codebook quantization (per-row k-means, 16 centroids): "Post-Training 4-bit
 * Quantization on Embedding Tables", 提出的方法 (proposed method), bullet 3 (codebook
 * quantization through k-means clustering, values mapped to a non-uniform set);
 * 主要发现 (main findings), bullet 3 (its sizes, 18.8%-37.5% of FP32, fit 16 binary16
 * centroids per row). Row format: the same d nibbles as above, and a codebook
 * [n_rows][16] of binary16 bit patterns; element k decodes as codebook[q_k].
 * The pages fix no algorithm details; this library computes, in binary32:
 *   1. c_j = fma(j, (xmax - xmin) / 15, xmin), j = 0..15.
 *   2. `iters` times: q_k = the j minimising |x_k - c_j| (ties to the lower j); for each
 *      j with members, c_j = their binary64 sum from +0 in index order / their count, the
 *      binary64 quotient rounded to binary32; a cluster without members keeps c_j.
 *   3. codebook_j = fp16(c_j); codes = the nearest stored centroid (ties to the lower j);
 *      row_loss = pairwise sum of (x_k - codebook[q_k])^2.
 */
#define DQ_KMEANS_MAX_ITERS 64

/* dq_quantize_rows_kmeans4 -- arguments as dq_quantize_rows_int4, with codebook
 * [n_rows][16] binary16 (output, 2-byte aligned), row_loss [n_rows] (nullable), iters in
 * [0, DQ_KMEANS_MAX_ITERS]; d_flags: DQ_FLAG_NONFINITE, DQ_FLAG_FP16_OVERFLOW.
 * Once an iteration's assignment q equals the previous iteration's, the centroids it
 * would compute are the current ones, so every later iteration repeats them: the
 * library stops there (the outputs are those of all `iters` iterations). row_iters
 * [n_rows] (int32, nullable, device): the centroid updates run for each row, at most
 * iters (rows processed together run until all of them have repeated). */
dq_status dq_quantize_rows_kmeans4(const float *x, int64_t n_rows, int32_t d, int64_t x_ld,
                                   uint8_t *codes, int64_t codes_ld, uint16_t *codebook,
                                   float *row_loss, int32_t *row_iters, int32_t iters,
                                   uint32_t *d_flags, void *cuda_stream);

/* dq_dequantize_rows_kmeans4 -- out[r][k] = codebook[r][q_k] (exact). */
dq_status dq_dequantize_rows_kmeans4(const uint8_t *codes, int64_t codes_ld,
                                     const uint16_t *codebook, int64_t n_rows, int32_t d,
                                     float *out, int64_t out_ld, void *cuda_stream);

/* One codebook-quantized table for the bag (device pointers). */
typedef struct dq_kmeans_table {
    const uint8_t *codes;
    const uint16_t *codebook;  /* [n_rows][16] binary16 */
    int64_t n_rows;
    int64_t codes_ld;          /* >= (d+1)/2 */
} dq_kmeans_table;

/* dq_embbag_kmeans4_fwd -- the sum-pooled lookup of dq_embbag_int4_fwd over codebook
 * tables: out[b][t*d + k] = binary32 sum, in id order, of codebook[id][q_k] over the
 * bag (a bag of one id returns the dequantized row exactly). Same arguments, skips,
 * clamping and flags as dq_embbag_int4_fwd. */
dq_status dq_embbag_kmeans4_fwd(const dq_kmeans_table *tables, int32_t n_tables, int32_t d,
                                const int32_t *indices, const int32_t *offsets, int32_t batch,
                                float *out, uint32_t *d_flags, void *cuda_stream);

/* One table of the bag backward: its binary32 master rows and their packed form.
 * All pointers are device pointers. */
typedef struct dq_master_table {
    float *master;          /* [n_rows][master_ld] binary32, 4-byte aligned; touched rows updated */
    int64_t master_ld;      /* >= d */
    uint8_t *codes;         /* packed rows (format above); touched rows rewritten */
    int64_t codes_ld;       /* >= (d+1)/2 */
    uint16_t *scale_bias;   /* [n_rows][2] binary16 patterns, 2-byte aligned; touched rows rewritten */
    int64_t n_rows;         /* >= 0; all tables together hold at most 2^32 - 2 rows */
} dq_master_table;

/*
 * dq_embbag_int4_bwd_workspace_bytes -- device workspace that dq_embbag_int4_bwd_sgd
 * needs for n_indices entries of width d (about 20 + 4.5 d bytes per entry); 0 for
 * arguments outside d in 1..DQ_MAX_D, n_indices in [0, 2^31).
 */
size_t dq_embbag_int4_bwd_workspace_bytes(int32_t d, int64_t n_indices);

/*
 * dq_embbag_int4_bwd_sgd -- backward of dq_embbag_int4_fwd with an SGD step on
 * binary32 master rows and re-quantization of the touched rows: the training step
 * of "Deep Quantized Recommendation Model (DQRM)", repository page (embedding
 * tables trained at INT4 with quantization-aware training). The pages fix no
 * arithmetic for it; this library computes:
 *   1. Entries: every position p of bag (t, b) with a valid id gives the entry
 *      (key = rows of tables 0..t-1 + id, p); the entries are sorted by (key, p).
 *   2. G (row gradient), element k: the binary64 sum of grad_out[b][t*d + k] over the
 *      row's entries inside each window of 64 consecutive sorted entries (windows at
 *      sorted positions 0, 64, 128, ...), summed from +0 in list order; those window
 *      parts added from +0 in window order in binary64; rounded once to binary32.
 *   3. master[id][k] = fma(-lr, G_k, master[id][k]) (binary32, one rounding).
 *   4. Each touched row is quantized again from its new master values (as
 *      dq_quantize_rows_int4 with `mode`, without row_loss/best_ij); untouched rows
 *      keep their codes, scale/bias and master values.
 * The result does not depend on scheduling: repeated calls give identical bits. Step 2
 * is the binary64 sum of the row's entries in list order, associated differently: it
 * equals that plain sum rounded once to binary32 except where the sum lies within
 * binary64 rounding error of a binary32 rounding boundary (then the two differ by one
 * ulp).
 *
 *   tables      HOST array of n_tables dq_master_table (1..DQ_MAX_TABLES)
 *   d           1..DQ_MAX_D
 *   indices, offsets, batch   as for dq_embbag_int4_fwd, but the offsets must be a CSR
 *               array: offsets[0] = 0, nondecreasing, offsets[n_tables*batch] =
 *               n_indices. Otherwise nothing is changed and DQ_FLAG_BAD_OFFSETS is
 *               raised (checked on the device)
 *   n_indices   number of ids, [0, 2^31); 0 is a no-op
 *   grad_out    [batch][n_tables*d] binary32, 4-byte aligned: gradient of the lookup
 *   lr          finite learning rate
 *   mode        DQ_MODE_GREEDY or DQ_MODE_MINMAX for the re-quantization
 *   workspace   device buffer, 256-byte aligned, of at least
 *               dq_embbag_int4_bwd_workspace_bytes(d, n_indices) bytes, owned by the
 *               caller and not in use by another call in flight; no contents kept
 *   d_flags     device uint32 (nullable): DQ_FLAG_BAD_INDEX (invalid ids, skipped),
 *               DQ_FLAG_BAD_OFFSETS, DQ_FLAG_NONFINITE, DQ_FLAG_FP16_OVERFLOW
 * Masters and packed tables must not overlap each other, the workspace or grad_out.
 */
dq_status dq_embbag_int4_bwd_sgd(const dq_master_table *tables, int32_t n_tables, int32_t d,
                                 const int32_t *indices, const int32_t *offsets, int32_t batch,
                                 int64_t n_indices, const float *grad_out, float lr, int32_t mode,
                                 void *workspace, size_t workspace_bytes, uint32_t *d_flags,
                                 void *cuda_stream);

/*
 * dq_embbag_int4_bwd_sgd_noalloc -- dq_embbag_int4_bwd_sgd without a caller
 * workspace, for callers that cannot allocate device memory (a plugin inside a host
 * program that owns the allocator, a process under a fixed memory budget, a server
 * that must not grow its device footprint). The paper has no counterpart: this is a
 * deployment convenience of this library.
 *
 * Its scratch is one static device array of DQ_BWD_STATIC_SCRATCH_BYTES (32 MiB),
 * held by every GPU that loads the library until the process exits. The call
 * allocates nothing. Arguments and results are those of dq_embbag_int4_bwd_sgd; a
 * call whose dq_embbag_int4_bwd_workspace_bytes(d, n_indices) exceeds the array is
 * rejected with DQ_ERR_INVALID_ARG (at most 378,856 entries at d = 16, 114,687 at
 * d = 64, 59,427 at d = 128).
 * The first call on a device looks up the array's device address there (once per
 * device), so make it before any stream capture. The address is cached per device
 * ordinal for the life of the process: after a cudaDeviceReset of a device the cached
 * address is stale, so do not call this entry point on that device again in the same
 * process. All calls share the array: calls
 * whose work overlaps on the GPU (several streams or host threads) race and must be
 * serialized by the caller. Each call clears what must start at zero itself.
 */
#define DQ_BWD_STATIC_SCRATCH_BYTES (32u << 20)
dq_status dq_embbag_int4_bwd_sgd_noalloc(const dq_master_table *tables, int32_t n_tables, int32_t d,
                                         const int32_t *indices, const int32_t *offsets, int32_t batch,
                                         int64_t n_indices, const float *grad_out, float lr, int32_t mode,
                                         uint32_t *d_flags, void *cuda_stream);

/* Static text for a status code. */
const char *dq_status_string(dq_status s);

/* The calling thread's last error message ("" if none); valid until its next call. */
const char *dq_last_error(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int32_t dq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DQ_H */
