// dq_kmeans.cu -- codebook 4-bit quantization (per-row k-means, 16 centroids), its
// dequantization and its sum-pooled bag, on sm_100a.
//
// "Post-Training 4-bit Quantization on Embedding Tables" (Guan et al., 2019), review
// page, section 提出的方法 (proposed method), bullet 3: codebook quantization through
// k-means clustering maps a row's values to a non-uniform set; section 主要发现 (main
// findings), bullet 3: it gives the lowest normalized l2 loss at 18.8%-37.5% of the
// FP32 size (16 binary16 centroids and d nibbles per row). The steps (dq.h states them):
// centroids start at the 16 levels of the min/max quantizer, `iters` Lloyd iterations
// in binary32 (nearest centroid by |x - c|, ties to the lower index; the mean of a
// cluster = its pairwise member sum / its size; an empty cluster keeps its centroid),
// binary16 storage, final codes against the stored centroids.
//
// Layout as the greedy quantizer's: a row of d <= P = next_pow2(d) elements in
// registers, W lanes per row, M = P / W contiguous elements per lane. A cluster's mean
// is its members' binary64 sum in index order over their count. When the row's
// nonzero values span at most 29 - ceil(log2 d) binades, every partial sum of its
// members is an integer multiple of the smallest value's ulp below 2^53 of them, i.e.
// exact in binary64, and any order gives the index-order sum: each element is then
// added once into its own cluster's binary64 accumulator (one per lane, in shared
// memory), and the W lanes' accumulators are added per cluster. Other rows (rare:
// values near zero beside large ones, non-finite values) are summed by one lane per
// row in index order. A warp stops iterating once every row's assignment has repeated
// (a fixed point of the iteration).
#include <cfloat>

#include "dq_internal.cuh"

namespace dq {
namespace {

constexpr float kLevels = 15.0f;

// Pairwise sum of v[0..M) (M a power of two), bottom-up: the recursive-halving tree.
template <int M>
__device__ __forceinline__ float block_pairwise(float (&v)[M])
{
#pragma unroll
    for (int s = 1; s < M; s <<= 1) {
#pragma unroll
        for (int i = 0; i < M; i += 2 * s)
            v[i] = __fadd_rn(v[i], v[i + s]);
    }
    return v[0];
}

template <int W>
__device__ __forceinline__ float row_pairwise(float lane_sum)
{
#pragma unroll
    for (int o = 1; o < W; o <<= 1)
        lane_sum = __fadd_rn(lane_sum, __shfl_xor_sync(0xffffffffu, lane_sum, o));
    return lane_sum;
}

// A warp's shared memory for the centroid update: per lane and cluster a binary64 sum
// and a count ([cluster][lane]: the warp's accesses are conflict-free whatever the
// clusters), or, on the sequential path, the lanes' elements and codes in index order.
// One per warp, as warps of a block may take different paths.
union KmeansUpdate {
    struct {
        double s[16][32];
        int32_t n[16][32];
    } acc;
    struct {
        float x[32 * 32];
        uint8_t q[32 * 32];
    } seq;
};

// q[m] = argmin_j fl(|fl(x[m] - c_j)|), ties to the lower j, for the lane's M elements;
// the centroids are read from shared memory, one j at a time (a short loop body keeps
// the kernel small enough for the instruction cache)
template <int M>
__device__ __forceinline__ void nearest_all(const float (&x)[M], const float *c, uint8_t (&q)[M])
{
    float bd[M];
    const float c0 = c[0];
#pragma unroll
    for (int m = 0; m < M; ++m) {
        bd[m] = fabsf(__fsub_rn(x[m], c0));
        q[m] = 0;
    }
#pragma unroll 1
    for (int j = 1; j < 16; ++j) {
        const float cj = c[j];
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const float dj = fabsf(__fsub_rn(x[m], cj));
            const bool better = dj < bd[m];
            bd[m] = better ? dj : bd[m];
            q[m] = better ? (uint8_t)j : q[m];
        }
    }
}

// Same result as nearest_all when the 16 centroids are finite and non-decreasing:
// fl(x - c) is monotone in c, so |fl(x - c_j)| does not rise while c_j <= x and does not
// fall after it; the first minimum is the last c_j <= x (moved left over equal
// distances) or the centroid after it. Four probes of a binary search find that c_j.
template <int M>
__device__ __forceinline__ void nearest_sorted(const float (&x)[M], const float *c, uint8_t (&q)[M])
{
#pragma unroll
    for (int m = 0; m < M; ++m) {
        int cnt = 0;  // number of c_j <= x
#pragma unroll
        for (int step = 8; step >= 1; step >>= 1)
            cnt = c[cnt + step - 1] <= x[m] ? cnt + step : cnt;
        int j = 0;
        if (cnt > 0) {
            j = cnt - 1;
            const float dl = fabsf(__fsub_rn(x[m], c[j]));
            const bool right = j < 15 && fabsf(__fsub_rn(x[m], c[j + 1])) < dl;
            if (right) {
                j += 1;
            } else {
                while (j > 0 && fabsf(__fsub_rn(x[m], c[j - 1])) == dl)
                    --j;
            }
        }
        q[m] = (uint8_t)j;
    }
}

// Are the row's centroids finite and non-decreasing (the condition of nearest_sorted)?
__device__ __forceinline__ bool sorted_finite(const float *c)
{
    bool ok = isfinite(c[0]);
#pragma unroll
    for (int j = 1; j < 16; ++j)
        ok &= isfinite(c[j]) && c[j - 1] <= c[j];
    return ok;
}

template <int M>
__device__ __forceinline__ void nearest(const float (&x)[M], const float *c, uint8_t (&q)[M])
{
    if (sorted_finite(c))
        nearest_sorted<M>(x, c, q);
    else
        nearest_all<M>(x, c, q);
}

// One row per W lanes, M contiguous elements per lane; FULL: d == M * W.
template <int M, int W, bool FULL>
__global__ void __launch_bounds__(128) kmeans_rows_kernel(const KmeansArgs a)
{
    const int sub = threadIdx.x & (W - 1);
    int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / W;
    const bool active = row < a.n;
    if (!active)
        row = a.n - 1;  // idle lanes shadow the last row so the warp stays converged
    const int d = a.d;
    const int kbase = sub * M;
    const float *xr = a.x + row * a.ld + kbase;
    float x[M];
    bool nonfinite = false;
    float mn = FLT_MAX, mx = -FLT_MAX;
#pragma unroll
    for (int m = 0; m < M; ++m) {
        const bool ok = FULL || kbase + m < d;
        x[m] = ok ? __ldg(xr + m) : 0.0f;
        if (ok) {
            mn = fminf(mn, x[m]);
            mx = fmaxf(mx, x[m]);
            nonfinite |= !isfinite(x[m]);
        }
    }
    // binary exponent fields of the lane's nonzero values (subnormals count as 1: the
    // same ulp), for the row's span
    int emax = 0, emin = 255;
#pragma unroll
    for (int m = 0; m < M; ++m) {
        const uint32_t u = __float_as_uint(x[m]) & 0x7fffffffu;
        if ((FULL || kbase + m < d) && u != 0u) {
            const int e = max((int)(u >> 23), 1);
            emax = max(emax, e);
            emin = min(emin, e);
        }
    }
    int nf = nonfinite ? 1 : 0;
#pragma unroll
    for (int o = 1; o < W; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
        emin = min(emin, __shfl_xor_sync(0xffffffffu, emin, o));
        nf |= __shfl_xor_sync(0xffffffffu, nf, o);
    }
    const int clog2d = d > 1 ? 32 - __clz(d - 1) : 0;
    const bool exact_row = nf == 0 && (emax == 0 || emax - emin <= 29 - clog2d);
    const bool exact = __all_sync(0xffffffffu, exact_row);  // the warp's update path
    __shared__ KmeansUpdate upd_all[4];
    KmeansUpdate &upd = upd_all[threadIdx.x >> 5];
    const int lane = threadIdx.x & 31;
    const int row0 = lane & ~(W - 1);  // the row's first lane in the warp
    // the row's 16 centroids live in shared memory (every lane of the row writes the
    // same values; __syncwarp orders the writes before the reads)
    __shared__ float cs_all[128 / W][17];  // padded: rows' slots start in different banks
    float *c = cs_all[threadIdx.x / W];
    // K1: the min/max levels
    const float step = __fdiv_rn(__fsub_rn(mx, mn), kLevels);
    if (sub == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            c[j] = __fmaf_rn((float)j, step, mn);
    }
    __syncwarp();
    // K2: Lloyd iterations. When an assignment repeats the previous one, the update would
    // reproduce the current centroids, and so would every later iteration: the warp stops
    // once all its rows have repeated (rows that repeated earlier recompute their own
    // centroids unchanged until then).
    uint8_t q[M];
    constexpr int kWords = (M + 7) / 8;  // the lane's codes, 4 bits each
    uint32_t prev[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w)
        prev[w] = 0u;
    int it = 0;
    for (; it < a.iters; ++it) {
        nearest<M>(x, c, q);
        uint32_t pk[kWords];
#pragma unroll
        for (int w = 0; w < kWords; ++w)
            pk[w] = 0u;
#pragma unroll
        for (int m = 0; m < M; ++m)
            pk[m / 8] |= (uint32_t)q[m] << (4 * (m % 8));
        bool same = it > 0;
#pragma unroll
        for (int w = 0; w < kWords; ++w) {
            same &= pk[w] == prev[w];
            prev[w] = pk[w];
        }
        if (__all_sync(0xffffffffu, same))
            break;
        __syncwarp();  // every lane has read the centroids before they change
        if (exact) {
            // every element into its own cluster's accumulator of this lane
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                upd.acc.s[j][lane] = 0.0;
                upd.acc.n[j][lane] = 0;
            }
#pragma unroll
            for (int m = 0; m < M; ++m) {
                if (FULL || kbase + m < d) {
                    const int j = q[m];
                    upd.acc.s[j][lane] += (double)x[m];
                    upd.acc.n[j][lane] += 1;
                }
            }
            __syncwarp();
            // lane `sub` of the row takes clusters sub, sub + W, ...
            for (int j = sub; j < 16; j += W) {
                double sj = 0.0;
                int nj = 0;
#pragma unroll 4
                for (int l = 0; l < W; ++l) {
                    sj += upd.acc.s[j][row0 + l];
                    nj += upd.acc.n[j][row0 + l];
                }
                if (nj > 0)
                    c[j] = __double2float_rn(__ddiv_rn(sj, (double)nj));
            }
        } else {
            // one lane per row adds the members in index order
#pragma unroll
            for (int m = 0; m < M; ++m) {
                upd.seq.x[lane * M + m] = x[m];
                upd.seq.q[lane * M + m] = q[m];
            }
            __syncwarp();
            if (sub == 0) {
                double sj[16];
                int nj[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    sj[j] = 0.0;
                    nj[j] = 0;
                }
                for (int k = 0; k < d; ++k) {
                    const int j = upd.seq.q[row0 * M + k];
                    sj[j] += (double)upd.seq.x[row0 * M + k];
                    nj[j] += 1;
                }
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (nj[j] > 0)
                        c[j] = __double2float_rn(__ddiv_rn(sj[j], (double)nj[j]));
            }
        }
        __syncwarp();  // the updated centroids, and the accumulators free again
    }
    // K3: binary16 centroids, final codes, loss
    __half h[16];
    if (sub == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            h[j] = __float2half_rn(c[j]);
            c[j] = __half2float(h[j]);
        }
    }
    __syncwarp();
    nearest<M>(x, c, q);
    float e2[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
        const bool ok = FULL || kbase + m < d;
        if (!ok)
            q[m] = 0;
        const float e = __fsub_rn(x[m], c[q[m]]);
        e2[m] = ok ? __fmul_rn(e, e) : 0.0f;
    }
    const float loss = row_pairwise<W>(block_pairwise<M>(e2));
    if (!active)
        return;
    if (a.row_iters && sub == 0)
        a.row_iters[row] = it;
    uint8_t *cr = a.codes + row * a.codes_ld + kbase / 2;
#pragma unroll
    for (int m = 0; m < (M + 1) / 2; ++m) {
        const int k0 = 2 * m;
        if (FULL || kbase + k0 < d) {
            const unsigned lo = q[k0];
            const unsigned hi = (k0 + 1 < M) ? q[k0 + 1] : 0u;
            cr[m] = (uint8_t)(lo | (hi << 4));
        }
    }
    if (sub == 0) {
        uint16_t *cb = a.codebook + 16 * row;
        bool over = false;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            cb[j] = __half_as_ushort(h[j]);
            over |= isinf(c[j]);
        }
        if (a.row_loss)
            a.row_loss[row] = loss;
        if (over)
            raise_flag(a.flags, DQ_FLAG_FP16_OVERFLOW);
    }
    if (nonfinite)
        raise_flag(a.flags, DQ_FLAG_NONFINITE);
}

template <int M, int W>
cudaError_t launch_kmeans_mw(const KmeansArgs &a, cudaStream_t stream)
{
    constexpr int kBlock = 128;
    const int64_t grid = (a.n * W + kBlock - 1) / kBlock;
    if (a.d == M * W)
        kmeans_rows_kernel<M, W, true><<<(unsigned)grid, kBlock, 0, stream>>>(a);
    else
        kmeans_rows_kernel<M, W, false><<<(unsigned)grid, kBlock, 0, stream>>>(a);
    return cudaGetLastError();
}

// xhat = w(C[q]): one thread per pair of elements.
__global__ void __launch_bounds__(256) kmeans_dequant_kernel(const KmeansDequantArgs a)
{
    const int pairs = (a.d + 1) / 2;
    const int64_t total = a.n * pairs;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / pairs;
        const int m = (int)(i - r * pairs);
        const unsigned byte = __ldg(a.codes + r * a.codes_ld + m);
        const uint16_t *cb = a.codebook + 16 * r;
        float *o = a.out + r * a.out_ld + 2 * m;
        o[0] = __half2float(__ushort_as_half(__ldg(cb + (byte & 15u))));
        if (2 * m + 1 < a.d)
            o[1] = __half2float(__ushort_as_half(__ldg(cb + (byte >> 4))));
    }
}

// One warp per bag (t, b); lane l owns elements l, l + 32, ... (CH chunks of 32); per id,
// lanes 0..15 read the row's 16 centroids and each lane takes its elements' centroids by
// shuffle. The sum runs in binary32 in id order, so a bag of one id returns the
// dequantized row. The next bag's offsets, and the id at its own position (where a
// one-id bag of an all-one-hot call keeps it), are loaded while the current bag is summed.
template <int CH>
__device__ __forceinline__ void bag_per_warp(const KmeansBagTables &tabs, const KmeansBagArgs &a, int64_t G,
                                             int32_t total)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int32_t np0 = 0, np1 = 0, nid = -1;
    if (warp < G) {
        np0 = __ldg(a.offsets + warp);
        np1 = __ldg(a.offsets + warp + 1);
        nid = warp < total ? __ldg(a.indices + warp) : -1;
    }
    for (int64_t g = warp; g < G; g += warps) {
        int32_t p0 = np0, p1 = np1;
        const int32_t own = nid;
        const int64_t gn = g + warps;
        if (gn < G) {
            np0 = __ldg(a.offsets + gn);
            np1 = __ldg(a.offsets + gn + 1);
            nid = gn < total ? __ldg(a.indices + gn) : -1;
        }
        const int t = (int)div_batch((uint32_t)g, a.div);
        const int64_t b = g - (int64_t)t * a.batch;
        p0 = p0 < 0 ? 0 : (p0 > total ? total : p0);
        p1 = p1 < 0 ? 0 : (p1 > total ? total : p1);
        if (p1 < p0) {
            if (lane == 0)
                raise_flag(a.flags, DQ_FLAG_BAD_OFFSETS);
            p1 = p0;
        }
        const int64_t n_rows = tabs.n_rows[t];
        const uint16_t *cbt = tabs.codebook[t];
        const uint8_t *ct = tabs.codes[t];
        const int64_t cld = tabs.codes_ld[t];
        float acc[CH];
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
            acc[ch] = 0.0f;
        for (int32_t p = p0; p < p1; ++p) {
            const int32_t id = (int64_t)p == g ? own : __ldg(a.indices + p);
            if (id < 0 || id >= n_rows) {
                if (lane == 0)
                    raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
                continue;
            }
            const float cj = lane < 16 ? __half2float(__ushort_as_half(__ldg(cbt + 16 * (int64_t)id + lane))) : 0.0f;
            const uint8_t *cr = ct + (int64_t)id * cld;
#pragma unroll
            for (int ch = 0; ch < CH; ++ch) {
                const int k = ch * 32 + lane;
                unsigned qk = 0;
                if (k < a.d)
                    qk = (__ldg(cr + k / 2) >> (4 * (k & 1))) & 15u;
                acc[ch] = __fadd_rn(acc[ch], __shfl_sync(0xffffffffu, cj, (int)qk));
            }
        }
        float *out = a.out + b * (int64_t)a.T * a.d + (int64_t)t * a.d;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
            const int k = ch * 32 + lane;
            if (k < a.d)
                out[k] = acc[ch];
        }
    }
}

// Short bags (under two ids on average): a warp takes 32 consecutive bags. Lane j does bag
// j's bookkeeping (offsets, the id, row pointers, output row) into a per-warp table in
// shared memory; then the warp writes the bags' rows in groups of 8, with the 8 bags'
// centroids and codes loaded before any is decoded (lanes 0..15 hold a centroid each,
// every lane CH code bytes). Empty bags and bags of an invalid id write +0; bags of two or
// more ids are summed afterwards, one at a time, in id order.
constexpr int64_t kTileMinBags = 65536;   // 2048 tiles of 32 bags: enough to fill the GPU

struct CbSlot {
    const uint16_t *cb;   // the row's 16 centroids (one-id bags)
    const uint8_t *cr;    // the row's codes
    float *out;           // the bag's output row
    int32_t p0, p1;       // the clamped offsets (bags of two or more ids)
    int32_t kind;         // 0: one valid id, 1: write +0, 2: two or more ids
    int32_t t;
};

template <int CH>
__device__ __forceinline__ void bag_tiles(const KmeansBagTables &tabs, const KmeansBagArgs &a, int64_t G,
                                          int32_t total, CbSlot *slots)
{
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    for (int64_t g0 = ((int64_t)blockIdx.x * wpb + (threadIdx.x >> 5)) * 32; g0 < G; g0 += (int64_t)gridDim.x * wpb * 32) {
        const int64_t g = g0 + lane;
        unsigned multi = 0;
        if (g < G) {
            int32_t p0 = __ldg(a.offsets + g), p1 = __ldg(a.offsets + g + 1);
            const int32_t own = g < total ? __ldg(a.indices + g) : -1;
            p0 = p0 < 0 ? 0 : (p0 > total ? total : p0);
            p1 = p1 < 0 ? 0 : (p1 > total ? total : p1);
            if (p1 < p0) {
                raise_flag(a.flags, DQ_FLAG_BAD_OFFSETS);
                p1 = p0;
            }
            const int t = (int)div_batch((uint32_t)g, a.div);
            const int64_t b = g - (int64_t)t * a.batch;
            CbSlot sl;
            sl.out = a.out + b * (int64_t)a.T * a.d + (int64_t)t * a.d;
            sl.p0 = p0;
            sl.p1 = p1;
            sl.t = t;
            sl.cb = nullptr;
            sl.cr = nullptr;
            sl.kind = 1;
            if (p1 == p0 + 1) {
                const int32_t id = (int64_t)p0 == g ? own : __ldg(a.indices + p0);
                if (id >= 0 && (int64_t)id < tabs.n_rows[t]) {
                    sl.cb = tabs.codebook[t] + 16 * (int64_t)id;
                    sl.cr = tabs.codes[t] + (int64_t)id * tabs.codes_ld[t];
                    sl.kind = 0;
                } else {
                    raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
                }
            } else if (p1 > p0 + 1) {
                sl.kind = 2;
            }
            slots[lane] = sl;
        }
        multi = __ballot_sync(0xffffffffu, g < G && slots[lane].kind == 2);
        __syncwarp();
        const int nb = (int)min((int64_t)32, G - g0);
        for (int j0 = 0; j0 < nb; j0 += 8) {
            float cj[8];
            unsigned q[8][CH];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u;
                const bool one = j < nb && slots[j].kind == 0;
                cj[u] = (one && lane < 16) ? __half2float(__ushort_as_half(__ldg(slots[j].cb + lane))) : 0.0f;
#pragma unroll
                for (int ch = 0; ch < CH; ++ch) {
                    const int k = ch * 32 + lane;
                    q[u][ch] = (one && k < a.d) ? (unsigned)__ldg(slots[j].cr + k / 2) : 0u;
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u;
                if (j >= nb)
                    break;
                const int kind = slots[j].kind;   // warp-uniform
                if (kind == 2)
                    continue;
                float *o = slots[j].out;
#pragma unroll
                for (int ch = 0; ch < CH; ++ch) {
                    const int k = ch * 32 + lane;
                    const unsigned qk = (q[u][ch] >> (4 * (k & 1))) & 15u;
                    const float v = __shfl_sync(0xffffffffu, cj[u], (int)qk);
                    if (k < a.d)
                        o[k] = kind == 0 ? __fadd_rn(0.0f, v) : 0.0f;
                }
            }
        }
        while (multi) {   // bags of two or more ids, one at a time
            const int j = __ffs(multi) - 1;
            multi &= multi - 1;
            const CbSlot sl = slots[j];
            const int64_t n_rows = tabs.n_rows[sl.t];
            const uint16_t *cbt = tabs.codebook[sl.t];
            const uint8_t *ct = tabs.codes[sl.t];
            const int64_t cld = tabs.codes_ld[sl.t];
            float acc[CH];
#pragma unroll
            for (int ch = 0; ch < CH; ++ch)
                acc[ch] = 0.0f;
            for (int32_t p = sl.p0; p < sl.p1; ++p) {
                const int32_t id = __ldg(a.indices + p);
                if (id < 0 || id >= n_rows) {
                    if (lane == 0)
                        raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
                    continue;
                }
                const float c = lane < 16 ? __half2float(__ushort_as_half(__ldg(cbt + 16 * (int64_t)id + lane))) : 0.0f;
                const uint8_t *cr = ct + (int64_t)id * cld;
#pragma unroll
                for (int ch = 0; ch < CH; ++ch) {
                    const int k = ch * 32 + lane;
                    unsigned qk = 0;
                    if (k < a.d)
                        qk = (__ldg(cr + k / 2) >> (4 * (k & 1))) & 15u;
                    acc[ch] = __fadd_rn(acc[ch], __shfl_sync(0xffffffffu, c, (int)qk));
                }
            }
#pragma unroll
            for (int ch = 0; ch < CH; ++ch) {
                const int k = ch * 32 + lane;
                if (k < a.d)
                    sl.out[k] = acc[ch];
            }
        }
        __syncwarp();   // the slots are rewritten by the next tile
    }
}

template <int CH>
__global__ void __launch_bounds__(256) kmeans_bag_kernel(const __grid_constant__ KmeansBagTables tabs,
                                                         const KmeansBagArgs a)
{
    const int64_t G = (int64_t)a.T * a.batch;
    bag_per_warp<CH>(tabs, a, G, __ldg(a.offsets + G));
}

// Rows of d = 16·E elements with E/2-byte aligned code pieces: each half-warp takes every
// other id of the bag (two of them loaded before either is added), its 16 lanes holding the
// row's 16 centroids and each lane decoding E consecutive elements from one E/2-byte load;
// the halves' sums are added at the end (two interleaved id-order sums: a bag of one id still
// returns the dequantized row).
template <int E>
__device__ __forceinline__ void load_codes(const uint8_t *p, uint32_t (&w)[(E + 7) / 8])
{
    if constexpr (E == 4)
        w[0] = __ldg(reinterpret_cast<const uint16_t *>(p));
    else if constexpr (E == 8)
        w[0] = __ldg(reinterpret_cast<const uint32_t *>(p));
    else {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
        w[0] = v.x;
        w[1] = v.y;
    }
}

template <int E>
__global__ void __launch_bounds__(256) kmeans_bag_half_kernel(const __grid_constant__ KmeansBagTables tabs,
                                                              const KmeansBagArgs a)
{
    constexpr int NW = (E + 7) / 8;
    const int lane = threadIdx.x & 31;
    const int h = lane >> 4, c = lane & 15;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t G = (int64_t)a.T * a.batch;
    const int32_t total = __ldg(a.offsets + G);
    int32_t np0 = 0, np1 = 0, nid = -1;
    if (warp < G) {
        np0 = __ldg(a.offsets + warp);
        np1 = __ldg(a.offsets + warp + 1);
        nid = warp < total ? __ldg(a.indices + warp) : -1;
    }
    for (int64_t g = warp; g < G; g += warps) {
        int32_t p0 = np0, p1 = np1;
        const int32_t own = nid;
        const int64_t gn = g + warps;
        if (gn < G) {
            np0 = __ldg(a.offsets + gn);
            np1 = __ldg(a.offsets + gn + 1);
            nid = gn < total ? __ldg(a.indices + gn) : -1;
        }
        const int t = (int)div_batch((uint32_t)g, a.div);
        const int64_t b = g - (int64_t)t * a.batch;
        p0 = p0 < 0 ? 0 : (p0 > total ? total : p0);
        p1 = p1 < 0 ? 0 : (p1 > total ? total : p1);
        if (p1 < p0) {
            if (lane == 0)
                raise_flag(a.flags, DQ_FLAG_BAD_OFFSETS);
            p1 = p0;
        }
        const int64_t n_rows = tabs.n_rows[t];
        const uint16_t *cbt = tabs.codebook[t];
        const uint8_t *ct = tabs.codes[t] + c * (E / 2);
        const int64_t cld = tabs.codes_ld[t];
        float acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            acc[e] = 0.0f;
        bool bad = false;
        for (int32_t q0 = p0; q0 < p1; q0 += 4) {   // this half's ids: q0 + h, q0 + 2 + h
            int32_t id[2];
            bool ok[2];
            float cj[2];
            uint32_t w[2][NW];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int32_t p = q0 + 2 * u + h;
                id[u] = -1;
                if (p < p1)
                    id[u] = (int64_t)p == g ? own : __ldg(a.indices + p);
                ok[u] = id[u] >= 0 && (int64_t)id[u] < n_rows;
                bad |= p < p1 && !ok[u];
                cj[u] = 0.0f;
#pragma unroll
                for (int k = 0; k < NW; ++k)
                    w[u][k] = 0u;
                if (ok[u]) {
                    cj[u] = __half2float(__ushort_as_half(__ldg(cbt + 16 * (int64_t)id[u] + c)));
                    load_codes<E>(ct + (int64_t)id[u] * cld, w[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const unsigned qk = (w[u][e / 8] >> (4 * (e % 8))) & 15u;
                    const float v = __shfl_sync(0xffffffffu, cj[u], (h << 4) | (int)qk);
                    if (ok[u])
                        acc[e] = __fadd_rn(acc[e], v);
                }
            }
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0)
            raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
        float *out = a.out + b * (int64_t)a.T * a.d + (int64_t)t * a.d + c * E;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float other = __shfl_xor_sync(0xffffffffu, acc[e], 16);
            if (h == 0)
                out[e] = __fadd_rn(acc[e], other);
        }
    }
}

// d <= 16: each half-warp walks its own bags (lane c of the half: element c and centroid c),
// so a warp has two bags in flight; the halves' shuffles name only their own 16 lanes.
__global__ void __launch_bounds__(256) kmeans_bag16_kernel(const __grid_constant__ KmeansBagTables tabs,
                                                           const KmeansBagArgs a)
{
    const int lane = threadIdx.x & 31;
    const int h = lane >> 4, c = lane & 15;
    const unsigned hmask = 0xffffu << (16 * h);
    const int64_t half = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * 2 + h;
    const int64_t halves = (((int64_t)gridDim.x * blockDim.x) >> 5) * 2;
    const int64_t G = (int64_t)a.T * a.batch;
    const int32_t total = __ldg(a.offsets + G);
    int32_t np0 = 0, np1 = 0, nid = -1;
    if (half < G) {
        np0 = __ldg(a.offsets + half);
        np1 = __ldg(a.offsets + half + 1);
        nid = half < total ? __ldg(a.indices + half) : -1;
    }
    for (int64_t g = half; g < G; g += halves) {
        int32_t p0 = np0, p1 = np1;
        const int32_t own = nid;
        const int64_t gn = g + halves;
        if (gn < G) {
            np0 = __ldg(a.offsets + gn);
            np1 = __ldg(a.offsets + gn + 1);
            nid = gn < total ? __ldg(a.indices + gn) : -1;
        }
        const int t = (int)div_batch((uint32_t)g, a.div);
        const int64_t b = g - (int64_t)t * a.batch;
        p0 = p0 < 0 ? 0 : (p0 > total ? total : p0);
        p1 = p1 < 0 ? 0 : (p1 > total ? total : p1);
        if (p1 < p0) {
            if (c == 0)
                raise_flag(a.flags, DQ_FLAG_BAD_OFFSETS);
            p1 = p0;
        }
        const int64_t n_rows = tabs.n_rows[t];
        const uint16_t *cbt = tabs.codebook[t];
        const uint8_t *ct = tabs.codes[t];
        const int64_t cld = tabs.codes_ld[t];
        float acc = 0.0f;
        for (int32_t p = p0; p < p1; ++p) {
            const int32_t id = (int64_t)p == g ? own : __ldg(a.indices + p);
            if (id < 0 || id >= n_rows) {
                if (c == 0)
                    raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
                continue;
            }
            const float cj = __half2float(__ushort_as_half(__ldg(cbt + 16 * (int64_t)id + c)));
            unsigned qk = 0;
            if (c < a.d)
                qk = (__ldg(ct + (int64_t)id * cld + c / 2) >> (4 * (c & 1))) & 15u;
            acc = __fadd_rn(acc, __shfl_sync(hmask, cj, (int)qk, 16));
        }
        if (c < a.d)
            a.out[b * (int64_t)a.T * a.d + (int64_t)t * a.d + c] = acc;
    }
}

// Calls of many bags at d <= 64: the id count (the last offset) picks the layout, 32 bags
// per warp when the bags hold under two ids on average, else one warp per bag. (A kernel
// of its own: the tile layout's registers would cost the smaller calls occupancy.)
template <int CH>
__global__ void __launch_bounds__(256) kmeans_bag_tile_kernel(const __grid_constant__ KmeansBagTables tabs,
                                                              const KmeansBagArgs a)
{
    __shared__ CbSlot slots_all[8][32];
    const int64_t G = (int64_t)a.T * a.batch;
    const int32_t total = __ldg(a.offsets + G);
    if ((int64_t)total < 2 * G)
        bag_tiles<CH>(tabs, a, G, total, slots_all[threadIdx.x >> 5]);
    else
        bag_per_warp<CH>(tabs, a, G, total);
}

} // namespace

cudaError_t launch_kmeans(const KmeansArgs &a, cudaStream_t stream)
{
    int p = 1;
    while (p < a.d)
        p <<= 1;
    switch (p) {
    case 1: return launch_kmeans_mw<1, 1>(a, stream);
    case 2: return launch_kmeans_mw<2, 1>(a, stream);
    case 4: return launch_kmeans_mw<4, 1>(a, stream);
    case 8: return launch_kmeans_mw<8, 1>(a, stream);
    case 16: return launch_kmeans_mw<16, 1>(a, stream);
    case 32: return launch_kmeans_mw<16, 2>(a, stream);
    case 64: return launch_kmeans_mw<16, 4>(a, stream);
    case 128: return launch_kmeans_mw<16, 8>(a, stream);
    case 256: return launch_kmeans_mw<16, 16>(a, stream);
    case 512: return launch_kmeans_mw<16, 32>(a, stream);
    case 1024: return launch_kmeans_mw<32, 32>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_kmeans_dequantize(const KmeansDequantArgs &a, int num_sms, cudaStream_t stream)
{
    const int64_t total = a.n * ((a.d + 1) / 2);
    const int64_t need = (total + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 16;
    kmeans_dequant_kernel<<<(unsigned)(need < cap ? need : cap), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_kmeans_bag(const KmeansBagTables &tabs, const KmeansBagArgs &a, int num_sms, cudaStream_t stream)
{
    const int64_t G = (int64_t)a.T * a.batch;
    const int64_t need = (G * 32 + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 16;
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    const int chunks = (a.d + 31) / 32;
    if (G >= kTileMinBags && chunks <= 2) {
        if (chunks <= 1)
            kmeans_bag_tile_kernel<1><<<grid, 256, 0, stream>>>(tabs, a);
        else
            kmeans_bag_tile_kernel<2><<<grid, 256, 0, stream>>>(tabs, a);
        return cudaGetLastError();
    }
    // d = 64, 128, 256 with every table's code rows E/2-byte aligned: two ids per warp
    const int E = a.d / 16;
    bool half = (a.d == 64 || a.d == 128 || a.d == 256);
    for (int t = 0; half && t < a.T; ++t)
        half = tabs.codes_ld[t] % (E / 2) == 0 && (reinterpret_cast<uintptr_t>(tabs.codes[t]) % (E / 2)) == 0;
    if (half) {
        if (E == 4)
            kmeans_bag_half_kernel<4><<<grid, 256, 0, stream>>>(tabs, a);
        else if (E == 8)
            kmeans_bag_half_kernel<8><<<grid, 256, 0, stream>>>(tabs, a);
        else
            kmeans_bag_half_kernel<16><<<grid, 256, 0, stream>>>(tabs, a);
        return cudaGetLastError();
    }
    if (a.d <= 16) {
        const int64_t need16 = (G * 16 + 255) / 256;
        kmeans_bag16_kernel<<<(unsigned)(need16 < cap ? need16 : cap), 256, 0, stream>>>(tabs, a);
        return cudaGetLastError();
    }
    if (chunks <= 1)
        kmeans_bag_kernel<1><<<grid, 256, 0, stream>>>(tabs, a);
    else if (chunks <= 2)
        kmeans_bag_kernel<2><<<grid, 256, 0, stream>>>(tabs, a);
    else if (chunks <= 4)
        kmeans_bag_kernel<4><<<grid, 256, 0, stream>>>(tabs, a);
    else if (chunks <= 8)
        kmeans_bag_kernel<8><<<grid, 256, 0, stream>>>(tabs, a);
    else if (chunks <= 16)
        kmeans_bag_kernel<16><<<grid, 256, 0, stream>>>(tabs, a);
    else
        kmeans_bag_kernel<32><<<grid, 256, 0, stream>>>(tabs, a);
    return cudaGetLastError();
}

} // namespace dq
