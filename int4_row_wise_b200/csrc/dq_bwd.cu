// dq_bwd.cu -- backward of the sum-pooled INT4 embedding bag: grouping the bag
// entries by row and reducing each row's gradient, deterministically.
//
// The training step after the lookup in "Deep Quantized Recommendation Model
// (DQRM)", repository page (embedding tables trained at INT4 by quantization-aware
// training on binary32 masters): every entry (bag (t, b), id) adds the bag's output
// gradient g[b][t*d .. t*d + d) to the gradient of row id of table t; the touched
// masters take an SGD step and are quantized again (dq_quantize.cu, fused with the
// SGD update).
//
// Order of the sums (dq.h states it): the entries, keyed by the global row
// key = key_base[t] + id, are stably sorted by key (so positions ascend within a
// row); the sorted list is cut into windows of 64 entries; a row's gradient is the
// binary64 sum of its entries inside each window, then of those window parts in
// window order, rounded once to binary32. The result is the same whatever the
// scheduling, so the updated masters and their codes are reproducible.
//
// Kernels, in stream order:
//   bwd_keys_kernel      one lane per bag: writes (key, bag) of each of its entries;
//                        checks that offsets are a CSR array (else nothing changes)
//   radix_hist_kernel    LSD radix sort, 8-bit digits, ceil(bits(total rows) / 8)
//   radix_scan_kernel    passes of three kernels each: per-tile digit counts,
//   radix_scatter_kernel their digit-major exclusive scan, and a stable scatter
//                        (warp-striped tiles ranked with ballots, no atomics)
//   bwd_window_kernel    one warp per window: sums each row's part in binary64;
//                        a row wholly inside the window gets its G and a list slot,
//                        a row crossing a window edge leaves a binary64 part
//   bwd_span_kernel      one warp per row that spans windows: adds its parts in
//                        window order and lists it
// Every loop is bounded by sizes known at launch; no kernel waits on another.
#include "dq_internal.cuh"

namespace dq {
namespace {

constexpr int kWin = 64;                          // entries per window of the sorted list
constexpr int kSortThreads = 256;
constexpr int kSortItems = 8;
constexpr int kTile = kSortThreads * kSortItems;  // entries per sort tile
constexpr int kDigits = 256;
constexpr int kRedThreads = 256;                  // 8 warps per block in the reductions

// Lanes of the warp whose 8-bit digit equals this lane's (only lanes with ok set).
__device__ __forceinline__ unsigned digit_peers(uint32_t dg, bool ok)
{
    unsigned peers = __ballot_sync(0xffffffffu, ok);
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        const bool bit = (dg >> b) & 1u;
        const unsigned bb = __ballot_sync(0xffffffffu, bit);
        peers &= bit ? bb : ~bb;
    }
    return peers;
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    return (1u << (threadIdx.x & 31)) - 1u;
}

// Exclusive scan of one value per thread over a block of kSortThreads threads.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_tot, uint32_t &block_total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o)
            inc += y;
    }
    if (lane == 31)
        warp_tot[warp] = inc;
    __syncthreads();
    uint32_t before = 0, all = 0;
    for (int w = 0; w < kSortThreads / 32; ++w) {
        const uint32_t t = warp_tot[w];
        before += w < warp ? t : 0u;
        all += t;
    }
    __syncthreads();
    block_total = all;
    return before + inc - v;
}

// ---------------------------------------------------------------------------
// entries
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) bwd_keys_kernel(const BwdArgs a)
{
    const int64_t G = (int64_t)a.T * a.batch;
    const uint32_t sentinel = a.key_base[a.T];
    bool bad = false, bad_id = false;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < G; g += stride) {
        int64_t p0 = a.offsets[g], p1 = a.offsets[g + 1];
        bad |= p1 < p0;
        p0 = p0 < 0 ? 0 : (p0 > a.n ? a.n : p0);  // keep every write inside the entry arrays
        p1 = p1 < p0 ? p0 : (p1 > a.n ? a.n : p1);
        const int t = (int)div_batch((uint32_t)g, a.div);
        const uint32_t base = a.key_base[t], rows = a.key_base[t + 1] - base;
        for (int64_t p = p0; p < p1; ++p) {
            const int32_t id = __ldg(a.indices + p);
            const bool ok = id >= 0 && (uint32_t)id < rows;
            bad_id |= !ok;
            a.keys[0][p] = ok ? base + (uint32_t)id : sentinel;
            a.bags[0][p] = (int32_t)g;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0)
        bad |= a.offsets[0] != 0 || (int64_t)a.offsets[G] != a.n;
    if (bad) {
        atomicOr(a.hdr, 1u);
        raise_flag(a.flags, DQ_FLAG_BAD_OFFSETS);
    }
    if (bad_id)
        raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
}

// ---------------------------------------------------------------------------
// LSD radix sort of (key, bag) pairs
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kSortThreads) radix_hist_kernel(const uint32_t *keys, int64_t n, int shift,
                                                                  uint32_t *hist, int64_t tiles)
{
    __shared__ uint32_t cnt[kDigits];
    cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kTile;
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < kSortItems; ++j) {
        const int64_t p = base + j * kSortThreads + threadIdx.x;
        const bool ok = p < n;
        const uint32_t dg = ok ? (__ldg(keys + p) >> shift) & 255u : 0u;
        const unsigned peers = digit_peers(dg, ok);
        if (ok && lane == __ffs(peers) - 1)
            atomicAdd(&cnt[dg], (uint32_t)__popc(peers));
    }
    __syncthreads();
    hist[threadIdx.x * tiles + blockIdx.x] = cnt[threadIdx.x];
}

// One block per digit: exclusive scan of the digit's per-tile counts, in place.
__global__ void __launch_bounds__(kSortThreads) radix_scan_kernel(uint32_t *hist, int64_t tiles, uint32_t *totals)
{
    __shared__ uint32_t warp_tot[kSortThreads / 32];
    uint32_t *row = hist + (int64_t)blockIdx.x * tiles;
    uint32_t carry = 0;
    for (int64_t c0 = 0; c0 < tiles; c0 += kSortThreads * 4) {
        const int64_t i0 = c0 + threadIdx.x * 4;
        uint32_t v[4], local = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[k] = i0 + k < tiles ? row[i0 + k] : 0u;
            local += v[k];
        }
        uint32_t chunk_total;
        uint32_t run = carry + block_exclusive_scan(local, warp_tot, chunk_total);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (i0 + k < tiles)
                row[i0 + k] = run;
            run += v[k];
        }
        carry += chunk_total;
    }
    if (threadIdx.x == 0)
        totals[blockIdx.x] = carry;
}

// Stable scatter of one tile: warp w takes entries [w*256, w*256 + 256) of the tile
// in rounds of 32 consecutive entries, so (warp, round, lane) is the entry order.
__global__ void __launch_bounds__(kSortThreads) radix_scatter_kernel(const uint32_t *keys_in, const int32_t *bags_in,
                                                                     uint32_t *keys_out, int32_t *bags_out, int64_t n,
                                                                     int shift, const uint32_t *hist,
                                                                     const uint32_t *totals, int64_t tiles)
{
    __shared__ uint32_t digit_base[kDigits];
    __shared__ uint32_t wcnt[kSortThreads / 32][kDigits];
    __shared__ uint32_t warp_tot[kSortThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    {
        uint32_t all;
        const uint32_t before = block_exclusive_scan(totals[threadIdx.x], warp_tot, all);
        digit_base[threadIdx.x] = before + hist[threadIdx.x * tiles + blockIdx.x];
#pragma unroll
        for (int w = 0; w < kSortThreads / 32; ++w)
            wcnt[w][threadIdx.x] = 0;
    }
    __syncthreads();
    const int64_t wbase = (int64_t)blockIdx.x * kTile + warp * 32 * kSortItems;
    uint32_t k[kSortItems], rank[kSortItems];
    int32_t v[kSortItems];
#pragma unroll
    for (int j = 0; j < kSortItems; ++j) {
        const int64_t p = wbase + j * 32 + lane;
        k[j] = p < n ? __ldg(keys_in + p) : 0u;
        v[j] = p < n ? __ldg(bags_in + p) : 0;
    }
#pragma unroll
    for (int j = 0; j < kSortItems; ++j) {
        const bool ok = wbase + j * 32 + lane < n;
        const uint32_t dg = (k[j] >> shift) & 255u;
        const unsigned peers = digit_peers(dg, ok);
        const uint32_t c = ok ? wcnt[warp][dg] : 0u;
        __syncwarp();
        if (ok && lane == __ffs(peers) - 1)
            wcnt[warp][dg] = c + (uint32_t)__popc(peers);
        __syncwarp();
        rank[j] = c + (uint32_t)__popc(peers & lanemask_lt());
    }
    __syncthreads();
    {   // per digit: the entries of earlier warps come first
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < kSortThreads / 32; ++w) {
            const uint32_t t = wcnt[w][threadIdx.x];
            wcnt[w][threadIdx.x] = run;
            run += t;
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kSortItems; ++j) {
        if (wbase + j * 32 + lane < n) {
            const uint32_t dg = (k[j] >> shift) & 255u;
            const uint32_t pos = digit_base[dg] + wcnt[warp][dg] + rank[j];
            keys_out[pos] = k[j];
            bags_out[pos] = v[j];
        }
    }
}

// ---------------------------------------------------------------------------
// reductions
// ---------------------------------------------------------------------------

// The lane's EPL elements [lane * EPL, lane * EPL + EPL) of a binary32 row (0 past d).
template <int EPL, bool VEC>
__device__ __forceinline__ void load_elems(const float *row, int lane, int d, float (&v)[EPL])
{
    const int k0 = lane * EPL;
    if constexpr (VEC) {
#pragma unroll
        for (int e = 0; e < EPL; e += 4) {
            const float4 q = k0 + e < d ? __ldg(reinterpret_cast<const float4 *>(row + k0 + e))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            v[e] = q.x;
            v[e + 1] = q.y;
            v[e + 2] = q.z;
            v[e + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e)
            v[e] = k0 + e < d ? __ldg(row + k0 + e) : 0.0f;
    }
}

// Lists a finished row: its key and G = the binary64 sum rounded once to binary32.
template <int EPL>
__device__ __forceinline__ void list_row(const BwdArgs &a, uint32_t slot, uint32_t key, const double (&s)[EPL],
                                         int lane)
{
    if (lane == 0)
        a.list[slot] = key;
    float *gr = a.grad_rows + (int64_t)slot * a.grad_ld + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e)
        if (lane * EPL + e < a.d)
            gr[e] = (float)s[e];
}

// Window j covers sorted entries [64 j, 64 j + 64). Lane l holds entries l and l + 32.
// Each block takes 8 consecutive windows per iteration (one per warp) and draws list
// slots for all of them with one atomic.
template <int EPL, bool VEC>
__global__ void __launch_bounds__(kRedThreads) bwd_window_kernel(const BwdArgs a)
{
    __shared__ uint32_t warp_cnt[kRedThreads / 32];
    __shared__ uint32_t block_slot;
    if (*(volatile uint32_t *)a.hdr)
        return;
    const uint32_t sent = a.key_base[a.T];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t *keys = a.keys[0];
    const int32_t *bags = a.bags[0];
    const int64_t windows = (a.n + kWin - 1) / kWin;
    const int64_t row_len = (int64_t)a.T * a.d;
    for (int64_t jb = (int64_t)blockIdx.x * (kRedThreads / 32); jb < windows; jb += (int64_t)gridDim.x * (kRedThreads / 32)) {
        const int64_t j = jb + warp;
        const bool live = j < windows;  // block-uniform loop; a warp past the end only joins the barriers
        const int64_t w0 = j * kWin;
        const int cnt = live ? (int)(a.n - w0 < kWin ? a.n - w0 : kWin) : 0;
        const uint32_t k_lo = lane < cnt ? __ldg(keys + w0 + lane) : sent;
        const uint32_t k_hi = lane + 32 < cnt ? __ldg(keys + w0 + 32 + lane) : sent;
        const int32_t g_lo = lane < cnt ? __ldg(bags + w0 + lane) : 0;
        const int32_t g_hi = lane + 32 < cnt ? __ldg(bags + w0 + 32 + lane) : 0;
        const uint32_t k_prev = live && j > 0 ? __ldg(keys + w0 - 1) : sent;
        const uint32_t k_next = live && w0 + kWin < a.n ? __ldg(keys + w0 + kWin) : sent;
        // neighbours of both entries of the lane
        const uint32_t up_lo = __shfl_up_sync(0xffffffffu, k_lo, 1), up_hi = __shfl_up_sync(0xffffffffu, k_hi, 1);
        const uint32_t dn_lo = __shfl_down_sync(0xffffffffu, k_lo, 1), dn_hi = __shfl_down_sync(0xffffffffu, k_hi, 1);
        const uint32_t lo31 = __shfl_sync(0xffffffffu, k_lo, 31), hi0 = __shfl_sync(0xffffffffu, k_hi, 0);
        const uint32_t prev_lo = lane == 0 ? k_prev : up_lo, prev_hi = lane == 0 ? lo31 : up_hi;
        const uint32_t next_lo = lane == 31 ? hi0 : dn_lo, next_hi = lane == 31 ? k_next : dn_hi;
        (void)prev_lo;
        (void)prev_hi;
        // a row is finished here when its last entry is here and it did not start before the window
        const bool fin_lo = k_lo != sent && k_lo != next_lo && k_lo != k_prev;
        const bool fin_hi = k_hi != sent && k_hi != next_hi && k_hi != k_prev;
        const unsigned b_lo = __ballot_sync(0xffffffffu, fin_lo), b_hi = __ballot_sync(0xffffffffu, fin_hi);
        const uint32_t n_fin = (uint32_t)(__popc(b_lo) + __popc(b_hi));
        if (lane == 0)
            warp_cnt[warp] = n_fin;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t tot = 0;
            for (int w = 0; w < kRedThreads / 32; ++w)
                tot += warp_cnt[w];
            block_slot = tot ? atomicAdd(a.hdr + 1, tot) : 0u;
        }
        __syncthreads();
        uint32_t slot = block_slot;
        for (int w = 0; w < warp; ++w)
            slot += warp_cnt[w];
        __syncthreads();  // warp_cnt and block_slot are rewritten next iteration
        if (!live)
            continue;

        double acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e)
            acc[e] = 0.0;
        bool from_before = true;  // the current part began at the window's first entry
        constexpr int U = EPL <= 4 ? 8 : (EPL <= 8 ? 4 : 2);
        for (int i0 = 0; i0 < cnt; i0 += U) {
            // gather U entries and issue their gradient loads before any add
            float gv[U][EPL];
            uint32_t kk[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u;
                const uint32_t ksrc = i < 32 ? k_lo : k_hi;
                const int32_t gsrc = i < 32 ? g_lo : g_hi;
                kk[u] = __shfl_sync(0xffffffffu, ksrc, i & 31);
                const int32_t g = __shfl_sync(0xffffffffu, gsrc, i & 31);
                const bool ok = i < cnt && kk[u] != sent;
                const int t = (int)div_batch((uint32_t)g, a.div);
                const int64_t b = (int64_t)g - (int64_t)t * a.batch;
                const float *row = a.grad + b * row_len + (int64_t)t * a.d;
                if (ok)
                    load_elems<EPL, VEC>(row, lane, a.d, gv[u]);
                else {
#pragma unroll
                    for (int e = 0; e < EPL; ++e)
                        gv[u][e] = 0.0f;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u;
                if (i >= cnt || kk[u] == sent)
                    break;  // uniform: the sentinel entries come last
#pragma unroll
                for (int e = 0; e < EPL; ++e)
                    acc[e] = acc[e] + (double)gv[u][e];
                const uint32_t nsrc = i < 32 ? next_lo : next_hi;
                const uint32_t knext = __shfl_sync(0xffffffffu, nsrc, i & 31);
                const bool part_end = knext != kk[u] || i == cnt - 1;
                if (!part_end)
                    continue;
                const bool began_before = from_before && kk[u] == k_prev;
                const bool goes_on = knext == kk[u];  // only at the window's last entry
                if (!began_before && !goes_on) {
                    list_row<EPL>(a, slot, kk[u], acc, lane);
                    ++slot;
                } else {
                    // the row's part: slot 1 = the part of the window where it starts,
                    // slot 0 = a part that began in an earlier window
                    const int which = began_before ? 0 : 1;
                    double *pp = a.partials + ((j * 2 + which) * (int64_t)a.d) + lane * EPL;
#pragma unroll
                    for (int e = 0; e < EPL; ++e)
                        if (lane * EPL + e < a.d)
                            pp[e] = acc[e];
                }
#pragma unroll
                for (int e = 0; e < EPL; ++e)
                    acc[e] = 0.0;
                from_before = false;
            }
        }
    }
}

// Rows spanning windows: found at the window where they end (their first entry of
// the window continues the previous window's last row, and they end inside it).
template <int EPL>
__global__ void __launch_bounds__(kRedThreads) bwd_span_kernel(const BwdArgs a)
{
    if (*(volatile uint32_t *)a.hdr)
        return;
    const uint32_t sent = a.key_base[a.T];
    const int lane = threadIdx.x & 31;
    const uint32_t *keys = a.keys[0];
    const int64_t windows = (a.n + kWin - 1) / kWin;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t j = 1 + warp0; j < windows; j += warps) {
        const int64_t w0 = j * kWin;
        const uint32_t k0 = __ldg(keys + w0);
        if (k0 == sent || __ldg(keys + w0 - 1) != k0)
            continue;
        const int cnt = (int)(a.n - w0 < kWin ? a.n - w0 : kWin);
        const bool other_lo = lane < cnt && __ldg(keys + w0 + lane) != k0;
        const bool other_hi = lane + 32 < cnt && __ldg(keys + w0 + 32 + lane) != k0;
        const bool ends_inside = __any_sync(0xffffffffu, other_lo || other_hi);
        if (!ends_inside && cnt == kWin && w0 + kWin < a.n && __ldg(keys + w0 + kWin) == k0)
            continue;  // the row goes on into the next window
        // first entry of the row: lower bound of k0 in [0, w0)
        int64_t lo = 0, hi = w0;
        while (lo < hi) {
            const int64_t mid = (lo + hi) >> 1;
            if (__ldg(keys + mid) < k0)
                lo = mid + 1;
            else
                hi = mid;
        }
        const int64_t j0 = lo / kWin;
        double s[EPL];
        {
            const double *p = a.partials + (j0 * 2 + 1) * (int64_t)a.d + lane * EPL;
#pragma unroll
            for (int e = 0; e < EPL; ++e)
                s[e] = lane * EPL + e < a.d ? p[e] : 0.0;
        }
        for (int64_t jj = j0 + 1; jj <= j; ++jj) {
            const double *p = a.partials + (jj * 2) * (int64_t)a.d + lane * EPL;
#pragma unroll
            for (int e = 0; e < EPL; ++e)
                s[e] = s[e] + (lane * EPL + e < a.d ? p[e] : 0.0);
        }
        uint32_t slot = 0;
        if (lane == 0)
            slot = atomicAdd(a.hdr + 1, 1u);
        slot = __shfl_sync(0xffffffffu, slot, 0);
        list_row<EPL>(a, slot, k0, s, lane);
    }
}

template <int EPL>
cudaError_t launch_reduce(const BwdArgs &a, int num_sms, cudaStream_t stream)
{
    const int64_t windows = (a.n + kWin - 1) / kWin;
    const int64_t blocks = (windows + kRedThreads / 32 - 1) / (kRedThreads / 32);
    const int64_t cap = (int64_t)num_sms * 8;
    const unsigned grid = (unsigned)(blocks < cap ? blocks : cap);
    const bool vec = EPL >= 4 && a.d % 4 == 0 && ((int64_t)a.T * a.d) % 4 == 0 &&
                     (reinterpret_cast<uintptr_t>(a.grad) & 15) == 0;
    if (vec) {
        if constexpr (EPL >= 4)
            bwd_window_kernel<EPL, true><<<grid, kRedThreads, 0, stream>>>(a);
    } else {
        bwd_window_kernel<EPL, false><<<grid, kRedThreads, 0, stream>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    if (windows > 1)
        bwd_span_kernel<EPL><<<grid, kRedThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

size_t align256(size_t x)
{
    return (x + 255) & ~(size_t)255;
}

} // namespace

BwdLayout bwd_layout(int64_t n, int d)
{
    BwdLayout L{};
    L.tiles = (n + kTile - 1) / kTile;
    L.windows = (n + kWin - 1) / kWin;
    L.grad_ld = (d + 3) / 4 * 4;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align256(bytes);
        return at;
    };
    L.hdr = take(256);
    L.keys0 = take((size_t)n * 4);
    L.keys1 = take((size_t)n * 4);
    L.bags0 = take((size_t)n * 4);
    L.bags1 = take((size_t)n * 4);
    L.hist = take((size_t)kDigits * (size_t)L.tiles * 4);
    L.totals = take((size_t)kDigits * 4);
    L.partials = take((size_t)L.windows * 2 * (size_t)d * 8);
    L.list = take((size_t)n * 4);
    L.grad_rows = take((size_t)n * (size_t)L.grad_ld * 4);
    L.total = off;
    return L;
}

// Sorts the entries (result in keys[0]/bags[0]) and reduces every row's gradient.
cudaError_t launch_bwd_sort_reduce(BwdArgs &a, int num_sms, cudaStream_t stream)
{
    const int64_t G = (int64_t)a.T * a.batch;
    {
        const int64_t need = (G + 255) / 256;
        const int64_t cap = (int64_t)num_sms * 16;
        bwd_keys_kernel<<<(unsigned)(need < cap ? need : cap), 256, 0, stream>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
    }
    // digits needed for keys 0..total (the total marks invalid entries)
    const uint32_t sentinel = a.key_base[a.T];
    int bits = 1;
    while (bits < 32 && (sentinel >> bits) != 0)
        ++bits;
    const int64_t tiles = (a.n + kTile - 1) / kTile;
    for (int shift = 0; shift < bits; shift += 8) {
        radix_hist_kernel<<<(unsigned)tiles, kSortThreads, 0, stream>>>(a.keys[0], a.n, shift, a.hist, tiles);
        radix_scan_kernel<<<kDigits, kSortThreads, 0, stream>>>(a.hist, tiles, a.totals);
        radix_scatter_kernel<<<(unsigned)tiles, kSortThreads, 0, stream>>>(a.keys[0], a.bags[0], a.keys[1], a.bags[1],
                                                                           a.n, shift, a.hist, a.totals, tiles);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess)
            return e;
        uint32_t *tk = a.keys[0];
        a.keys[0] = a.keys[1];
        a.keys[1] = tk;
        int32_t *tb = a.bags[0];
        a.bags[0] = a.bags[1];
        a.bags[1] = tb;
    }
    int epl = 1;
    while (epl * 32 < a.d)
        epl <<= 1;
    switch (epl) {
    case 1: return launch_reduce<1>(a, num_sms, stream);
    case 2: return launch_reduce<2>(a, num_sms, stream);
    case 4: return launch_reduce<4>(a, num_sms, stream);
    case 8: return launch_reduce<8>(a, num_sms, stream);
    case 16: return launch_reduce<16>(a, num_sms, stream);
    case 32: return launch_reduce<32>(a, num_sms, stream);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace dq
