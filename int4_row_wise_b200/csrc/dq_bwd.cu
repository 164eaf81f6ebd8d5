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
// scheduling, so the updated masters and their codes are reproducible. It is the
// binary64 sum of the row's entries in list order, associated by windows: it can
// differ from the plain sequential binary64 sum rounded once only where that sum lies
// within binary64 rounding error of a binary32 rounding boundary (one ulp then).
//
// Kernels, in stream order:
//   bwd_keys_kernel      one lane (or warp) per bag: writes (key, bag) of its entries;
//                        checks that offsets are a CSR array (else nothing changes)
//   radix_hist_kernel    LSD radix sort, 8-bit digits, ceil(bits(total rows) / 8)
//   radix_scan_kernel    passes of three kernels each: per-tile digit counts,
//   radix_scatter_kernel their digit-major exclusive scan, and a stable scatter
//                        (warp-striped tiles ranked with ballots, no atomics)
//   bwd_window_kernel    blocks take chunks of up to 8 windows (one atomic for the
//                        chunk's list slots); a warp sums whole windows, EPL elements
//                        per lane, the gradient rows staged in shared memory by
//                        cp.async in double-buffered 4 KB stages; it lists every row
//                        that ends in the window (with its G when the row lies wholly
//                        inside it); a row crossing a window edge leaves a binary64 part
//   bwd_span_kernel      one warp per (spanning row, 32 elements): adds its parts in
//                        window order, 32 parts prefetched to shared memory at a time
// Every loop is bounded by sizes known at launch; no kernel waits on another.
#include "dq_internal.cuh"

namespace dq {
namespace {

constexpr int kWin = 64;                          // entries per window of the sorted list
constexpr int kSortThreads = 256;
constexpr int kSortItems = 8;
constexpr int kTile = kSortThreads * kSortItems;  // entries per sort tile
constexpr int kDigits = 256;

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

// One lane per bag (short bags) or one warp per bag (WARP: bags of 8 or more ids on
// average, so the reads of indices and the writes of the entries are coalesced).
template <bool WARP>
__global__ void __launch_bounds__(256) bwd_keys_kernel(const BwdArgs a)
{
    const int64_t G = (int64_t)a.T * a.batch;
    const uint32_t sentinel = a.key_base[a.T];
    bool bad = false, bad_id = false;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per = WARP ? 32 : 1;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x / per;
    const int lane = WARP ? (int)(threadIdx.x & 31) : 0;
    for (int64_t g = tid / per; g < G; g += stride) {
        int64_t p0 = a.offsets[g], p1 = a.offsets[g + 1];
        bad |= p1 < p0;
        p0 = p0 < 0 ? 0 : (p0 > a.n ? a.n : p0);  // keep every write inside the entry arrays
        p1 = p1 < p0 ? p0 : (p1 > a.n ? a.n : p1);
        const int t = (int)div_batch((uint32_t)g, a.div);
        const uint32_t base = a.key_base[t], rows = a.key_base[t + 1] - base;
        for (int64_t p = p0 + lane; p < p1; p += per) {
            const int32_t id = __ldg(a.indices + p);
            const bool ok = id >= 0 && (uint32_t)id < rows;
            bad_id |= !ok;
            a.keys[0][p] = ok ? base + (uint32_t)id : sentinel;
            a.bags[0][p] = (int32_t)g;
        }
    }
    if (tid == 0)
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

constexpr uint32_t kNoSpan = 0xffffffffu;

constexpr int kWinWarps = 4;      // warps per block in bwd_window_kernel
constexpr int kChunk = 8;         // at most this many windows per block iteration
constexpr int kStageFloats = 1024; // 4 KB per stage: 32 / EPL rows (at least 1) of 32 * EPL floats

// L2 policy for the gradient rows: keep them (every bag's row is read once per id of
// the bag), while the G rows and parts written alongside stream past (st.global.cs).
__device__ __forceinline__ uint64_t evict_last_policy()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint64_t policy)
{
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "l"(policy));
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src, uint64_t policy)
{
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 4, %2;\n" ::"r"(d), "l"(src), "l"(policy));
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// Issues the cp.async copies of rows [r0, r0 + rows) of a window (row pointers in rp,
// NULL = skip; d elements each) into a stage of rows of 32 * EPL floats, and commits
// them as one group. VEC: 16-byte pieces (d % 4 == 0 and rows 16-byte aligned).
template <int EPL, bool VEC>
__device__ __forceinline__ void issue_stage(float *stage, const float *const *rp, int r0, int rows, int d, int lane,
                                            uint64_t policy)
{
    constexpr int ROW = 32 * EPL;
    const int piece = VEC ? 4 : 1;
    const int cpr = (d + piece - 1) / piece;  // copies per row
    if (cpr <= 32) {
        const int rpi = 32 / cpr;             // rows per pass of the warp
        const int sub = lane / cpr, col = lane - sub * cpr;
        if (sub < rpi) {
            for (int r = sub; r < rows; r += rpi) {
                const float *src = rp[r0 + r];
                if (src) {
                    if (VEC)
                        cp_async16(stage + r * ROW + col * 4, src + col * 4, policy);
                    else
                        cp_async4(stage + r * ROW + col, src + col, policy);
                }
            }
        }
    } else {
        for (int r = 0; r < rows; ++r) {
            const float *src = rp[r0 + r];
            if (!src)
                continue;
            for (int col = lane; col < cpr; col += 32) {
                if (VEC)
                    cp_async16(stage + r * ROW + col * 4, src + col * 4, policy);
                else
                    cp_async4(stage + r * ROW + col, src + col, policy);
            }
        }
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

// Blocks take chunks of up to 8 consecutive windows (window j = sorted entries
// [64 j, 64 j + 64)). Per chunk, the block reads the windows' keys into shared
// memory, finds each entry's gradient row, and counts the rows whose last entry lies
// in each window, drawing their list slots with one atomic. Each warp then takes
// whole windows. Lane l owns elements [l * EPL, l * EPL + EPL) of the rows: EPL
// independent binary64 chains. The window's gradient rows are copied to shared
// memory in stages of 32 / EPL rows (4 KB; the next stage's copies are issued before
// the current one is summed), and the warp walks the window's parts (runs of one
// row): a part's entries are added in order from +0. A row whose entries all lie in
// the window is listed with its G; a row that ends here but began earlier is listed
// too, its G left to bwd_span_kernel (span_slot[j]); a row's part that does not
// finish it is stored in partials.
template <int EPL, bool VEC>
__global__ void __launch_bounds__(kWinWarps * 32) bwd_window_kernel(const BwdArgs a, const int chunk)
{
    constexpr int ROW = 32 * EPL;
    constexpr int SR = kStageFloats / ROW;  // rows per stage, divides 64
    extern __shared__ __align__(16) float stage_all[];  // [warps][2][kStageFloats]
    __shared__ const float *rp[kChunk][kWin];
    __shared__ uint32_t ks[kChunk][kWin + 2];            // the window's keys, then the ones before and after
    __shared__ uint32_t n_end[kChunk], slot_base[kChunk];
    if (*(volatile uint32_t *)a.hdr)
        return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    float *stage2 = stage_all + (size_t)warp * 2 * kStageFloats;
    const uint64_t policy = evict_last_policy();
    const uint32_t sent = a.key_base[a.T];
    const uint32_t *keys = a.keys[0];
    const int32_t *bags = a.bags[0];
    const int64_t windows = (a.n + kWin - 1) / kWin;
    const int64_t row_len = (int64_t)a.T * a.d;
    const int k0 = lane * EPL;
    for (int64_t c0 = (int64_t)blockIdx.x * chunk; c0 < windows; c0 += (int64_t)gridDim.x * chunk) {
        const int nw = windows - c0 < chunk ? (int)(windows - c0) : chunk;
        for (int cw = warp; cw < nw; cw += nwarps) {
            const int64_t j = c0 + cw, w0 = j * kWin;
            const int cnt = (int)(a.n - w0 < kWin ? a.n - w0 : kWin);
            const uint32_t k_lo = lane < cnt ? __ldg(keys + w0 + lane) : sent;
            const uint32_t k_hi = lane + 32 < cnt ? __ldg(keys + w0 + 32 + lane) : sent;
            const uint32_t k_next = w0 + kWin < a.n ? __ldg(keys + w0 + kWin) : sent;
            ks[cw][lane] = k_lo;
            ks[cw][lane + 32] = k_hi;
            if (lane == 0) {
                ks[cw][kWin] = j > 0 ? __ldg(keys + w0 - 1) : sent;
                ks[cw][kWin + 1] = k_next;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t key = h ? k_hi : k_lo;
                const float *row = nullptr;
                if (key != sent) {
                    const int32_t g = __ldg(bags + w0 + lane + 32 * h);
                    const int t = (int)div_batch((uint32_t)g, a.div);
                    row = a.grad + ((int64_t)g - (int64_t)t * a.batch) * row_len + (int64_t)t * a.d;
                }
                rp[cw][lane + 32 * h] = row;
            }
            const uint32_t dn_lo = __shfl_down_sync(0xffffffffu, k_lo, 1), dn_hi = __shfl_down_sync(0xffffffffu, k_hi, 1);
            const uint32_t hi0 = __shfl_sync(0xffffffffu, k_hi, 0);
            const uint32_t next_lo = lane == 31 ? hi0 : dn_lo, next_hi = lane == 31 ? k_next : dn_hi;
            const bool end_lo = k_lo != sent && k_lo != next_lo, end_hi = k_hi != sent && k_hi != next_hi;
            const int ends = __popc(__ballot_sync(0xffffffffu, end_lo)) + __popc(__ballot_sync(0xffffffffu, end_hi));
            if (lane == 0)
                n_end[cw] = (uint32_t)ends;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t tot = 0;
            for (int cw = 0; cw < nw; ++cw) {
                slot_base[cw] = tot;
                tot += n_end[cw];
            }
            const uint32_t base = tot ? atomicAdd(a.hdr + 1, tot) : 0u;
            for (int cw = 0; cw < nw; ++cw)
                slot_base[cw] += base;
        }
        __syncthreads();
        // this warp's stages: windows warp, warp + nwarps, ... of the chunk, 64 / SR each
        auto win_cnt = [&](int cw) { return (int)(a.n - (c0 + cw) * kWin < kWin ? a.n - (c0 + cw) * kWin : kWin); };
        int buf = 0;
        if (warp < nw) {
            const int c = win_cnt(warp);
            issue_stage<EPL, VEC>(stage2, rp[warp], 0, c < SR ? c : SR, a.d, lane, policy);
        }
        for (int cw = warp; cw < nw; cw += nwarps) {
            const int64_t j = c0 + cw;
            const int cnt = win_cnt(cw);
            const uint32_t k_lo = ks[cw][lane], k_hi = ks[cw][lane + 32];
            const uint32_t k_prev = ks[cw][kWin], k_next = ks[cw][kWin + 1];
            const uint32_t nx_lo = ks[cw][lane + 1];
            const uint32_t nx_hi = lane == 31 ? k_next : ks[cw][lane + 33];
            // valid entries form a prefix (invalid ones sort last); part ends as a mask
            const unsigned v_lo = __ballot_sync(0xffffffffu, k_lo != sent), v_hi = __ballot_sync(0xffffffffu, k_hi != sent);
            const int nv = __popc(v_lo) + __popc(v_hi);
            uint64_t ends = (uint64_t)__ballot_sync(0xffffffffu, k_lo != sent && k_lo != nx_lo) |
                            ((uint64_t)__ballot_sync(0xffffffffu, k_hi != sent && k_hi != nx_hi) << 32);
            if (nv == cnt && nv > 0)
                ends |= 1ull << (nv - 1);  // the window's last entry ends a part even if its row goes on
            uint32_t slot = slot_base[cw], span_slot = kNoSpan;
            double acc[EPL];
#pragma unroll
            for (int e = 0; e < EPL; ++e)
                acc[e] = 0.0;
            int i = 0;  // next entry to add
            bool first_part = true;
            for (int s0 = 0; s0 < cnt; s0 += SR, buf ^= 1) {
                // the stage after this one (this window's next, or the warp's next window's first)
                const int ns0 = s0 + SR;
                const bool more_here = ns0 < cnt;
                const int ncw = cw + nwarps;
                if (more_here) {
                    issue_stage<EPL, VEC>(stage2 + (buf ^ 1) * kStageFloats, rp[cw], ns0,
                                          cnt - ns0 < SR ? cnt - ns0 : SR, a.d, lane, policy);
                    asm volatile("cp.async.wait_group 1;\n" ::: "memory");
                } else if (ncw < nw) {
                    const int c = win_cnt(ncw);
                    issue_stage<EPL, VEC>(stage2 + (buf ^ 1) * kStageFloats, rp[ncw], 0, c < SR ? c : SR, a.d, lane,
                                          policy);
                    asm volatile("cp.async.wait_group 1;\n" ::: "memory");
                } else {
                    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
                }
                __syncwarp();
                const float *stage = stage2 + buf * kStageFloats + k0;
                const int s1 = s0 + SR < nv ? s0 + SR : nv;  // entries of this stage to add
                while (i < s1) {
                    const int e_end = ends ? __ffsll((long long)ends) - 1 : kWin;
                    const int stop = e_end < s1 ? e_end + 1 : s1;
                    for (; i < stop; ++i) {
                        const float *v = stage + (i - s0) * ROW;
                        if constexpr (EPL >= 4) {
#pragma unroll
                            for (int e = 0; e < EPL; e += 4) {
                                const float4 q = *reinterpret_cast<const float4 *>(v + e);
                                acc[e] = acc[e] + (double)q.x;
                                acc[e + 1] = acc[e + 1] + (double)q.y;
                                acc[e + 2] = acc[e + 2] + (double)q.z;
                                acc[e + 3] = acc[e + 3] + (double)q.w;
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < EPL; ++e)
                                acc[e] = acc[e] + (double)v[e];
                        }
                    }
                    if (stop != e_end + 1)
                        break;  // the part goes on into the next stage
                    ends &= ends - 1;
                    const uint32_t key = ks[cw][e_end];
                    const bool began_before = first_part && key == k_prev;
                    const bool goes_on = e_end == kWin - 1 && key == k_next;
                    if (!began_before && !goes_on) {
                        if (lane == 0)
                            a.list[slot] = key;
                        float *gr = a.grad_rows + (int64_t)slot * a.grad_ld + k0;
#pragma unroll
                        for (int e = 0; e < EPL; ++e)
                            if (k0 + e < a.d)
                                __stcs(gr + e, (float)acc[e]);
                        ++slot;
                    } else {
                        // slot 1 = the part of the window where the row starts,
                        // slot 0 = a part of a row that began in an earlier window
                        const int which = began_before ? 0 : 1;
                        double *pp = a.partials + (j * 2 + which) * (int64_t)a.d + k0;
#pragma unroll
                        for (int e = 0; e < EPL; ++e)
                            if (k0 + e < a.d)
                                __stcs(pp + e, acc[e]);
                        if (began_before && !goes_on) {
                            if (lane == 0)
                                a.list[slot] = key;
                            span_slot = slot++;
                        }
                    }
#pragma unroll
                    for (int e = 0; e < EPL; ++e)
                        acc[e] = 0.0;
                    first_part = false;
                }
                __syncwarp();  // this stage is refilled two stages on
            }
            if (lane == 0)
                a.span_slot[j] = span_slot;
        }
        __syncthreads();  // rp, ks, n_end and slot_base are rewritten for the next chunk
    }
}

// G of the rows that span windows, listed by bwd_window_kernel at the window where
// they end: the parts in window order, summed in binary64. One warp per (window,
// 32-element slice of the row), one element per lane; the parts of 32 windows at a
// time are copied to shared memory first (cp.async), so their loads are all in flight.
constexpr int kSpanWarps = 4;
constexpr int kSpanAhead = 32;

__device__ __forceinline__ void cp_async8(void *dst, const void *src)
{
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(d), "l"(src));
}

__global__ void __launch_bounds__(kSpanWarps * 32) bwd_span_kernel(const BwdArgs a)
{
    __shared__ double ahead[kSpanWarps][kSpanAhead][32];
    if (*(volatile uint32_t *)a.hdr)
        return;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t *keys = a.keys[0];
    const int64_t windows = (a.n + kWin - 1) / kWin;
    const int slices = (a.d + 31) / 32;
    const int64_t items = windows * slices;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t it = warp0; it < items; it += warps) {
        const int64_t j = it / slices;
        const int slice = (int)(it - j * slices);
        const uint32_t slot = __ldg(a.span_slot + j);
        if (slot == kNoSpan)
            continue;
        // the row's first entry: keys[64 j - 1] == keys[64 j] == k0; gallop back, then bisect
        const int64_t w0 = j * kWin;
        const uint32_t k0 = __ldg(keys + w0);
        int64_t hi = w0 - 1, step = kWin, lo = hi - step;
        while (lo >= 0 && __ldg(keys + lo) == k0) {
            hi = lo;
            step *= 2;
            lo = hi - step;
        }
        if (lo < -1)
            lo = -1;
        while (hi - lo > 1) {  // keys[lo] < k0 (or lo == -1), keys[hi] == k0
            const int64_t mid = (lo + hi) >> 1;
            if (__ldg(keys + mid) == k0)
                hi = mid;
            else
                lo = mid;
        }
        const int64_t j0 = hi / kWin;
        const int k = slice * 32 + lane;
        const bool ok = k < a.d;
        double s = ok ? a.partials[(j0 * 2 + 1) * (int64_t)a.d + k] : 0.0;
        for (int64_t jb = j0 + 1; jb <= j; jb += kSpanAhead) {
            const int m = j - jb + 1 < kSpanAhead ? (int)(j - jb + 1) : kSpanAhead;
            if (ok)
                for (int u = 0; u < m; ++u)
                    cp_async8(&ahead[warp][u][lane], a.partials + ((jb + u) * 2) * (int64_t)a.d + k);
            cp_async_wait_all();
            for (int u = 0; u < m; ++u)
                s = s + ahead[warp][u][lane];
        }
        if (ok)
            a.grad_rows[(int64_t)slot * a.grad_ld + k] = (float)s;
    }
}

template <int EPL>
cudaError_t launch_window(const BwdArgs &a, int num_sms, cudaStream_t stream)
{
    const int64_t windows = (a.n + kWin - 1) / kWin;
    // chunks of up to 8 windows (about 24 warps per SM: 8 KB of stages per warp),
    // smaller when there are too few windows to fill the GPU
    int chunk = kChunk, wpb = kWinWarps;
    int64_t blocks_wanted = 0;
    for (;; chunk >>= 1) {
        wpb = chunk < kWinWarps ? chunk : kWinWarps;
        blocks_wanted = (int64_t)num_sms * (24 / wpb);
        if (chunk == 1 || (windows + chunk - 1) / chunk >= blocks_wanted)
            break;
    }
    const int64_t chunks = (windows + chunk - 1) / chunk;
    const unsigned grid = (unsigned)(chunks < blocks_wanted ? chunks : blocks_wanted);
    const size_t smem = (size_t)wpb * 2 * kStageFloats * sizeof(float);
    const bool vec = a.d % 4 == 0 && ((int64_t)a.T * a.d) % 4 == 0 && (reinterpret_cast<uintptr_t>(a.grad) & 15) == 0;
    cudaError_t e;
    if (vec) {
        e = cudaFuncSetAttribute(bwd_window_kernel<EPL, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            bwd_window_kernel<EPL, true><<<grid, wpb * 32, smem, stream>>>(a, chunk);
    } else {
        e = cudaFuncSetAttribute(bwd_window_kernel<EPL, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            bwd_window_kernel<EPL, false><<<grid, wpb * 32, smem, stream>>>(a, chunk);
    }
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

cudaError_t launch_reduce(const BwdArgs &a, int num_sms, cudaStream_t stream)
{
    int epl = 1;
    while (epl * 32 < a.d)
        epl <<= 1;
    cudaError_t e;
    switch (epl) {
    case 1: e = launch_window<1>(a, num_sms, stream); break;
    case 2: e = launch_window<2>(a, num_sms, stream); break;
    case 4: e = launch_window<4>(a, num_sms, stream); break;
    case 8: e = launch_window<8>(a, num_sms, stream); break;
    case 16: e = launch_window<16>(a, num_sms, stream); break;
    case 32: e = launch_window<32>(a, num_sms, stream); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess)
        return e;
    const int64_t windows = (a.n + kWin - 1) / kWin;
    if (windows > 1) {
        const int64_t items = windows * ((a.d + 31) / 32);
        const int64_t need = (items + kSpanWarps - 1) / kSpanWarps;
        const int64_t cap2 = (int64_t)num_sms * 16;
        bwd_span_kernel<<<(unsigned)(need < cap2 ? need : cap2), kSpanWarps * 32, 0, stream>>>(a);
    }
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
    L.span_slot = take((size_t)L.windows * 4);
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
        const bool warp_per_bag = a.n >= 8 * G;
        const int64_t need = warp_per_bag ? (G * 32 + 255) / 256 : (G + 255) / 256;
        const int64_t cap = (int64_t)num_sms * 16;
        const unsigned grid = (unsigned)(need < cap ? need : cap);
        if (warp_per_bag)
            bwd_keys_kernel<true><<<grid, 256, 0, stream>>>(a);
        else
            bwd_keys_kernel<false><<<grid, 256, 0, stream>>>(a);
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
    return launch_reduce(a, num_sms, stream);
}

} // namespace dq
