// dq_quantize.cu -- greedy row-wise INT4 quantization on sm_100a.
//
// "Post-Training 4-bit Quantization on Embedding Tables" (Guan et al., 2019), review
// page, section 提出的方法 (proposed method): a uniform 4-bit quantizer per row whose
// clipping thresholds come from a greedy search toward a local minimum of the
// squared error (bullet 1), with the scale and bias stored as FP16 (bullet 2).
// The grid (200 steps), the stop (width <= 0.16 * range, i.e. 168 moves), the
// tie rules and the rounding of every step are the ones dq.h states.
//
// Layout: a row of d <= P = next_pow2(d) elements is held in registers by W lanes
// of one warp, M = P / W contiguous elements per lane (M = 16 for P >= 16). The
// search is pure FP32 ALU work: 337 loss evaluations x d elements per row. The two
// candidates of a move are evaluated side by side (ILP), and the per-element work
// runs on packed f32x2 FMA/ADD/MUL, which issue once for two lanes' worth of FP32
// work: a lane pairs element m with element m + M/2, so the packed adds of the
// error tree are exactly the pairwise (recursive-halving) order, and an XOR
// butterfly over the W lanes finishes it. Every lane of a row gets the identical
// binary32 loss.
//
// Codes during the search: q = clamp(rint((x - lo) / s), 0, 15) needs an IEEE
// quotient. The kernel instead forms u = sat(fma(x, r, -lo*r)) with r = rcp(w),
// w = hi - lo (= 15 s up to one rounding), and rounds 15u with a magic-number add.
// |15u - (x - lo)/s| <= 5.6e-6 + 9e-7 * |lo * r| (rcp error <= 1 ulp), so 15u rounds
// like the IEEE quotient unless both lie within about 6e-6 + 9e-7 K of a
// half-integer (K bounds |lo * r| over the row's walk). Then |e| / s is within about
// that of 1/2 for either code, so an element whose e^2 falls in a narrow window
// around s^2 / 4 (about 3 in 10^5) is recomputed with IEEE division. The codes the
// search sees are therefore exactly the IEEE ones.
//
// s = w / 15 uses Markstein's correction step for a known divisor (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Dev. 34(1), 1990): q0 = w * RN(1/15), rem = fma(-q0, 15, w),
// s = fma(rem, RN(1/15), q0). It equals the IEEE quotient for every positive
// normal binary32 w (checked exhaustively); the fast path only uses w >= 1e-36.
#include <cfloat>

#include "dq_internal.cuh"

namespace dq {
namespace {

constexpr float kSteps = 200.0f;         // grid steps over the row's range
constexpr int kMoves = 168;              // moves while width > 0.16 * range
constexpr float kLevels = 15.0f;         // 2^4 - 1
constexpr float kMagic = 12582912.0f;    // 1.5 * 2^23: x + kMagic rounds x in [0, 2^22) to an integer
constexpr float kInv15 = 1.0f / 15.0f;   // RN(1/15)
constexpr float kFastWMin = 1.0e-36f;    // w in [kFastWMin, kFastWMax]: s normal, 1/w normal
constexpr float kFastWMax = 1.0e36f;
constexpr float kFastLoR = 65536.0f;     // |lo * r| above this: IEEE path

__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float fma_sat(float a, float b, float c)
{
    float r;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// w / 15 rounded to nearest even, for positive normal w (Markstein correction).
__device__ __forceinline__ float div15(float w)
{
    const float q0 = __fmul_rn(w, kInv15);
    const float rem = __fmaf_rn(-q0, kLevels, w);
    return __fmaf_rn(rem, kInv15, q0);
}

// q = clamp(rint(fl(fl(x - lo) / s)), 0, 15) with an IEEE quotient; 0 when s == 0.
__device__ __forceinline__ float exact_code(float x, float lo, float s)
{
    if (s == 0.0f)
        return 0.0f;
    float q = rintf(__fdiv_rn(__fsub_rn(x, lo), s));
    return fminf(fmaxf(q, 0.0f), kLevels);
}

// Sum over the W lanes of a row (the whole warp takes every shuffle: the walk's path
// is chosen per warp, see quantize_one).
template <int W>
__device__ __forceinline__ float row_sum(float v)
{
#pragma unroll
    for (int o = 1; o < W; o <<= 1)
        v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int W>
__device__ __forceinline__ void row_minmax(float &mn, float &mx)
{
#pragma unroll
    for (int o = 1; o < W; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
}

// One clip range [lo, hi] of the search, with what its elements share.
struct Clip {
    float lo, s;            // bias and scale of the candidate quantizer
    float r, nlr;           // rcp(hi - lo) and -RN(lo * r): u = sat(fma(x, r, nlr))
    uint32_t c_lo, c_span;  // e^2 with bits in [c_lo, c_lo + c_span): near a rounding tie
};

// The tie window of a row, as multiples of s^2. With q the division-free code and
// y = (x - lo) / s exactly: |15u - y| <= 3.7e-6 + 8.9e-7 K (the rounding of r, -lo*r,
// u and s; K bounds |lo * r| over the row's walk) and the IEEE quotient is within
// 1.9e-6 of y, so where the two codes differ, |y - q| is within 5.6e-6 + 8.9e-7 K of
// 1/2, and the computed |e| / s within b_min = 6.6e-6 + 1.8e-6 K of 1/2 (the rounding
// of xhat and e adds at most 2^-24 (15 K + 16)). The window uses b = 1.2e-5 + 3e-6 K,
// about 1.7 b_min: e^2 in s^2 [(1/2 - b)^2, (1/2 + b)^2], widened by 1e-6 for the
// rounding of s^2, of the bounds and of e^2.
struct TieWindow {
    float kl, kh;
};

__device__ __forceinline__ TieWindow tie_window(float K)
{
    const float b = __fmaf_rn(K, 3.0e-6f, 1.2e-5f);
    TieWindow t;
    t.kl = __fmul_rn(__fmaf_rn(-b, 1.0f - b, 0.25f), 0.999999f);
    t.kh = __fmul_rn(__fmaf_rn(b, 1.0f + b, 0.25f), 1.000001f);
    return t;
}

__device__ __forceinline__ Clip clip_fast(float lo, float hi, const TieWindow &tw)
{
    Clip c;
    c.lo = lo;
    const float w = __fsub_rn(hi, lo);
    c.r = rcp_approx(w);
    c.nlr = __fmul_rn(-lo, c.r);
    c.s = div15(w);
    const float s2 = __fmul_rn(c.s, c.s);
    c.c_lo = __float_as_uint(__fmul_rn(s2, tw.kl));
    c.c_span = __float_as_uint(__fmul_rn(s2, tw.kh)) - c.c_lo;
    return c;
}

__device__ __forceinline__ float sq_err_exact(float x, float lo, float s)
{
    const float q = exact_code(x, lo, s);
    const float e = __fsub_rn(x, __fmaf_rn(q, s, lo));
    return __fmul_rn(e, e);
}

// Element k of the lane sits in slot .x of pair k (k < H) or slot .y of pair k - H.
template <int H, bool HAS_Y, bool FULL>
__device__ __forceinline__ bool valid_x(int kbase, int h, int d) { return FULL || kbase + h < d; }
template <int H, bool HAS_Y, bool FULL>
__device__ __forceinline__ bool valid_y(int kbase, int h, int d) { return HAS_Y && (FULL || kbase + h + H < d); }

// Squared errors of the lane's elements for one clip (packed f32x2). Sets `hard` if
// an element's code must be recomputed with IEEE division.
template <int H, bool HAS_Y, bool FULL>
__device__ __forceinline__ void errors_packed(const float2 (&xp)[H], const Clip &c, int kbase, int d,
                                              float2 (&C)[H], bool &hard)
{
    const float2 k15 = make_float2(kLevels, kLevels), kmag = make_float2(kMagic, kMagic);
    const float2 km1 = make_float2(-1.0f, -1.0f);
    const float2 ns2 = make_float2(-c.s, -c.s), lo2 = make_float2(c.lo, c.lo);
    // The tie test as the smallest unsigned offset of e^2's bits above c_lo, one fused
    // add-and-min per element (measured 1-3 % faster than or-ing per-element compares;
    // at 32 elements per lane with a ragged row it costs a spill, so that one keeps them)
    constexpr bool kMinChain = H < 16 || FULL;
    uint32_t m0 = 0xffffffffu, m1 = 0xffffffffu;
#pragma unroll
    for (int h = 0; h < H; ++h) {
        const float2 U = make_float2(fma_sat(xp[h].x, c.r, c.nlr), fma_sat(xp[h].y, c.r, c.nlr));
        const float2 Z = __ffma2_rn(U, k15, kmag);     // kMagic + rint(15u)
        const float2 NQ = __ffma2_rn(Z, km1, kmag);    // -q, exact
        const float2 XH = __ffma2_rn(NQ, ns2, lo2);    // q*s + lo, rounded once
        const float2 E = __ffma2_rn(XH, km1, xp[h]);   // x - xhat
        C[h] = __fmul2_rn(E, E);
        if constexpr (kMinChain) {   // one add-and-min per element
            m0 = min(__float_as_uint(C[h].x) - c.c_lo, m0);
            if (HAS_Y)
                m1 = min(__float_as_uint(C[h].y) - c.c_lo, m1);
        } else {
            hard |= __float_as_uint(C[h].x) - c.c_lo < c.c_span;
            if (HAS_Y)
                hard |= __float_as_uint(C[h].y) - c.c_lo < c.c_span;
        }
        if (!valid_x<H, HAS_Y, FULL>(kbase, h, d))
            C[h].x = 0.0f;
        if (!valid_y<H, HAS_Y, FULL>(kbase, h, d))
            C[h].y = 0.0f;
    }
    if constexpr (kMinChain)
        hard |= min(m0, m1) < c.c_span;
}

// Recomputes with IEEE division every element whose fast code was too close to a tie.
template <int H, bool HAS_Y, bool FULL>
__device__ __forceinline__ void errors_fixup(const float2 (&xp)[H], const Clip &c, int kbase, int d,
                                             float2 (&C)[H])
{
#pragma unroll
    for (int h = 0; h < H; ++h) {
        if (valid_x<H, HAS_Y, FULL>(kbase, h, d) && __float_as_uint(C[h].x) - c.c_lo < c.c_span)
            C[h].x = sq_err_exact(xp[h].x, c.lo, c.s);
        if (valid_y<H, HAS_Y, FULL>(kbase, h, d) && __float_as_uint(C[h].y) - c.c_lo < c.c_span)
            C[h].y = sq_err_exact(xp[h].y, c.lo, c.s);
    }
}

// Every element with IEEE division (rows outside the fast path's range).
template <int H, bool HAS_Y, bool FULL>
__device__ __forceinline__ void errors_exact(const float2 (&xp)[H], float lo, float hi, int kbase, int d,
                                             float2 (&C)[H])
{
    const float s = __fdiv_rn(__fsub_rn(hi, lo), kLevels);
#pragma unroll
    for (int h = 0; h < H; ++h) {
        C[h].x = valid_x<H, HAS_Y, FULL>(kbase, h, d) ? sq_err_exact(xp[h].x, lo, s) : 0.0f;
        C[h].y = valid_y<H, HAS_Y, FULL>(kbase, h, d) ? sq_err_exact(xp[h].y, lo, s) : 0.0f;
    }
}

// Pairwise sum of the lane's squared errors: slot .x holds the first half of the
// lane's elements, slot .y the second, so packed adds run both halves' trees.
template <int H>
__device__ __forceinline__ float tree_sum2(float2 (&C)[H])
{
#pragma unroll
    for (int w = 1; w < H; w <<= 1) {
#pragma unroll
        for (int k = 0; k < H; k += 2 * w)
            C[k] = __fadd2_rn(C[k], C[k + w]);
    }
    return __fadd_rn(C[0].x, C[0].y);
}

// The 168 moves of the greedy walk. FAST: division-free codes with tie fix-up;
// otherwise IEEE division for every element. All lanes of a row see the same losses.
template <int H, bool HAS_Y, bool FULL, bool FAST, int W>
__device__ __forceinline__ void greedy_walk(const float2 (&xp)[H], int kbase, int d, float mn, float mx,
                                            float step, const TieWindow &tw, float &lbest, float &fbi,
                                            float &fbj)
{
    float fi = 0.0f, fj = 0.0f;  // grid indices as exact small floats (i + j <= 168)
    float lo_i = __fmaf_rn(0.0f, step, mn), hi_j = __fmaf_rn(-0.0f, step, mx);
    float lo_i1 = __fmaf_rn(1.0f, step, mn), hi_j1 = __fmaf_rn(-1.0f, step, mx);
    for (int mv = 0; mv < kMoves; ++mv) {
        // left candidate (i+1, j) = a, right candidate (i, j+1) = b
        float2 Ca[H], Cb[H];
        if constexpr (FAST) {
            const Clip ca = clip_fast(lo_i1, hi_j, tw), cb = clip_fast(lo_i, hi_j1, tw);
            // each candidate is reduced as soon as its errors exist; a candidate with
            // an element too close to a rounding tie (rare) is evaluated again with
            // the IEEE fix-up
            bool hard_a = false, hard_b = false;
            errors_packed<H, HAS_Y, FULL>(xp, ca, kbase, d, Ca, hard_a);
            float la = tree_sum2<H>(Ca);
            errors_packed<H, HAS_Y, FULL>(xp, cb, kbase, d, Cb, hard_b);
            float lb = tree_sum2<H>(Cb);
            if (hard_a || hard_b) {
                if (hard_a) {
                    errors_packed<H, HAS_Y, FULL>(xp, ca, kbase, d, Ca, hard_a);
                    errors_fixup<H, HAS_Y, FULL>(xp, ca, kbase, d, Ca);
                    la = tree_sum2<H>(Ca);
                }
                if (hard_b) {
                    errors_packed<H, HAS_Y, FULL>(xp, cb, kbase, d, Cb, hard_b);
                    errors_fixup<H, HAS_Y, FULL>(xp, cb, kbase, d, Cb);
                    lb = tree_sum2<H>(Cb);
                }
            }
            Ca[0].x = la;
            Cb[0].x = lb;
        } else {
            errors_exact<H, HAS_Y, FULL>(xp, lo_i1, hi_j, kbase, d, Ca);
            errors_exact<H, HAS_Y, FULL>(xp, lo_i, hi_j1, kbase, d, Cb);
            Ca[0].x = tree_sum2<H>(Ca);
            Cb[0].x = tree_sum2<H>(Cb);
        }
        const float la = row_sum<W>(Ca[0].x);
        const float lb = row_sum<W>(Cb[0].x);
        const bool right = lb < la;  // ties move left
        const float l = right ? lb : la;
        fi = right ? fi : fi + 1.0f;
        fj = right ? fj + 1.0f : fj;
        lo_i = right ? lo_i : lo_i1;
        hi_j = right ? hi_j1 : hi_j;
        lo_i1 = __fmaf_rn(fi + 1.0f, step, mn);
        hi_j1 = __fmaf_rn(-(fj + 1.0f), step, mx);
        const bool better = l < lbest;  // the first lowest loss is kept
        lbest = better ? l : lbest;
        fbi = better ? fi : fbi;
        fbj = better ? fj : fbj;
    }
}

// Where a row of the plain kernel lives: row r of the caller's arrays. The pointers
// are formed where they are used, so nothing but r stays live across the search.
struct PlainRow {
    const QuantArgs &a;
    int64_t r;
    __device__ __forceinline__ const float *x() const { return a.x + r * a.ld; }
    __device__ __forceinline__ uint8_t *codes() const { return a.codes + r * a.codes_ld; }
    __device__ __forceinline__ uint16_t *scale_bias() const { return a.scale_bias + 2 * r; }
    __device__ __forceinline__ float *loss() const { return a.row_loss ? a.row_loss + r : nullptr; }
    __device__ __forceinline__ uint8_t *best_ij() const { return a.best_ij ? a.best_ij + 2 * r : nullptr; }
};

// A row listed by the bag backward: entry i names master row id of table t and its
// gradient row G_i; the master row is first moved to fma(-lr, G, w) (and written back).
struct ListedRow {
    const RequantArgs &a;
    int64_t i;
    int t;
    int64_t id;
    __device__ __forceinline__ const float *x() const { return a.tabs.master[t] + id * a.tabs.master_ld[t]; }
    __device__ __forceinline__ float *x_out() const { return a.tabs.master[t] + id * a.tabs.master_ld[t]; }
    __device__ __forceinline__ const float *grad() const { return a.grad_rows + i * a.grad_ld; }
    __device__ __forceinline__ uint8_t *codes() const { return a.tabs.codes[t] + id * a.tabs.codes_ld[t]; }
    __device__ __forceinline__ uint16_t *scale_bias() const { return a.tabs.scale_bias[t] + 2 * id; }
    __device__ __forceinline__ float *loss() const { return nullptr; }
    __device__ __forceinline__ uint8_t *best_ij() const { return nullptr; }
};

// One row per W lanes; M elements per lane; FULL: d == M * W (no padding);
// VEC: 16-byte loads of x and vector stores of the codes are aligned. SGD: the row is
// x + (-lr) * grad, rounded once per element, and is stored back before the search.
template <int M, int W, bool FULL, bool VEC, bool SGD, class Row>
__device__ __forceinline__ void quantize_one(const Row &src, const int d, const bool active, const int greedy,
                                             const float lr, uint32_t *flags)
{
    constexpr bool HAS_Y = M > 1;
    constexpr int H = HAS_Y ? M / 2 : 1;
    const int sub = threadIdx.x & (W - 1);
    const int kbase = sub * M;
    const float *xr = src.x() + kbase;

    // the lane's M elements: element k in xp[k].x (k < H) or xp[k - H].y
    float2 xp[H];
    if constexpr (VEC) {
        float v[M];
#pragma unroll
        for (int m = 0; m < M; m += 4) {
            float4 q4 = SGD ? *reinterpret_cast<const float4 *>(xr + m)
                            : __ldg(reinterpret_cast<const float4 *>(xr + m));
            if constexpr (SGD) {
                const float4 g4 = __ldg(reinterpret_cast<const float4 *>(src.grad() + kbase + m));
                q4.x = __fmaf_rn(-lr, g4.x, q4.x);
                q4.y = __fmaf_rn(-lr, g4.y, q4.y);
                q4.z = __fmaf_rn(-lr, g4.z, q4.z);
                q4.w = __fmaf_rn(-lr, g4.w, q4.w);
                if (active)
                    *reinterpret_cast<float4 *>(src.x_out() + kbase + m) = q4;
            }
            v[m] = q4.x;
            v[m + 1] = q4.y;
            v[m + 2] = q4.z;
            v[m + 3] = q4.w;
        }
#pragma unroll
        for (int h = 0; h < H; ++h)
            xp[h] = make_float2(v[h], v[h + H]);
    } else {
#pragma unroll
        for (int h = 0; h < H; ++h) {
            const bool vx = valid_x<H, HAS_Y, FULL>(kbase, h, d), vy = valid_y<H, HAS_Y, FULL>(kbase, h, d);
            xp[h].x = vx ? (SGD ? xr[h] : __ldg(xr + h)) : 0.0f;
            xp[h].y = vy ? (SGD ? xr[h + H] : __ldg(xr + h + H)) : 0.0f;
            if constexpr (SGD) {
                const float *gr = src.grad() + kbase;
                float *xo = src.x_out() + kbase;
                if (vx) {
                    xp[h].x = __fmaf_rn(-lr, __ldg(gr + h), xp[h].x);
                    if (active)
                        xo[h] = xp[h].x;
                }
                if (vy) {
                    xp[h].y = __fmaf_rn(-lr, __ldg(gr + h + H), xp[h].y);
                    if (active)
                        xo[h + H] = xp[h].y;
                }
            }
        }
    }

    float mn = FLT_MAX, mx = -FLT_MAX;
    bool nonfinite = false;
#pragma unroll
    for (int h = 0; h < H; ++h) {
        if (valid_x<H, HAS_Y, FULL>(kbase, h, d)) {
            mn = fminf(mn, xp[h].x);
            mx = fmaxf(mx, xp[h].x);
            nonfinite |= !isfinite(xp[h].x);
        }
        if (valid_y<H, HAS_Y, FULL>(kbase, h, d)) {
            mn = fminf(mn, xp[h].y);
            mx = fmaxf(mx, xp[h].y);
            nonfinite |= !isfinite(xp[h].y);
        }
    }
    row_minmax<W>(mn, mx);

    const float range = __fsub_rn(mx, mn);
    const float step = __fdiv_rn(range, kSteps);
    // Fast path, decided once per row. Every candidate has |lo| <= max(|xmin|, |xmax|)
    // and width > 30 * step (the walk stops at 32 steps; when K <= 2^16 the grid
    // points' rounding costs less than 0.25 step), so K bounds |lo * rcp(hi - lo)|
    // for the whole walk, the starting clip included, and sets the tie margin.
    const float w_min = __fmul_rn(step, 30.0f);
    const float K = __fmul_rn(fmaxf(fabsf(mn), fabsf(mx)), rcp_approx(w_min));
    const bool fast_row = range <= kFastWMax && w_min >= kFastWMin && K <= kFastLoR;
    const TieWindow tw = tie_window(K);
    float lbest;
    {
        // the starting clip (0, 0): grid points lo(0) = fma(0, step, xmin), hi(0) = fma(-0, step, xmax)
        float2 C0[H];
        if (fast_row) {
            const Clip c0 = clip_fast(__fmaf_rn(0.0f, step, mn), __fmaf_rn(-0.0f, step, mx), tw);
            bool hard = false;
            errors_packed<H, HAS_Y, FULL>(xp, c0, kbase, d, C0, hard);
            if (hard)
                errors_fixup<H, HAS_Y, FULL>(xp, c0, kbase, d, C0);
        } else {
            errors_exact<H, HAS_Y, FULL>(xp, mn, mx, kbase, d, C0);
        }
        lbest = row_sum<W>(tree_sum2<H>(C0));
    }
    float fbi = 0.0f, fbj = 0.0f;
    // A constant row has loss 0 at every grid point: the walk cannot change (0, 0).
    const bool walk_row = greedy && range != 0.0f;
    if constexpr (W == 1) {
        // one row per lane: the walk has no shuffles, each row takes its own path
        if (walk_row) {
            if (fast_row)
                greedy_walk<H, HAS_Y, FULL, true, W>(xp, kbase, d, mn, mx, step, tw, lbest, fbi, fbj);
            else
                greedy_walk<H, HAS_Y, FULL, false, W>(xp, kbase, d, mn, mx, step, tw, lbest, fbi, fbj);
        }
    } else if (__any_sync(0xffffffffu, walk_row)) {
        // the walk's row shuffles run on the whole warp: the warp walks if any of its rows
        // does (the others keep (0, 0)) and takes the fast path when every walking row
        // qualifies; the two paths give identical losses
        const bool fast = __all_sync(0xffffffffu, !walk_row || fast_row);
        float lb = lbest, bi = 0.0f, bj = 0.0f;
        if (fast)
            greedy_walk<H, HAS_Y, FULL, true, W>(xp, kbase, d, mn, mx, step, tw, lb, bi, bj);
        else
            greedy_walk<H, HAS_Y, FULL, false, W>(xp, kbase, d, mn, mx, step, tw, lb, bi, bj);
        if (walk_row) {
            lbest = lb;
            fbi = bi;
            fbj = bj;
        }
    }
    const int bi = (int)fbi, bj = (int)fbj;

    // Final parameters in binary16 and the codes with IEEE division.
    const float lo = __fmaf_rn(fbi, step, mn);
    const float hi = __fmaf_rn(-fbj, step, mx);
    const float s = __fdiv_rn(__fsub_rn(hi, lo), kLevels);
    const __half s16 = __float2half_rn(s), b16 = __float2half_rn(lo);
    const float S = __half2float(s16), B = __half2float(b16);
    uint8_t packed[(M + 1) / 2];
#pragma unroll
    for (int m = 0; m < (M + 1) / 2; ++m) {
        const int k0 = 2 * m, k1 = 2 * m + 1;
        const float x0 = k0 < H ? xp[k0 % H].x : xp[(k0 - H) % H].y;
        const unsigned q0 = (FULL || kbase + k0 < d) ? (unsigned)exact_code(x0, B, S) : 0u;
        unsigned q1 = 0u;
        if (k1 < M && (FULL || kbase + k1 < d)) {
            const float x1 = k1 < H ? xp[k1 % H].x : xp[(k1 - H) % H].y;
            q1 = (unsigned)exact_code(x1, B, S);
        }
        packed[m] = (uint8_t)(q0 | (q1 << 4));
    }
    if (!active)
        return;

    uint8_t *cr = src.codes() + kbase / 2;
    if constexpr (VEC && M >= 2) {
        if constexpr (M == 32) {
            uint4 w;
            memcpy(&w, packed, 16);
            *reinterpret_cast<uint4 *>(cr) = w;
        } else if constexpr (M == 16) {
            uint2 w;
            memcpy(&w, packed, 8);
            *reinterpret_cast<uint2 *>(cr) = w;
        } else if constexpr (M == 8) {
            uint32_t w;
            memcpy(&w, packed, 4);
            *reinterpret_cast<uint32_t *>(cr) = w;
        } else if constexpr (M == 4) {
            uint16_t w;
            memcpy(&w, packed, 2);
            *reinterpret_cast<uint16_t *>(cr) = w;
        } else {
            cr[0] = packed[0];
        }
    } else {
#pragma unroll
        for (int m = 0; m < (M + 1) / 2; ++m)
            if (FULL || kbase + 2 * m < d)
                cr[m] = packed[m];
    }
    if (sub == 0) {
        uint16_t *sb = src.scale_bias();
        sb[0] = __half_as_ushort(s16);
        sb[1] = __half_as_ushort(b16);
        if (float *lp = src.loss())
            *lp = lbest;
        if (uint8_t *ij = src.best_ij()) {
            ij[0] = (uint8_t)bi;
            ij[1] = (uint8_t)bj;
        }
        if (isinf(S) || isinf(B))
            raise_flag(flags, DQ_FLAG_FP16_OVERFLOW);
    }
    if (nonfinite)
        raise_flag(flags, DQ_FLAG_NONFINITE);
}

template <int M, int W, bool FULL, bool VEC>
__global__ void __launch_bounds__(128) quantize_rows_kernel(const QuantArgs a, const int greedy)
{
    int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / W;
    const bool active = row < a.n;
    if (!active)
        row = a.n - 1;  // idle lanes shadow the last row so the warp stays converged
    quantize_one<M, W, FULL, VEC, false>(PlainRow{a, row}, a.d, active, greedy, 0.0f, a.flags);
}

// Table of a global row key: the last table whose first key is <= key.
__device__ __forceinline__ int table_of_key(const RequantTables &tabs, int n_tables, uint32_t key)
{
    int lo = 0, hi = n_tables;  // tabs.key_base[lo] <= key < tabs.key_base[hi] (key_base[n_tables] = total)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tabs.key_base[mid] <= key)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

// Re-quantization of the rows the bag backward listed, with their SGD step fused in.
// Grid-stride over the list (its length is known on the device only); the loop
// bound is warp-uniform, so the row's lanes stay converged for the shuffles.
template <int M, int W, bool FULL, bool VEC>
__global__ void __launch_bounds__(128) requant_rows_kernel(const RequantArgs a, const int greedy)
{
    if (*a.bad)
        return;
    const int64_t count = *a.count;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t first = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); first < count * W;
         first += stride) {
        int64_t i = (first + (threadIdx.x & 31)) / W;
        const bool active = i < count;
        if (!active)
            i = count - 1;
        const uint32_t key = a.list[i];
        const int t = table_of_key(a.tabs, a.n_tables, key);
        quantize_one<M, W, FULL, VEC, true>(ListedRow{a, i, t, (int64_t)(key - a.tabs.key_base[t])}, a.d, active,
                                            greedy, a.lr, a.flags);
    }
}



template <int M, int W>
cudaError_t launch_mw(const QuantArgs &a, int greedy, cudaStream_t stream)
{
    constexpr int kBlock = 128;   // measured: finer blocks shorten the last wave
    const int64_t threads = a.n * W;
    const int64_t grid = (threads + kBlock - 1) / kBlock;
    const bool full = a.d == M * W;
    const bool vec = full && (M % 4 == 0) && (a.ld % 4 == 0) &&
                     (reinterpret_cast<uintptr_t>(a.x) & 15) == 0 &&
                     (a.codes_ld % ((M + 1) / 2) == 0) &&
                     (reinterpret_cast<uintptr_t>(a.codes) % ((M + 1) / 2)) == 0;
    if (vec) {
        if constexpr (M % 4 == 0)
            quantize_rows_kernel<M, W, true, true><<<(unsigned)grid, kBlock, 0, stream>>>(a, greedy);
    } else if (full) {
        quantize_rows_kernel<M, W, true, false><<<(unsigned)grid, kBlock, 0, stream>>>(a, greedy);
    } else {
        quantize_rows_kernel<M, W, false, false><<<(unsigned)grid, kBlock, 0, stream>>>(a, greedy);
    }
    return cudaGetLastError();
}

template <int M, int W>
cudaError_t launch_requant_mw(const RequantArgs &a, int64_t max_rows, int greedy, int num_sms,
                              cudaStream_t stream)
{
    constexpr int kBlock = 128;
    // one lane group per row of the host's bound (max_rows): the blocks past the listed
    // rows exit at once, and the hardware balances the rest as for the plain quantizer
    // (a capped grid-stride loop left a ragged last round per warp); the grid-stride
    // loop stays for bounds above the grid limit
    const int64_t need = (max_rows * W + kBlock - 1) / kBlock;
    const int64_t cap = (int64_t)num_sms * 4096;
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    const bool full = a.d == M * W;
    bool vec = full && (M % 4 == 0) && (a.grad_ld % 4 == 0) &&
               (reinterpret_cast<uintptr_t>(a.grad_rows) & 15) == 0;
    for (int t = 0; t < a.n_tables && vec; ++t)
        vec = a.tabs.master_ld[t] % 4 == 0 && (reinterpret_cast<uintptr_t>(a.tabs.master[t]) & 15) == 0 &&
              a.tabs.codes_ld[t] % ((M + 1) / 2) == 0 &&
              reinterpret_cast<uintptr_t>(a.tabs.codes[t]) % ((M + 1) / 2) == 0;
    if (vec) {
        if constexpr (M % 4 == 0)
            requant_rows_kernel<M, W, true, true><<<grid, kBlock, 0, stream>>>(a, greedy);
    } else if (full) {
        requant_rows_kernel<M, W, true, false><<<grid, kBlock, 0, stream>>>(a, greedy);
    } else {
        requant_rows_kernel<M, W, false, false><<<grid, kBlock, 0, stream>>>(a, greedy);
    }
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_requant(const RequantArgs &a, int64_t max_rows, int mode, int num_sms, cudaStream_t stream)
{
    if (max_rows <= 0)
        return cudaSuccess;
    int p = 1;
    while (p < a.d)
        p <<= 1;
    const int greedy = mode == DQ_MODE_GREEDY;
    switch (p) {
    case 1: return launch_requant_mw<1, 1>(a, max_rows, greedy, num_sms, stream);
    case 2: return launch_requant_mw<2, 1>(a, max_rows, greedy, num_sms, stream);
    case 4: return launch_requant_mw<4, 1>(a, max_rows, greedy, num_sms, stream);
    case 8: return launch_requant_mw<8, 1>(a, max_rows, greedy, num_sms, stream);
    case 16: return launch_requant_mw<16, 1>(a, max_rows, greedy, num_sms, stream);
    case 32: return launch_requant_mw<16, 2>(a, max_rows, greedy, num_sms, stream);
    case 64: return launch_requant_mw<16, 4>(a, max_rows, greedy, num_sms, stream);
    case 128: return launch_requant_mw<16, 8>(a, max_rows, greedy, num_sms, stream);
    case 256: return launch_requant_mw<16, 16>(a, max_rows, greedy, num_sms, stream);
    case 512: return launch_requant_mw<16, 32>(a, max_rows, greedy, num_sms, stream);
    case 1024: return launch_requant_mw<32, 32>(a, max_rows, greedy, num_sms, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_quantize(const QuantArgs &a, int mode, int /*num_sms*/, cudaStream_t stream)
{
    int p = 1;
    while (p < a.d)
        p <<= 1;
    const int greedy = mode == DQ_MODE_GREEDY;
    switch (p) {
    case 1: return launch_mw<1, 1>(a, greedy, stream);
    case 2: return launch_mw<2, 1>(a, greedy, stream);
    case 4: return launch_mw<4, 1>(a, greedy, stream);
    case 8: return launch_mw<8, 1>(a, greedy, stream);
    case 16: return launch_mw<16, 1>(a, greedy, stream);
    case 32: return launch_mw<16, 2>(a, greedy, stream);
    case 64: return launch_mw<16, 4>(a, greedy, stream);
    case 128: return launch_mw<16, 8>(a, greedy, stream);
    case 256: return launch_mw<16, 16>(a, greedy, stream);
    case 512: return launch_mw<16, 32>(a, greedy, stream);
    case 1024: return launch_mw<32, 32>(a, greedy, stream);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace dq
