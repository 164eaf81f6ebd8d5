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
// search is pure FP32 ALU work: 337 loss evaluations x d elements per row, each
// element ~10 instructions, two candidates evaluated side by side for ILP. The
// loss is a pairwise sum: an in-lane binary tree over M elements, then an XOR
// butterfly over the W lanes, which is the same recursive-halving order, so
// every lane of the row gets the identical binary32 value.
//
// The code of an element during the search, q = clamp(rint((x - lo) / s), 0, 15)
// with an IEEE quotient, is computed without a division: u = sat((x - lo) * rcp(w))
// (w = hi - lo ~ 15 s), then rint(15 u) by a magic-number add. 15 u is within
// 4e-6 of the exact quotient, so it rounds the same way as the IEEE quotient
// unless it lies within 2^-16 of a half-integer; those rare elements are flagged
// and recomputed with the IEEE division. The codes the search sees are therefore
// exactly the IEEE ones.
#include <cfloat>

#include "dq_internal.cuh"

namespace dq {
namespace {

constexpr float kSteps = 200.0f;         // grid steps over the row's range
constexpr int kMoves = 168;              // moves while width > 0.16 * range
constexpr float kLevels = 15.0f;         // 2^4 - 1
constexpr float kMagic = 12582912.0f;    // 1.5 * 2^23: x + kMagic rounds x in [0, 2^22) to an integer
constexpr float kHardGap = 0.5f - 1.52587890625e-05f;  // flag |15u - q| beyond 0.5 - 2^-16
constexpr float kFastWMin = 1.0e-36f;    // w in [kFastWMin, kFastWMax]: s normal, 1/w normal
constexpr float kFastWMax = 1.0e36f;

__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float mul_sat(float a, float b)
{
    float r;
    asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// q = clamp(rint(fl(fl(x - lo) / s)), 0, 15) with an IEEE quotient; 0 when s == 0.
__device__ __forceinline__ float exact_code(float x, float lo, float s)
{
    if (s == 0.0f)
        return 0.0f;
    float q = rintf(__fdiv_rn(__fsub_rn(x, lo), s));
    return fminf(fmaxf(q, 0.0f), kLevels);
}

template <int M>
__device__ __forceinline__ float tree_sum(float (&c)[M])
{
#pragma unroll
    for (int w = 1; w < M; w <<= 1) {
#pragma unroll
        for (int k = 0; k < M; k += 2 * w)
            c[k] = __fadd_rn(c[k], c[k + w]);
    }
    return c[0];
}

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

// Squared reconstruction errors of this lane's M elements for one clip range,
// with IEEE codes (exact path).
template <int M, bool FULL>
__device__ __forceinline__ void errors_exact(const float (&v)[M], int kbase, int d, float lo, float s,
                                             float (&c)[M])
{
#pragma unroll
    for (int m = 0; m < M; ++m) {
        float q = exact_code(v[m], lo, s);
        float xh = __fmaf_rn(q, s, lo);
        float e = __fsub_rn(v[m], xh);
        c[m] = (FULL || kbase + m < d) ? __fmul_rn(e, e) : 0.0f;
    }
}

// The two candidate losses of one move, (lo_a, hi_a) and (lo_b, hi_b), for this
// lane's elements (before the cross-lane butterfly).
template <int M, bool FULL>
__device__ __forceinline__ void lane_loss_pair(const float (&v)[M], int kbase, int d, float lo_a,
                                               float hi_a, float lo_b, float hi_b, float &la, float &lb)
{
    const float wa = __fsub_rn(hi_a, lo_a), wb = __fsub_rn(hi_b, lo_b);
    const float sa = __fdiv_rn(wa, kLevels), sb = __fdiv_rn(wb, kLevels);
    float ca[M], cb[M];
    const bool fast = wa >= kFastWMin && wa <= kFastWMax && wb >= kFastWMin && wb <= kFastWMax;
    bool hard_a = !fast, hard_b = !fast;
    if (fast) {
        const float ra = rcp_approx(wa), rb = rcp_approx(wb);
        const float nsa = -sa, nsb = -sb;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const float ta = __fsub_rn(v[m], lo_a), tb = __fsub_rn(v[m], lo_b);
            const float ua = mul_sat(ta, ra), ub = mul_sat(tb, rb);
            const float za = __fmaf_rn(ua, kLevels, kMagic), zb = __fmaf_rn(ub, kLevels, kMagic);
            const float nqa = __fsub_rn(kMagic, za), nqb = __fsub_rn(kMagic, zb);   // -q, exact
            const float da = __fmaf_rn(ua, kLevels, nqa), db = __fmaf_rn(ub, kLevels, nqb);
            hard_a |= fabsf(da) > kHardGap;
            hard_b |= fabsf(db) > kHardGap;
            const float xa = __fmaf_rn(nqa, nsa, lo_a), xb = __fmaf_rn(nqb, nsb, lo_b);  // q*s + lo, once rounded
            const float ea = __fsub_rn(v[m], xa), eb = __fsub_rn(v[m], xb);
            ca[m] = (FULL || kbase + m < d) ? __fmul_rn(ea, ea) : 0.0f;
            cb[m] = (FULL || kbase + m < d) ? __fmul_rn(eb, eb) : 0.0f;
        }
    }
    if (hard_a)
        errors_exact<M, FULL>(v, kbase, d, lo_a, sa, ca);
    if (hard_b)
        errors_exact<M, FULL>(v, kbase, d, lo_b, sb, cb);
    la = tree_sum<M>(ca);
    lb = tree_sum<M>(cb);
}

template <int M, bool FULL>
__device__ __forceinline__ float lane_loss_one(const float (&v)[M], int kbase, int d, float lo, float hi)
{
    float c[M];
    errors_exact<M, FULL>(v, kbase, d, lo, __fdiv_rn(__fsub_rn(hi, lo), kLevels), c);
    return tree_sum<M>(c);
}

// One row per W lanes; M elements per lane; FULL: d == M * W (no padding);
// VEC: 16-byte loads of x and vector stores of the codes are aligned.
template <int M, int W, bool FULL, bool VEC>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const QuantArgs a, const int greedy)
{
    const int sub = threadIdx.x & (W - 1);
    int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / W;
    const bool active = row < a.n;
    if (!active)
        row = a.n - 1;  // idle lanes shadow the last row so the warp stays converged
    const int d = a.d;
    const int kbase = sub * M;
    const float *xr = a.x + row * a.ld + kbase;

    float v[M];
    if constexpr (VEC) {
#pragma unroll
        for (int m = 0; m < M; m += 4) {
            const float4 q4 = __ldg(reinterpret_cast<const float4 *>(xr + m));
            v[m] = q4.x;
            v[m + 1] = q4.y;
            v[m + 2] = q4.z;
            v[m + 3] = q4.w;
        }
    } else {
#pragma unroll
        for (int m = 0; m < M; ++m)
            v[m] = (FULL || kbase + m < d) ? __ldg(xr + m) : 0.0f;
    }

    float mn = FLT_MAX, mx = -FLT_MAX;
    bool nonfinite = false;
#pragma unroll
    for (int m = 0; m < M; ++m) {
        if (FULL || kbase + m < d) {
            mn = fminf(mn, v[m]);
            mx = fmaxf(mx, v[m]);
            nonfinite |= !isfinite(v[m]);
        }
    }
    row_minmax<W>(mn, mx);

    const float range = __fsub_rn(mx, mn);
    const float step = __fdiv_rn(range, kSteps);
    float lbest = row_sum<W>(lane_loss_one<M, FULL>(v, kbase, d, mn, mx));
    int i = 0, j = 0, bi = 0, bj = 0;
    if (greedy) {
        for (int mv = 0; mv < kMoves; ++mv) {
            const float lo_l = __fmaf_rn((float)(i + 1), step, mn), hi_l = __fmaf_rn(-(float)j, step, mx);
            const float lo_r = __fmaf_rn((float)i, step, mn), hi_r = __fmaf_rn(-(float)(j + 1), step, mx);
            float ll, lr;
            lane_loss_pair<M, FULL>(v, kbase, d, lo_l, hi_l, lo_r, hi_r, ll, lr);
            ll = row_sum<W>(ll);
            lr = row_sum<W>(lr);
            float l;
            if (lr < ll) {
                ++j;
                l = lr;
            } else {
                ++i;
                l = ll;
            }
            if (l < lbest) {
                lbest = l;
                bi = i;
                bj = j;
            }
        }
    }

    // Final parameters in binary16 and the codes with IEEE division.
    const float lo = __fmaf_rn((float)bi, step, mn);
    const float hi = __fmaf_rn(-(float)bj, step, mx);
    const float s = __fdiv_rn(__fsub_rn(hi, lo), kLevels);
    const __half s16 = __float2half_rn(s), b16 = __float2half_rn(lo);
    const float S = __half2float(s16), B = __half2float(b16);
    uint8_t packed[(M + 1) / 2];
#pragma unroll
    for (int m = 0; m < (M + 1) / 2; ++m) {
        const int k0 = 2 * m, k1 = 2 * m + 1;
        const unsigned q0 = (FULL || kbase + k0 < d) ? (unsigned)exact_code(v[k0], B, S) : 0u;
        unsigned q1 = 0u;
        if (k1 < M && (FULL || kbase + k1 < d))
            q1 = (unsigned)exact_code(v[k1], B, S);
        packed[m] = (uint8_t)(q0 | (q1 << 4));
    }
    if (!active)
        return;

    uint8_t *cr = a.codes + row * a.codes_ld + kbase / 2;
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
        a.scale_bias[2 * row] = __half_as_ushort(s16);
        a.scale_bias[2 * row + 1] = __half_as_ushort(b16);
        if (a.row_loss)
            a.row_loss[row] = lbest;
        if (a.best_ij) {
            a.best_ij[2 * row] = (uint8_t)bi;
            a.best_ij[2 * row + 1] = (uint8_t)bj;
        }
        if (isinf(S) || isinf(B))
            raise_flag(a.flags, DQ_FLAG_FP16_OVERFLOW);
    }
    if (nonfinite)
        raise_flag(a.flags, DQ_FLAG_NONFINITE);
}

template <int M, int W>
cudaError_t launch_mw(const QuantArgs &a, int greedy, cudaStream_t stream)
{
    constexpr int kBlock = 256;
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

} // namespace

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
