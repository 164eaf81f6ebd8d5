// dq_bag.cu -- INT4 row dequantization and the sum-pooled INT4 embedding bag on sm_100a.
//
// Row format: "Post-Training 4-bit Quantization on Embedding Tables", section
// 提出的方法 (proposed method), bullet 2 (FP16 scale and bias per row), with the
// codes packed two per byte. Lookup: "Deep Learning Recommendation Model for
// Personalization and Recommendation Systems", section 提出的方法 (proposed
// method), bullet 1, summed over each bag of ids.
//
// Both kernels are bound by HBM (and, for long bags, by integer/FP32 issue):
// packed rows are read with 8- or 16-byte vector loads, outputs written with
// 16-byte stores, and a nibble becomes a float with one LOP3 and one FADD:
// OR-ing 0x4B000000 onto the nibble left in place at bits 4k..4k+3 gives the
// float 2^23 + q*2^(4k); subtracting 2^23 leaves q*2^(4k) exactly, and an FMA
// with scale*2^(-4k) (an exact power-of-two rescaling) gives fma(q, scale, bias)
// bit for bit. Nibbles 5..7 of a word are shifted down by 12 bits first.
#include "dq_internal.cuh"

namespace dq {
namespace {

constexpr float kTwo23 = 8388608.0f;

struct RowParams {
    float s[5];   // scale * 2^(-4k), k = 0..4
    float b;
};

__device__ __forceinline__ RowParams row_params(uint32_t sbw)
{
    RowParams p;
    const float S = __half2float(__ushort_as_half((unsigned short)(sbw & 0xffffu)));
    p.b = __half2float(__ushort_as_half((unsigned short)(sbw >> 16)));
    p.s[0] = S;
    p.s[1] = __fmul_rn(S, 0.0625f);
    p.s[2] = __fmul_rn(S, 0.00390625f);
    p.s[3] = __fmul_rn(S, 0.000244140625f);
    p.s[4] = __fmul_rn(S, 1.52587890625e-05f);
    return p;
}

// The 8 dequantized values of one 32-bit code word (elements 8w .. 8w+7).
__device__ __forceinline__ void decode_word(uint32_t w, const RowParams &p, float (&x)[8])
{
    const uint32_t hi = w >> 12;  // nibbles 5, 6, 7 -> bit positions 8, 12, 16
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const float f = __fsub_rn(__uint_as_float((w & (0xfu << (4 * k))) | 0x4B000000u), kTwo23);
        x[k] = __fmaf_rn(f, p.s[k], p.b);
    }
#pragma unroll
    for (int k = 5; k < 8; ++k) {
        const int kk = k - 3;
        const float f = __fsub_rn(__uint_as_float((hi & (0xfu << (4 * kk))) | 0x4B000000u), kTwo23);
        x[k] = __fmaf_rn(f, p.s[kk], p.b);
    }
}

// ---------------------------------------------------------------------------
// dequantize: one thread per 16-element chunk (8 code bytes -> 64 output bytes)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dequant16_kernel(const DequantArgs a)
{
    const int cpr = a.d / 16;
    const int64_t total = a.n * cpr;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total;
         c += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = c / cpr;
        const int part = (int)(c - row * cpr);
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(a.codes + row * a.codes_ld) + part);
        const uint32_t sbw = __ldg(reinterpret_cast<const uint32_t *>(a.scale_bias) + row);
        const RowParams p = row_params(sbw);
        float x0[8], x1[8];
        decode_word(w.x, p, x0);
        decode_word(w.y, p, x1);
        float4 *o = reinterpret_cast<float4 *>(a.out + row * a.out_ld) + part * 4;
        __stcs(o + 0, make_float4(x0[0], x0[1], x0[2], x0[3]));
        __stcs(o + 1, make_float4(x0[4], x0[5], x0[6], x0[7]));
        __stcs(o + 2, make_float4(x1[0], x1[1], x1[2], x1[3]));
        __stcs(o + 3, make_float4(x1[4], x1[5], x1[6], x1[7]));
    }
}

// any d, any alignment: one thread per code byte (2 elements)
__global__ void __launch_bounds__(256) dequant_generic_kernel(const DequantArgs a)
{
    const int bpr = (a.d + 1) / 2;
    const int64_t total = a.n * bpr;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total;
         c += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = c / bpr;
        const int m = (int)(c - row * bpr);
        const uint8_t byte = a.codes[row * a.codes_ld + m];
        const float S = __half2float(__ushort_as_half(a.scale_bias[2 * row]));
        const float B = __half2float(__ushort_as_half(a.scale_bias[2 * row + 1]));
        float *o = a.out + row * a.out_ld + 2 * m;
        o[0] = __fmaf_rn((float)(byte & 15u), S, B);
        if (2 * m + 1 < a.d)
            o[1] = __fmaf_rn((float)(byte >> 4), S, B);
    }
}

// ---------------------------------------------------------------------------
// embedding bag: G = d / E lanes per bag, E outputs (E/2 code bytes) per lane
// ---------------------------------------------------------------------------
template <int E>
struct CodeVec;
template <>
struct CodeVec<16> {
    using T = uint2;
    static __device__ __forceinline__ uint32_t word(const T &v, int i) { return i == 0 ? v.x : v.y; }
};
template <>
struct CodeVec<32> {
    using T = uint4;
    static __device__ __forceinline__ uint32_t word(const T &v, int i)
    {
        return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
    }
};

constexpr int kBagBlock = 256;
constexpr int kBagUnroll = 4;

template <int E>
__global__ void __launch_bounds__(kBagBlock) embbag_kernel(const __grid_constant__ BagTables tabs,
                                                           const BagArgs a)
{
    using V = typename CodeVec<E>::T;
    constexpr int NW = E / 8;
    const int G = a.d / E;                      // lanes per bag, a power of two <= 32
    const int bags_per_block = kBagBlock / G;
    const int64_t total = (int64_t)a.T * a.batch;
    const int64_t g0 = (int64_t)blockIdx.x * bags_per_block;

    __shared__ int32_t soff[kBagBlock + 1];
    for (int k = threadIdx.x; k <= bags_per_block; k += kBagBlock) {
        const int64_t gi = g0 + k;
        soff[k] = gi <= total ? __ldg(a.offsets + gi) : 0;
    }
    __syncthreads();

    const int lb = threadIdx.x / G, sub = threadIdx.x - lb * G;
    const int64_t g = g0 + lb;
    if (g >= total)
        return;
    const int t = (int)(g / a.batch);
    const int b = (int)(g - (int64_t)t * a.batch);
    const int32_t n_ids = max(__ldg(a.offsets + total), 0);  // the id count
    int32_t p = soff[lb];
    int32_t p1 = soff[lb + 1];
    if (p1 < p || p < 0 || p1 > n_ids) {
        if (sub == 0)
            raise_flag(a.flags, DQ_FLAG_BAD_OFFSETS);
        p = min(max(p, 0), n_ids);
        p1 = max(min(p1, n_ids), p);
    }
    const uint8_t *codes = tabs.codes[t] + sub * (E / 2);
    const uint32_t *sbp = reinterpret_cast<const uint32_t *>(tabs.scale_bias[t]);
    const int64_t n_rows = tabs.n_rows[t];
    const int64_t ld = tabs.codes_ld[t];

    float acc[E];
#pragma unroll
    for (int k = 0; k < E; ++k)
        acc[k] = 0.0f;
    bool bad = false;

    for (; p < p1; p += kBagUnroll) {
        int32_t id[kBagUnroll];
        bool ok[kBagUnroll];
#pragma unroll
        for (int u = 0; u < kBagUnroll; ++u) {
            id[u] = (p + u < p1) ? __ldg(a.indices + p + u) : 0;
            ok[u] = (p + u < p1) && id[u] >= 0 && (int64_t)id[u] < n_rows;
            bad |= (p + u < p1) && !ok[u];
        }
        V w[kBagUnroll];
        uint32_t sbw[kBagUnroll];
#pragma unroll
        for (int u = 0; u < kBagUnroll; ++u) {
            const int64_t r = ok[u] ? id[u] : 0;
            if (ok[u]) {
                w[u] = __ldg(reinterpret_cast<const V *>(codes + r * ld));
                sbw[u] = __ldg(sbp + r);
            }
        }
#pragma unroll
        for (int u = 0; u < kBagUnroll; ++u) {
            if (ok[u]) {
                const RowParams prm = row_params(sbw[u]);
#pragma unroll
                for (int i = 0; i < NW; ++i) {
                    float x[8];
                    decode_word(CodeVec<E>::word(w[u], i), prm, x);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        acc[8 * i + k] = __fadd_rn(acc[8 * i + k], x[k]);
                }
            }
        }
    }
    if (bad && sub == 0)
        raise_flag(a.flags, DQ_FLAG_BAD_INDEX);

    float4 *o = reinterpret_cast<float4 *>(a.out + (int64_t)b * a.T * a.d + (int64_t)t * a.d + sub * E);
#pragma unroll
    for (int k = 0; k < E; k += 4)
        o[k / 4] = make_float4(acc[k], acc[k + 1], acc[k + 2], acc[k + 3]);
}

// any d, any alignment: one warp per bag, lanes stride over the elements
__global__ void __launch_bounds__(256) embbag_generic_kernel(const __grid_constant__ BagTables tabs,
                                                             const BagArgs a)
{
    const int64_t total = (int64_t)a.T * a.batch;
    const int lane = threadIdx.x & 31;
    const int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (g >= total)
        return;
    const int t = (int)(g / a.batch);
    const int b = (int)(g - (int64_t)t * a.batch);
    const int32_t n_ids = max(__ldg(a.offsets + total), 0);  // the id count
    int32_t p0 = __ldg(a.offsets + g), p1 = __ldg(a.offsets + g + 1);
    if (p1 < p0 || p0 < 0 || p1 > n_ids) {
        if (lane == 0)
            raise_flag(a.flags, DQ_FLAG_BAD_OFFSETS);
        p0 = min(max(p0, 0), n_ids);
        p1 = max(min(p1, n_ids), p0);
    }
    float *o = a.out + (int64_t)b * a.T * a.d + (int64_t)t * a.d;
    const int64_t n_rows = tabs.n_rows[t];
    for (int k0 = 0; k0 < a.d; k0 += 32) {
        const int k = k0 + lane;
        float acc = 0.0f;
        bool bad = false;
        for (int32_t p = p0; p < p1; ++p) {
            const int32_t id = __ldg(a.indices + p);
            if (id < 0 || (int64_t)id >= n_rows) {
                bad = true;
                continue;
            }
            if (k < a.d) {
                const uint8_t byte = tabs.codes[t][(int64_t)id * tabs.codes_ld[t] + k / 2];
                const float S = __half2float(__ushort_as_half(tabs.scale_bias[t][2 * (int64_t)id]));
                const float B = __half2float(__ushort_as_half(tabs.scale_bias[t][2 * (int64_t)id + 1]));
                acc = __fadd_rn(acc, __fmaf_rn((float)((byte >> (4 * (k & 1))) & 15u), S, B));
            }
        }
        if (bad && lane == 0 && k0 == 0)
            raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
        if (k < a.d)
            o[k] = acc;
    }
}

int grid_for(int64_t work, int block, int num_sms)
{
    const int64_t need = (work + block - 1) / block;
    const int64_t cap = (int64_t)num_sms * (2048 / block) * 4;  // four waves of full occupancy
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

} // namespace

cudaError_t launch_dequantize(const DequantArgs &a, int num_sms, cudaStream_t stream)
{
    const bool fast = a.d % 16 == 0 && a.codes_ld % 8 == 0 && a.out_ld % 4 == 0 &&
                      (reinterpret_cast<uintptr_t>(a.codes) & 7) == 0 &&
                      (reinterpret_cast<uintptr_t>(a.out) & 15) == 0 &&
                      (reinterpret_cast<uintptr_t>(a.scale_bias) & 3) == 0;
    if (fast)
        dequant16_kernel<<<grid_for(a.n * (a.d / 16), 256, num_sms), 256, 0, stream>>>(a);
    else
        dequant_generic_kernel<<<grid_for(a.n * ((a.d + 1) / 2), 256, num_sms), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_embbag(const BagTables &tabs, const BagArgs &a, int /*num_sms*/, cudaStream_t stream)
{
    const int64_t total = (int64_t)a.T * a.batch;
    int E = 0;
    if (a.d == 16)
        E = 16;
    else if (a.d % 32 == 0 && a.d / 32 <= 32 && ((a.d / 32) & (a.d / 32 - 1)) == 0)
        E = 32;
    bool fast = E != 0 && (reinterpret_cast<uintptr_t>(a.out) & 15) == 0;
    for (int t = 0; fast && t < a.T; ++t)
        fast = tabs.codes_ld[t] % (E / 2) == 0 && (reinterpret_cast<uintptr_t>(tabs.codes[t]) % (E / 2)) == 0 &&
               (reinterpret_cast<uintptr_t>(tabs.scale_bias[t]) & 3) == 0;
    if (fast) {
        const int G = a.d / E;
        const int bags_per_block = kBagBlock / G;
        const int64_t grid = (total + bags_per_block - 1) / bags_per_block;
        if (E == 16)
            embbag_kernel<16><<<(unsigned)grid, kBagBlock, 0, stream>>>(tabs, a);
        else
            embbag_kernel<32><<<(unsigned)grid, kBagBlock, 0, stream>>>(tabs, a);
    } else {
        const int64_t grid = (total * 32 + 255) / 256;
        embbag_generic_kernel<<<(unsigned)grid, 256, 0, stream>>>(tabs, a);
    }
    return cudaGetLastError();
}

} // namespace dq
