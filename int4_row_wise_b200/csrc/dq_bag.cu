// dq_bag.cu -- INT4 row dequantization and the sum-pooled INT4 embedding bag on sm_100a.
//
// Row format: "Post-Training 4-bit Quantization on Embedding Tables", section
// 提出的方法 (proposed method), bullet 2 (FP16 scale and bias per row), with the
// codes packed two per byte. Lookup: "Deep Learning Recommendation Model for
// Personalization and Recommendation Systems", section 提出的方法 (proposed
// method), bullet 1, summed over each bag of ids.
//
// Both kernels are bound by HBM (and, for long bags, by instruction issue): packed
// rows are read with 8- or 16-byte vector loads, outputs written with 16-byte stores.
// A nibble becomes a float without integer-to-float conversion. The dequantize kernel
// and the long-bag lookup byte-permute each nibble alone into bits 20..23 of a zero
// word, the float q * 2^-129 (a subnormal or the least normal binade, exact either
// way), and multiply it by scale * 2^129 inside the FMA: one instruction per element
// before the FMA, and no subtraction; rows with |scale| >= 1/2, where scale * 2^129
// would overflow, take an exponent trick instead. The dequantize kernel's fallback ORs
// 0x4B000000 onto the nibble left in place at bits 4k..4k+3 (the float
// 2^23 + q*2^(4k); subtracting 2^23 leaves q*2^(4k) exactly, and an FMA with
// scale*2^(-4k), an exact power-of-two rescaling, gives fma(q, scale, bias) bit for
// bit). The one-hot lookup and the long-bag fallback mask the even and odd nibbles
// into the low halves of bytes and byte-permute each under the exponent byte 0x4B
// (the float 2^23 + q).
#include "dq_internal.cuh"

namespace dq {
namespace {

constexpr float kTwo23 = 8388608.0f;
constexpr float kTwo64 = 18446744073709551616.0f, kTwo65 = 36893488147419103232.0f;

// scale * 2^129, the factor that turns the subnormal q * 2^-129 (a nibble placed at bits
// 20..23 of a zero word) back into q * scale inside an FMA: two power-of-two products,
// exact for |scale| < 1/2.
__device__ __forceinline__ float scale_up(float S) { return __fmul_rn(__fmul_rn(S, kTwo64), kTwo65); }

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
// dequantize: one thread per 4 elements (2 code bytes -> one 16-byte store), so that a
// warp's store covers 512 contiguous bytes
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dequant16_kernel(const DequantArgs a, const int cpr_log2)
{
    // one float4 of output per thread: a warp's store covers 512 contiguous bytes
    const int cpr = a.d / 4;
    const uint64_t total = (uint64_t)a.n * cpr;
    for (uint64_t c = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total;
         c += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t row = cpr_log2 >= 0 ? c >> cpr_log2 : c / (uint64_t)cpr;
        const int part = (int)(c - row * cpr);
        const uint32_t w = __ldg(reinterpret_cast<const uint16_t *>(a.codes + row * a.codes_ld) + part);
        const uint32_t sbw = __ldg(reinterpret_cast<const uint32_t *>(a.scale_bias) + row);
        const float S = __half2float(__ushort_as_half((unsigned short)(sbw & 0xffffu)));
        const float B = __half2float(__ushort_as_half((unsigned short)(sbw >> 16)));
        float4 x;
        if (fabsf(S) < 0.5f) {
            const float Sp = scale_up(S);
            const uint32_t lo = (w << 4) & 0xF0F0u, hi = w & 0xF0F0u;
            x.x = __fmaf_rn(__uint_as_float(__byte_perm(lo, 0u, 0x4044u)), Sp, B);
            x.y = __fmaf_rn(__uint_as_float(__byte_perm(hi, 0u, 0x4044u)), Sp, B);
            x.z = __fmaf_rn(__uint_as_float(__byte_perm(lo, 0u, 0x4144u)), Sp, B);
            x.w = __fmaf_rn(__uint_as_float(__byte_perm(hi, 0u, 0x4144u)), Sp, B);
        } else {
            const RowParams p = row_params(sbw);
            float x0[8];
            decode_word(w, p, x0);
            x = make_float4(x0[0], x0[1], x0[2], x0[3]);
        }
        __stcs(reinterpret_cast<float4 *>(a.out + row * a.out_ld) + part, x);
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
// embedding bag
//
// Two layouts in one kernel, chosen on the device from the id count (the last
// offset), so the host need not know the pooling:
//  - long bags (average pooling >= 4): d / E lanes cover a row (E elements, E / 2
//    code bytes each) and IS such lane groups take every IS-th id of the same bag,
//    four ids in flight and the next four ids loaded ahead; the IS partial sums meet
//    in a reduce-scatter over shuffles, and each lane stores E / IS finished sums;
//  - short bags (one-hot lookups): a warp takes 32 bags, each lane writes 16-byte
//    chunks of whole output rows straight from registers.
// Either way a bag's sum is binary32 accumulation of the binary32 fma(q, s, b)
// values, and a bag of one id returns its dequantized row exactly.
// ---------------------------------------------------------------------------
constexpr int kBagThreads = 256;

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


// Reduce-scatter of E sums over the IS id strides (lane bits 0..log2(IS)-1):
// afterwards lane `is` holds elements [is * E/IS, (is+1) * E/IS) in acc[0 .. E/IS).
template <int E, int IS>
__device__ __forceinline__ void reduce_scatter(float (&acc)[E], int is)
{
#pragma unroll
    for (int j = 0, half = E / 2; (1 << j) < IS; ++j, half /= 2) {
        // the highest stride bit splits first, so the kept chunk index is `is`
        const int bitpos = 31 - __clz(IS) - 1 - j;
        const bool upper = (is >> bitpos) & 1;
#pragma unroll
        for (int m = 0; m < E / 2; ++m) {
            if (m < half) {
                const float send = upper ? acc[m] : acc[m + half];
                const float keep = upper ? acc[m + half] : acc[m];
                acc[m] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 1 << bitpos));
            }
        }
    }
}

// One table's view for the bag currently handled by a lane.
struct TableView {
    const uint8_t *codes;     // this lane's element group within row 0
    const uint32_t *sb;       // {scale, bias} of row 0 as one 32-bit word
    uint32_t n_rows;          // rows addressable by an int32 id
    uint32_t ld;              // code bytes between rows
};

__device__ __forceinline__ TableView table_view(const BagTables &tabs, int t, int eg, int E)
{
    TableView v;
    v.codes = tabs.codes[t] + eg * (E / 2);
    v.sb = reinterpret_cast<const uint32_t *>(tabs.scale_bias[t]);
    v.n_rows = (uint32_t)min(tabs.n_rows[t], (int64_t)0x80000000LL);
    v.ld = (uint32_t)tabs.codes_ld[t];
    return v;
}

// acc[0..7] += fma(q_k, scale, bias) for the 8 nibbles of w, with the nibble placed at
// bits 20..23 of an otherwise zero word: the float q * 2^-129 exactly (below 2^-126 it
// is subnormal, the value is the integer word times 2^-149 either way), so
// fma(q * 2^-129, scale * 2^129, bias) is fma(q, scale, bias) bit for bit (the product
// is exact). ss = scale * 2^129 must be finite: |scale| < 1/2.
__device__ __forceinline__ void accumulate_word_d(uint32_t w, float2 ss, float2 bb, float2 (&acc)[4])
{
    const uint32_t lo = (w << 4) & 0xF0F0F0F0u, hi = w & 0xF0F0F0F0u;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t sel = 0x4044u | ((uint32_t)b << 8);
        const float2 v = make_float2(__uint_as_float(__byte_perm(lo, 0u, sel)), __uint_as_float(__byte_perm(hi, 0u, sel)));
        acc[b] = __fadd2_rn(acc[b], __ffma2_rn(v, ss, bb));
    }
}

// The same sums with the nibble under the exponent byte 0x4B (the float 2^23 + q, minus
// 2^23): any scale.
__device__ __forceinline__ void accumulate_word_m(uint32_t w, float2 ss, float2 bb, float2 (&acc)[4])
{
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    const float2 m23 = make_float2(-kTwo23, -kTwo23);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t sel = 0x7440u | (uint32_t)b;
        const float2 v = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, sel)),
                                                __uint_as_float(__byte_perm(hi, 0x4B000000u, sel))), m23);
        acc[b] = __fadd2_rn(acc[b], __ffma2_rn(v, ss, bb));
    }
}

// Scale and bias of a row as floats; an id outside the table (ok false) gets 0 and 0,
// so its row adds +0 (the sums never hold -0).
__device__ __forceinline__ void row_sb(uint32_t sbw, bool ok, float &S, float &B)
{
    sbw = ok ? sbw : 0u;
    S = __half2float(__ushort_as_half((unsigned short)(sbw & 0xffffu)));
    B = __half2float(__ushort_as_half((unsigned short)(sbw >> 16)));
}

// Sums the ids at positions q, q + step, ... < p1 into acc2, four loads in flight, with
// no branch per id: an out-of-range id (reported in `bad`) reads row 0 and adds +0.
// The table must have a row. A group whose rows all have |scale| < 1/2 takes the
// scaled-subnormal decode, any other the exponent-byte decode.
template <int E>
__device__ __forceinline__ void accumulate_ids(const int32_t *__restrict__ indices, int32_t q, int32_t p1,
                                               int step, const TableView &tv, float2 (&acc2)[E / 2],
                                               bool &bad)
{
    using V = typename CodeVec<E>::T;
    // the ids of the next group of four are loaded while the current group is summed
    uint32_t nxt[4];
    if (q + 3 * step < p1) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
            nxt[u] = (uint32_t)__ldg(indices + q + u * step);
    }
    for (; q + 3 * step < p1; q += 4 * step) {
        uint32_t id[4];
        bool ok[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            ok[u] = nxt[u] < tv.n_rows;
            bad |= !ok[u];
            id[u] = ok[u] ? nxt[u] : 0u;
        }
        V w[4];
        uint32_t sbw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            w[u] = __ldg(reinterpret_cast<const V *>(tv.codes + (uint64_t)id[u] * tv.ld));
            sbw[u] = __ldg(tv.sb + id[u]);
        }
        if (q + 7 * step < p1) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                nxt[u] = (uint32_t)__ldg(indices + q + (4 + u) * step);
        }
        float S[4], B[4];
        bool small = true;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            row_sb(sbw[u], ok[u], S[u], B[u]);
            small &= fabsf(S[u]) < 0.5f;
        }
        if (small) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float Sp = scale_up(S[u]);
                const float2 ss = make_float2(Sp, Sp), bb = make_float2(B[u], B[u]);
#pragma unroll
                for (int i = 0; i < E / 8; ++i)
                    accumulate_word_d(CodeVec<E>::word(w[u], i), ss, bb, *reinterpret_cast<float2(*)[4]>(&acc2[4 * i]));
            }
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 ss = make_float2(S[u], S[u]), bb = make_float2(B[u], B[u]);
#pragma unroll
                for (int i = 0; i < E / 8; ++i)
                    accumulate_word_m(CodeVec<E>::word(w[u], i), ss, bb, *reinterpret_cast<float2(*)[4]>(&acc2[4 * i]));
            }
        }
    }
    for (; q < p1; q += step) {
        const uint32_t v = (uint32_t)__ldg(indices + q);
        const bool ok = v < tv.n_rows;
        bad |= !ok;
        const uint32_t id = ok ? v : 0u;
        const V w = __ldg(reinterpret_cast<const V *>(tv.codes + (uint64_t)id * tv.ld));
        float S, B;
        row_sb(__ldg(tv.sb + id), ok, S, B);
        const float2 ss = make_float2(S, S), bb = make_float2(B, B);
#pragma unroll
        for (int i = 0; i < E / 8; ++i)
            accumulate_word_m(CodeVec<E>::word(w, i), ss, bb, *reinterpret_cast<float2(*)[4]>(&acc2[4 * i]));
    }
}

__device__ __forceinline__ void clamp_bag(int32_t &p, int32_t &p1, int32_t n_ids, bool report, uint32_t *flags)
{
    if (p1 < p || p < 0 || p1 > n_ids) {
        if (report)
            raise_flag(flags, DQ_FLAG_BAD_OFFSETS);
        p = min(max(p, 0), n_ids);
        p1 = max(min(p1, n_ids), p);
    }
}

// Long bags: IS id strides per element group, reduce-scatter, contiguous row stores.
template <int E, int IS, class D>
__device__ __forceinline__ void bag_tiles_long(const BagTables &tabs, const BagArgs &a, const D &dst,
                                               uint32_t total, int32_t n_ids)
{
    const int EG = a.d / E;
    const int G = EG * IS;     // lanes per bag, a power of two <= 32
    const uint32_t bags_per_block = kBagThreads / G;
    const int lg = threadIdx.x % G, lb = threadIdx.x / G;
    const int is = lg % IS, eg = lg / IS;
    const uint32_t batch = (uint32_t)a.batch;
    for (uint32_t tile = blockIdx.x; (uint64_t)tile * bags_per_block < total; tile += gridDim.x) {
        const uint32_t g = tile * bags_per_block + lb;
        const bool live = g < total;
        const int t = live ? (int)div_batch(g, a.div) : 0;
        const int b = live ? (int)(g - (uint32_t)t * batch) : 0;
        int32_t p = 0, p1 = 0;
        if (live) {
            p = __ldg(a.offsets + g);
            p1 = __ldg(a.offsets + g + 1);
            clamp_bag(p, p1, n_ids, lg == 0, a.flags);
        }
        const TableView tv = table_view(tabs, t, eg, E);
        float2 acc2[E / 2];
#pragma unroll
        for (int k = 0; k < E / 2; ++k)
            acc2[k] = make_float2(0.0f, 0.0f);
        bool bad = false;
        if (tv.n_rows > 0)
            accumulate_ids<E>(a.indices, p + is, p1, IS, tv, acc2, bad);
        else
            bad = p1 > p;
        if (bad)
            raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
        float acc[E];
#pragma unroll
        for (int k = 0; k < E / 2; ++k) {
            acc[2 * k] = acc2[k].x;
            acc[2 * k + 1] = acc2[k].y;
        }
        reduce_scatter<E, IS>(acc, is);
        if (live) {
            constexpr int C = E / IS;  // finished sums owned by this lane
            float *o = bag_row(tabs, a, dst, t, b) + eg * E + is * C;
            if constexpr (C % 4 == 0) {
#pragma unroll
                for (int k = 0; k < C; k += 4)
                    reinterpret_cast<float4 *>(o)[k / 4] = make_float4(acc[k], acc[k + 1], acc[k + 2], acc[k + 3]);
            } else if constexpr (C == 2) {
                *reinterpret_cast<float2 *>(o) = make_float2(acc[0], acc[1]);
            } else {
                o[0] = acc[0];
            }
        }
    }
}

// What a lane fetches ahead for one bag of the one-hot layout: its offsets and the id
// at the bag's own position g (where a one-hot bag keeps its id when every bag is).
struct ShortAhead {
    int32_t p, p1, id;
};

__device__ __forceinline__ ShortAhead short_ahead(const BagArgs &a, uint64_t g, uint32_t total, int32_t n_ids)
{
    ShortAhead s{0, 0, 0};
    if (g < total) {
        s.p = __ldg(a.offsets + g);
        s.p1 = __ldg(a.offsets + g + 1);
        s.id = (int64_t)g < n_ids ? __ldg(a.indices + g) : 0;
    }
    return s;
}

// The code bytes of EL elements (one lane's chunk of a row in the one-hot layout).
template <int EL>
struct ChunkVec;
template <>
struct ChunkVec<4> {
    using T = uint16_t;
    static __device__ __forceinline__ uint32_t word(const T &v, int) { return v; }
};
template <>
struct ChunkVec<8> {
    using T = uint32_t;
    static __device__ __forceinline__ uint32_t word(const T &v, int) { return v; }
};
template <>
struct ChunkVec<16> {
    using T = uint2;
    static __device__ __forceinline__ uint32_t word(const T &v, int i) { return i == 0 ? v.x : v.y; }
};
template <>
struct ChunkVec<32> {
    using T = uint4;
    static __device__ __forceinline__ uint32_t word(const T &v, int i)
    {
        return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
    }
};

// The EL dequantized values fma(q, scale, bias) of a chunk, as EL / 4 float4 (nibbles
// to floats by byte permutes under the exponent byte, as accumulate_word_m).
template <int EL>
__device__ __forceinline__ void dequant_chunk_to(const typename ChunkVec<EL>::T &c, uint32_t sbw, float4 (&x)[EL / 4])
{
    const float2 m23 = make_float2(-kTwo23, -kTwo23);
    const float S = __half2float(__ushort_as_half((unsigned short)(sbw & 0xffffu)));
    const float B = __half2float(__ushort_as_half((unsigned short)(sbw >> 16)));
    const float2 ss = make_float2(S, S), bb = make_float2(B, B);
    constexpr int WORDS = EL >= 8 ? EL / 8 : 1;
    constexpr int BYTES = EL >= 8 ? 4 : EL / 2;
#pragma unroll
    for (int i = 0; i < WORDS; ++i) {
        const uint32_t w = ChunkVec<EL>::word(c, i);
        const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int b = 0; b < BYTES; b += 2) {
            const uint32_t s0 = 0x7440u | (uint32_t)b, s1 = 0x7440u | (uint32_t)(b + 1);
            const float2 v0 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, s0)),
                                                     __uint_as_float(__byte_perm(hi, 0x4B000000u, s0))), m23);
            const float2 v1 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, s1)),
                                                     __uint_as_float(__byte_perm(hi, 0x4B000000u, s1))), m23);
            const float2 x0 = __ffma2_rn(v0, ss, bb), x1 = __ffma2_rn(v1, ss, bb);
            x[i * 2 + b / 2] = make_float4(x0.x, x0.y, x1.x, x1.y);
        }
    }
}

// Writes the EL dequantized values of a chunk as EL / 4 streaming float4 stores.
template <int EL>
__device__ __forceinline__ void dequant_chunk_store(const typename ChunkVec<EL>::T &c, uint32_t sbw, float4 *dst)
{
    float4 x[EL / 4];
    dequant_chunk_to<EL>(c, sbw, x);
#pragma unroll
    for (int k = 0; k < EL / 4; ++k)
        __stcs(dst + k, x[k]);
}

// One bag of a warp's tile in the one-hot layout, in shared memory.
struct OnehotSlot {
    const uint8_t *code;   // the row's code bytes (kind 0)
    const uint32_t *sb;    // the row's {scale, bias}
    float *out;            // the bag's output row (nullptr past the last bag)
    uint32_t kind;         // 0: one valid id; 1: zeros (empty bag, or one invalid id); 2: two or more ids
    uint32_t pad;
};

// Short bags (average pooling < 4, e.g. one-hot lookups): a warp takes 32 consecutive
// bags, one per lane for the bookkeeping (offsets, the id, the row and output
// addresses, kept in a per-warp table in shared memory); the offsets and the id of the
// next tile's bags are loaded one tile ahead. Then every lane produces one EL-element
// chunk of a bag's output row per sub-step: LB = d / EL lanes cover a row, so a warp
// store writes 32 / LB whole rows; the loads of UNR sub-steps are issued before any is
// decoded, and a one-id bag's row is fma(q, scale, bias) written directly (no sum).
// Bags with two or more ids are then summed one at a time by the warp's first LB lanes.
template <int EL, class D>
__device__ __forceinline__ void bag_tiles_onehot(const BagTables &tabs, const BagArgs &a, const D &dst,
                                                 uint32_t total, int32_t n_ids, OnehotSlot *slots)
{
    using CV = typename ChunkVec<EL>::T;
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int UNR = EL >= 16 ? 4 : 8;         // sub-steps whose loads are in flight together
    const int LB = a.d / EL;                      // lanes per row, a power of two <= 32
    const int lb_bits = 31 - __clz(LB);
    const int BPS = 32 >> lb_bits;                // bags per sub-step
    const int lane = threadIdx.x & 31;
    const int c = lane & (LB - 1);
    const int bsub = lane >> lb_bits;
    const uint64_t wpb = blockDim.x >> 5;
    const uint64_t stride = (uint64_t)gridDim.x * wpb * 32;
    const uint32_t batch = (uint32_t)a.batch;

    uint64_t g0 = ((uint64_t)blockIdx.x * wpb + (threadIdx.x >> 5)) * 32;
    ShortAhead nxt = short_ahead(a, g0 + lane, total, n_ids);
    for (; g0 < total; g0 += stride) {
        const ShortAhead cur = nxt;
        nxt = short_ahead(a, g0 + stride + lane, total, n_ids);
        const uint64_t g = g0 + lane;
        OnehotSlot sl{nullptr, nullptr, nullptr, 1u, 0u};
        if (g < total) {
            int32_t p = cur.p, p1 = cur.p1;
            clamp_bag(p, p1, n_ids, true, a.flags);
            const int t = (int)div_batch((uint32_t)g, a.div);
            const int b = (int)((uint32_t)g - (uint32_t)t * batch);
            sl.out = bag_row(tabs, a, dst, t, b);
            if (p1 == p + 1) {
                const uint32_t id = (int64_t)p == (int64_t)g ? (uint32_t)cur.id : (uint32_t)__ldg(a.indices + p);
                if ((int64_t)id < tabs.n_rows[t]) {
                    sl.code = tabs.codes[t] + (uint64_t)id * (uint64_t)tabs.codes_ld[t];
                    sl.sb = reinterpret_cast<const uint32_t *>(tabs.scale_bias[t]) + id;
                    sl.kind = 0u;
                } else {
                    raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
                }
            } else if (p1 > p) {
                sl.kind = 2u;
            }
        }
        slots[lane] = sl;
        __syncwarp();
        for (int s0 = 0; s0 < LB; s0 += UNR) {
            CV w[UNR];
            uint32_t sbw[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int s = s0 + u;
                if (s < LB) {
                    const OnehotSlot &q = slots[s * BPS + bsub];
                    if (q.kind == 0u) {
                        w[u] = __ldg(reinterpret_cast<const CV *>(q.code) + c);
                        sbw[u] = __ldg(q.sb);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int s = s0 + u;
                if (s < LB) {
                    const OnehotSlot &q = slots[s * BPS + bsub];
                    float4 *dst = reinterpret_cast<float4 *>(q.out + c * EL);
                    if (q.kind == 0u) {
                        dequant_chunk_store<EL>(w[u], sbw[u], dst);
                    } else if (q.kind == 1u && q.out != nullptr) {
#pragma unroll
                        for (int j = 0; j < EL / 4; ++j)
                            __stcs(dst + j, make_float4(0.0f, 0.0f, 0.0f, 0.0f));
                    }
                }
            }
        }
        // bags of two or more ids, one at a time: lanes 0..LB-1 sum their chunks in id order
        uint32_t multi = __ballot_sync(FULL, sl.kind == 2u);
        while (multi) {
            const int j = __ffs(multi) - 1;
            multi &= multi - 1;
            const uint64_t gj = g0 + j;
            int32_t p = __ldg(a.offsets + gj), p1 = __ldg(a.offsets + gj + 1);
            clamp_bag(p, p1, n_ids, false, a.flags);
            const int t = (int)div_batch((uint32_t)gj, a.div);
            const TableView tv = table_view(tabs, t, 0, 0);
            float acc[EL];
#pragma unroll
            for (int k = 0; k < EL; ++k)
                acc[k] = 0.0f;
            bool bad = false;
            if (lane < LB) {
                for (int32_t q0 = p; q0 < p1; q0 += 4) {   // four ids' rows in flight, added in id order
                    uint32_t id[4];
                    CV cw[4];
                    uint32_t sbw[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        id[u] = q0 + u < p1 ? (uint32_t)__ldg(a.indices + q0 + u) : 0xffffffffu;
                        if (id[u] < tv.n_rows) {
                            cw[u] = __ldg(reinterpret_cast<const CV *>(tv.codes + (uint64_t)id[u] * tv.ld) + c);
                            sbw[u] = __ldg(tv.sb + id[u]);
                        } else if (q0 + u < p1) {
                            bad = true;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (id[u] >= tv.n_rows)
                            continue;
                        float4 x4[EL / 4];
                        dequant_chunk_to<EL>(cw[u], sbw[u], x4);
#pragma unroll
                        for (int k = 0; k < EL / 4; ++k) {
                            acc[4 * k] = __fadd_rn(acc[4 * k], x4[k].x);
                            acc[4 * k + 1] = __fadd_rn(acc[4 * k + 1], x4[k].y);
                            acc[4 * k + 2] = __fadd_rn(acc[4 * k + 2], x4[k].z);
                            acc[4 * k + 3] = __fadd_rn(acc[4 * k + 3], x4[k].w);
                        }
                    }
                }
                float4 *dst = reinterpret_cast<float4 *>(slots[j].out + c * EL);
#pragma unroll
                for (int k = 0; k < EL / 4; ++k)
                    dst[k] = make_float4(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
            }
            if (__any_sync(FULL, bad) && lane == 0)
                raise_flag(a.flags, DQ_FLAG_BAD_INDEX);
        }
        __syncwarp();   // the slots are rewritten by the next tile
    }
}

// E1: elements per lane chunk of the one-hot layout; E, ISL: elements per lane and
// id strides of the long layout. The kernel reads the id count (the last offset) and
// takes the long layout when bags average 4 ids or more.
template <int E1, int E, int ISL, class D>
__global__ void __launch_bounds__(kBagThreads, E == 16 ? 4 : 1) embbag_kernel(const __grid_constant__ BagTables tabs,
                                                                             const BagArgs a,
                                                                             const __grid_constant__ D dst)
{
    __shared__ __align__(16) OnehotSlot slots[kBagThreads / 32][32];
    const int64_t total = (int64_t)a.T * a.batch;
    const int32_t n_ids = max(__ldg(a.offsets + total), 0);
    if (ISL > 1 && (int64_t)n_ids >= 4 * total)   // average pooling >= 4: split ids over lanes
        bag_tiles_long<E, ISL>(tabs, a, dst, (uint32_t)total, n_ids);
    else
        bag_tiles_onehot<E1>(tabs, a, dst, (uint32_t)total, n_ids, slots[threadIdx.x >> 5]);
}

// any d, any alignment: one warp per bag, lanes stride over the elements
__global__ void __launch_bounds__(256) embbag_generic_kernel(const __grid_constant__ BagTables tabs,
                                                             const BagArgs a, const __grid_constant__ BagDest dst)
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
    float *o = bag_row(tabs, a, dst, t, b);
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

// D: BagDest (rows into the owners' buffers) or NoDest (rows into out). Separate
// instantiations, so that the plain lookup's parameters and registers stay as they are.
template <class D>
void launch_fast(const BagTables &tabs, const BagArgs &a, const D &dst, int E, int isl, unsigned grid,
                 cudaStream_t stream)
{
    if (E == 32)
        embbag_kernel<32, 32, 1><<<grid, kBagThreads, 0, stream>>>(tabs, a, dst);   // d = 1024
    else if (isl == 8)
        embbag_kernel<4, 16, 8><<<grid, kBagThreads, 0, stream>>>(tabs, a, dst);    // d = 16, 32, 64
    else if (isl == 4)
        embbag_kernel<4, 16, 4><<<grid, kBagThreads, 0, stream>>>(tabs, a, dst);    // d = 128
    else if (isl == 2)
        embbag_kernel<8, 16, 2><<<grid, kBagThreads, 0, stream>>>(tabs, a, dst);    // d = 256
    else
        embbag_kernel<16, 16, 1><<<grid, kBagThreads, 0, stream>>>(tabs, a, dst);   // d = 512
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
    const bool fast = a.d % 4 == 0 && a.codes_ld % 2 == 0 && a.out_ld % 4 == 0 &&
                      (reinterpret_cast<uintptr_t>(a.codes) & 1) == 0 &&
                      (reinterpret_cast<uintptr_t>(a.out) & 15) == 0 &&
                      (reinterpret_cast<uintptr_t>(a.scale_bias) & 3) == 0;
    if (fast)
    {
        const int cpr = a.d / 4;   // float4 chunks per row; a power of two is a shift
        const int lg = (cpr & (cpr - 1)) == 0 ? 31 - __builtin_clz((unsigned)cpr) : -1;
        dequant16_kernel<<<grid_for(a.n * cpr, 256, num_sms), 256, 0, stream>>>(a, lg);
    }
    else
        dequant_generic_kernel<<<grid_for(a.n * ((a.d + 1) / 2), 256, num_sms), 256, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_embbag(const BagTables &tabs, const BagArgs &a, const BagDest &dst, int num_sms,
                          cudaStream_t stream)
{
    const int64_t total = (int64_t)a.T * a.batch;
    int E = 0;
    if (a.d % 16 == 0 && a.d / 16 <= 32 && ((a.d / 16) & (a.d / 16 - 1)) == 0)
        E = 16;
    else if (a.d % 32 == 0 && a.d / 32 <= 32 && ((a.d / 32) & (a.d / 32 - 1)) == 0)
        E = 32;
    bool fast = E != 0 && (reinterpret_cast<uintptr_t>(a.out) & 15) == 0;
    for (int r = 0; fast && r < dst.n; ++r)   // rows stored into the owners' buffers
        fast = (reinterpret_cast<uintptr_t>(dst.ptr[r]) & 15) == 0;
    for (int t = 0; fast && t < a.T; ++t)
        fast = tabs.codes_ld[t] % (E / 2) == 0 && (reinterpret_cast<uintptr_t>(tabs.codes[t]) % (E / 2)) == 0 &&
               (reinterpret_cast<uintptr_t>(tabs.scale_bias[t]) & 3) == 0;
    if (fast) {
        const int EG = a.d / E;
        const int isl = EG <= 4 ? 8 : EG == 8 ? 4 : EG == 16 ? 2 : 1;
        const int64_t long_tiles = (total + kBagThreads / (EG * isl) - 1) / (kBagThreads / (EG * isl));
        const int64_t onehot_blocks = (total + kBagThreads - 1) / kBagThreads;   // 32 bags per warp
        const int64_t need = long_tiles > onehot_blocks ? long_tiles : onehot_blocks;
        const int64_t cap = (int64_t)num_sms * 8;
        const unsigned grid = (unsigned)(need < cap ? need : cap);
        if (dst.n > 0)
            launch_fast(tabs, a, dst, E, isl, grid, stream);
        else
            launch_fast(tabs, a, NoDest{0}, E, isl, grid, stream);
    } else {
        const int64_t grid = (total * 32 + 255) / 256;
        embbag_generic_kernel<<<(unsigned)grid, 256, 0, stream>>>(tabs, a, dst);
    }
    return cudaGetLastError();
}

} // namespace dq
