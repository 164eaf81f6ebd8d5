// dq_l2.cu -- normalized l2 error of packed rows against their binary32 originals.
//
// "Post-Training 4-bit Quantization on Embedding Tables", section 提出的方法 (proposed
// method), bullet 5: the quantization error is measured as the normalized l2 loss
// across embedding dimensions; section 主要发现 (main findings), bullet 2: the greedy
// search gives the lowest one. Per row: sqrt(sum (x - xhat)^2) / sqrt(sum x^2), with
// xhat = fma(q, scale, bias) and both sums in binary64.
//
// HBM-bound: a row is read once (4d bytes of x, (d+1)/2 code bytes, 4 bytes of
// scale/bias) by G lanes (1 to 8, fewer than the row's 4-element chunks), each taking 4
// consecutive elements per step (a 16-byte load of x and 2 code bytes); a lane works on
// one row at a time (measured faster than 2, 4 or 8 rows in flight per lane: fewer
// registers, more resident warps), and binary64 partial sums meet in an XOR butterfly.
#include "dq_internal.cuh"

namespace dq {
namespace {

// The 4 elements k0..k0+3 of a row (x and codes).
template <bool VEC>
__device__ __forceinline__ void load_chunk(const float *xr, const uint8_t *cr, int k0, int d, float (&xv)[4],
                                           unsigned (&q)[4])
{
    if (VEC) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(xr + k0));
        xv[0] = v.x;
        xv[1] = v.y;
        xv[2] = v.z;
        xv[3] = v.w;
        const unsigned c = __ldg(reinterpret_cast<const unsigned short *>(cr + k0 / 2));
        q[0] = c & 15u;
        q[1] = (c >> 4) & 15u;
        q[2] = (c >> 8) & 15u;
        q[3] = (c >> 12) & 15u;
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = k0 + j;
            xv[j] = k < d ? __ldg(xr + k) : 0.0f;
            q[j] = k < d ? (__ldg(cr + k / 2) >> (4 * (k & 1))) & 15u : 0u;
        }
    }
}

// G lanes per row, U row blocks per warp iteration (all their loads issued first).
template <int G, bool VEC, int U>
__global__ void __launch_bounds__(256) row_l2_kernel(const L2Args a)
{
    const int lane = threadIdx.x & 31;
    const int sub = lane & (G - 1);
    constexpr int kRowsPerWarp = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    double local = 0.0;
    // warp-uniform loop: every lane takes part in each iteration's shuffles
    for (int64_t base = warp * kRowsPerWarp * U; base < a.n; base += warps * kRowsPerWarp * U) {
        int64_t row[U];
        bool live[U];
        float S[U], B[U];
        double se[U], sx[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            row[u] = base + u * kRowsPerWarp + lane / G;
            live[u] = row[u] < a.n;
            const int64_t r = live[u] ? row[u] : base;
            const uint32_t sbw = __ldg(reinterpret_cast<const uint32_t *>(a.scale_bias) + r);
            S[u] = __half2float(__ushort_as_half((unsigned short)(sbw & 0xffffu)));
            B[u] = __half2float(__ushort_as_half((unsigned short)(sbw >> 16)));
            se[u] = 0.0;
            sx[u] = 0.0;
        }
        for (int k0 = 4 * sub; k0 < a.d; k0 += 4 * G) {
            float xv[U][4];
            unsigned q[U][4];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t r = live[u] ? row[u] : base;
                load_chunk<VEC>(a.x + r * a.ld, a.codes + r * a.codes_ld, k0, a.d, xv[u], q[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (VEC || k0 + j < a.d) {
                        const double xk = (double)xv[u][j];
                        const double e = xk - (double)__fmaf_rn((float)q[u][j], S[u], B[u]);
                        se[u] = __fma_rn(e, e, se[u]);
                        sx[u] = __fma_rn(xk, xk, sx[u]);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int o = 1; o < G; o <<= 1) {
                se[u] += __shfl_xor_sync(0xffffffffu, se[u], o);
                sx[u] += __shfl_xor_sync(0xffffffffu, sx[u], o);
            }
            if (live[u] && sub == 0) {
                const double err = sx[u] > 0.0 ? sqrt(se[u] / sx[u]) : (se[u] > 0.0 ? INFINITY : 0.0);
                if (a.row_err)
                    a.row_err[row[u]] = err;
                local += err;
            }
        }
    }
    if (a.err_sum) {  // one atomic per block: warp shuffles, then the block's 8 warps
        __shared__ double warp_sum[8];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
            local += __shfl_xor_sync(0xffffffffu, local, o);
        if (lane == 0)
            warp_sum[threadIdx.x >> 5] = local;
        __syncthreads();
        if (threadIdx.x == 0) {
            double t = 0.0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w)
                t += warp_sum[w];
            if (t != 0.0)
                atomicAdd(a.err_sum, t);
        }
    }
}

template <int G>
cudaError_t launch_g(const L2Args &a, int num_sms, cudaStream_t stream)
{
    const bool vec = a.d % 4 == 0 && a.ld % 4 == 0 && (reinterpret_cast<uintptr_t>(a.x) & 15) == 0 &&
                     a.codes_ld % 2 == 0 && (reinterpret_cast<uintptr_t>(a.codes) & 1) == 0;
    constexpr int kU = 1;
    const int64_t rows_per_block = 256 / G * kU;
    const int64_t need = (a.n + rows_per_block - 1) / rows_per_block;
    const int64_t cap = (int64_t)num_sms * 8;
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    if (vec)
        row_l2_kernel<G, true, kU><<<grid, 256, 0, stream>>>(a);
    else
        row_l2_kernel<G, false, kU><<<grid, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

} // namespace

cudaError_t launch_row_l2(const L2Args &a, int num_sms, cudaStream_t stream)
{
    // lanes per row: few, so that a lane takes several 4-element chunks of a row and the
    // per-row work (the binary64 butterfly over the row's lanes, the division and square
    // root) is shared by more rows per warp; two lanes read a full 32-byte sector of x
    // per step (measured on the B200: d = 16 best with one lane per row, d = 64 and 128
    // with two, d = 256 with two or four)
    const int chunks = (a.d + 3) / 4;  // 4 elements per lane and step
    if (chunks <= 4)
        return launch_g<1>(a, num_sms, stream);
    if (chunks <= 32)
        return launch_g<2>(a, num_sms, stream);
    if (chunks <= 128)
        return launch_g<4>(a, num_sms, stream);
    return launch_g<8>(a, num_sms, stream);
}

} // namespace dq
