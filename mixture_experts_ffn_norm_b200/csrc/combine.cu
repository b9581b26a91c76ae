// Weighted combine fused with the shared-expert add and the output cast.
//
// "MoE update" page, MoE.forward excerpt: y (float32) += expert(x[idx]) * weights[idx, top];
// y += shared_experts(x); the result is y.type_as(x).  "Add shared output" page:
// delta_ffn = y_routed + y_shared, shape [B, T, d].
//
// CTA (t, part) gathers part `part` of token t's k expert-output rows (bf16, written by the second
// grouped GEMM at the rows the permutation assigned), sums them with the router weights in
// float32 in slot order, adds the shared expert's row and rounds once to bf16.  A token's row is
// split over several CTAs when there are few tokens (decode), so that every SM has loads in flight;
// each thread issues the loads of up to 8 slots before their FMAs.
// Also here: the same combine with the next block's RMSNorm fused in, the float32 partial of an
// expert slice, and the final bf16 cast of the reduced partials.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 128;

__device__ __forceinline__ void add_bf16x8(float (&a)[8], const uint4 v, float w) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        a[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), a[2 * i]);
        a[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), a[2 * i + 1]);
    }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(a))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(b))) << 16);
}

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const uint4* __restrict__ y, const uint4* __restrict__ ysh, const int* __restrict__ row_of,
               const float* __restrict__ w, int nv, int k, uint4* __restrict__ out) {
    __shared__ int rows[kMaxExperts];
    __shared__ float ws[kMaxExperts];
    const int t = blockIdx.x;
    for (int j = threadIdx.x; j < k; j += kCombineThreads) {
        rows[j] = row_of[static_cast<size_t>(t) * k + j];
        ws[j] = w[static_cast<size_t>(t) * k + j];
    }
    __syncthreads();
    const int per = (nv + gridDim.y - 1) / gridDim.y;
    const int v0 = blockIdx.y * per, v1 = min(nv, v0 + per);
    for (int v = v0 + threadIdx.x; v < v1; v += kCombineThreads) {
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < k; j0 += 8) {
            uint4 b[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (j0 + i < k) b[i] = y[static_cast<size_t>(rows[j0 + i]) * nv + v];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (j0 + i < k) add_bf16x8(a, b[i], ws[j0 + i]);
        }
        if (ysh) {
            const uint4 s = ysh[static_cast<size_t>(t) * nv + v];
            const uint32_t u[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[2 * i] += __uint_as_float(u[i] << 16);
                a[2 * i + 1] += __uint_as_float(u[i] & 0xFFFF0000u);
            }
        }
        out[static_cast<size_t>(t) * nv + v] = make_uint4(pack2(a[0], a[1]), pack2(a[2], a[3]), pack2(a[4], a[5]),
                                                          pack2(a[6], a[7]));
    }
}

constexpr int kNextThreads = 128;
constexpr int kNextVec = 8;   // 16-byte vectors per thread: d <= 128 * 8 * 8 = 8192

// The combine with the next block's attn_norm fused in ("MoE update" page, Block excerpt: the
// residual addition happens inside the next normalisation, `x, residual = self.attn_norm(x,
// residual)`; RMSNorm excerpt for the arithmetic).  One CTA per token: the MoE update
// delta = bf16(sum_j w_j y_j + y_shared) is formed exactly as combine_kernel forms it (optionally
// stored), then s = fp32(delta) + fp32(residual) with the block's new residual read from `resid`,
// `resid` <- bf16(s), and xn_next = bf16(g * (s * rsqrt(mean(s^2) + eps))) with the same exact
// mean of squares and IEEE sqrt / divide as the ffn_norm kernel.  The row stays in registers.
__global__ void __launch_bounds__(kNextThreads)
combine_next_norm_kernel(const uint4* __restrict__ y, const uint4* __restrict__ ysh, const int* __restrict__ row_of,
                         const float* __restrict__ w, int nv, int k, const float* __restrict__ gain, float eps, int d,
                         uint4* __restrict__ out, uint4* __restrict__ resid, uint4* __restrict__ xn_next) {
    __shared__ int rows[kMaxExperts];
    __shared__ float ws[kMaxExperts];
    __shared__ double red_hi[kNextThreads / 32], red_lo[kNextThreads / 32];
    __shared__ float rinv_sh;
    const int t = blockIdx.x;
    for (int j = threadIdx.x; j < k; j += kNextThreads) {
        rows[j] = row_of[static_cast<size_t>(t) * k + j];
        ws[j] = w[static_cast<size_t>(t) * k + j];
    }
    __syncthreads();
    const size_t row = static_cast<size_t>(t) * nv;
    float sv[kNextVec][8];
    double hi = 0.0, lo = 0.0;
#pragma unroll
    for (int i = 0; i < kNextVec; ++i) {
        const int v = threadIdx.x + kNextThreads * i;
        if (v >= nv) continue;
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < k; j0 += 8) {
            uint4 b[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (j0 + q < k) b[q] = y[static_cast<size_t>(rows[j0 + q]) * nv + v];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (j0 + q < k) add_bf16x8(a, b[q], ws[j0 + q]);
        }
        if (ysh) {
            const uint4 sh = ysh[row + v];
            const uint32_t u[4] = {sh.x, sh.y, sh.z, sh.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                a[2 * e] += __uint_as_float(u[e] << 16);
                a[2 * e + 1] += __uint_as_float(u[e] & 0xFFFF0000u);
            }
        }
        const uint4 dq = make_uint4(pack2(a[0], a[1]), pack2(a[2], a[3]), pack2(a[4], a[5]), pack2(a[6], a[7]));
        if (out) out[row + v] = dq;
        const uint4 r = resid[row + v];
        const uint32_t du[4] = {dq.x, dq.y, dq.z, dq.w}, ru[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sv[i][2 * e] = __fadd_rn(__uint_as_float(du[e] << 16), __uint_as_float(ru[e] << 16));
            sv[i][2 * e + 1] = __fadd_rn(__uint_as_float(du[e] & 0xFFFF0000u), __uint_as_float(ru[e] & 0xFFFF0000u));
        }
        resid[row + v] = make_uint4(pack2(sv[i][0], sv[i][1]), pack2(sv[i][2], sv[i][3]), pack2(sv[i][4], sv[i][5]),
                                    pack2(sv[i][6], sv[i][7]));
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double p = __dmul_rn(static_cast<double>(sv[i][e]), static_cast<double>(sv[i][e]));   // exact
            double sum, err;
            two_sum(hi, p, sum, err);
            hi = sum;
            lo = __dadd_rn(lo, err);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const double h2 = __shfl_xor_sync(0xFFFFFFFFu, hi, off);
        const double l2 = __shfl_xor_sync(0xFFFFFFFFu, lo, off);
        dd_add(hi, lo, h2, l2);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red_hi[warp] = hi;
        red_lo[warp] = lo;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double H = red_hi[0], Lo = red_lo[0];
        for (int q = 1; q < kNextThreads / 32; ++q) dd_add(H, Lo, red_hi[q], red_lo[q]);
        const float var = __double2float_rn(__ddiv_rn(__dadd_rn(H, Lo), static_cast<double>(d)));
        rinv_sh = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps)));
    }
    __syncthreads();
    const float rinv = rinv_sh;
#pragma unroll
    for (int i = 0; i < kNextVec; ++i) {
        const int v = threadIdx.x + kNextThreads * i;
        if (v >= nv) continue;
        const float4 g0 = reinterpret_cast<const float4*>(gain)[2 * v];
        const float4 g1 = reinterpret_cast<const float4*>(gain)[2 * v + 1];
        const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(gv[e], __fmul_rn(sv[i][e], rinv));   // weight * (x * rsqrt)
        xn_next[row + v] = make_uint4(pack2(o[0], o[1]), pack2(o[2], o[3]), pack2(o[4], o[5]), pack2(o[6], o[7]));
    }
}

// Expert slice (the pages' expert-parallel MoE.forward: each rank adds the outputs of its own
// experts into a float32 y, then `dist.all_reduce(y)`): the token's slots routed to experts in
// [ebeg, eend), weighted, in slot order, plus the shared expert's row when it ran on this rank;
// float32 out, no rounding (the sum over ranks is rounded once after the reduction).
__global__ void __launch_bounds__(kCombineThreads)
combine_partial_kernel(const uint4* __restrict__ y, const uint4* __restrict__ ysh, const int* __restrict__ row_of,
                       const int* __restrict__ idx, const float* __restrict__ w, int nv, int k, int ebeg, int eend,
                       float4* __restrict__ out) {
    __shared__ int rows[kMaxExperts];
    __shared__ float ws[kMaxExperts];
    const int t = blockIdx.x;
    for (int j = threadIdx.x; j < k; j += kCombineThreads) {
        const int e = idx[static_cast<size_t>(t) * k + j];
        rows[j] = row_of[static_cast<size_t>(t) * k + j];
        ws[j] = (e >= ebeg && e < eend) ? w[static_cast<size_t>(t) * k + j] : 0.0f;   // 0: not this rank's
    }
    __syncthreads();
    const int per = (nv + gridDim.y - 1) / gridDim.y;
    const int v0 = blockIdx.y * per, v1 = min(nv, v0 + per);
    for (int v = v0 + threadIdx.x; v < v1; v += kCombineThreads) {
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < k; ++j)
            if (ws[j] != 0.0f) add_bf16x8(a, y[static_cast<size_t>(rows[j]) * nv + v], ws[j]);
        if (ysh) {
            const uint4 sh = ysh[static_cast<size_t>(t) * nv + v];
            const uint32_t u[4] = {sh.x, sh.y, sh.z, sh.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                a[2 * e] += __uint_as_float(u[e] << 16);
                a[2 * e + 1] += __uint_as_float(u[e] & 0xFFFF0000u);
            }
        }
        float4* o = out + (static_cast<size_t>(t) * nv + v) * 2;
        o[0] = make_float4(a[0], a[1], a[2], a[3]);
        o[1] = make_float4(a[4], a[5], a[6], a[7]);
    }
}

}  // namespace

namespace {
// y [n] float32 -> bf16, round to nearest even (the layer's output cast, `y.type_as(x)`)
__global__ void round_bf16_kernel(const float4* __restrict__ y, uint2* __restrict__ out, int64_t n4) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 v = y[i];
        out[i] = make_uint2(pack2(v.x, v.y), pack2(v.z, v.w));
    }
}
}  // namespace

cudaError_t launch_round_bf16(const float* y, void* out, int64_t n, cudaStream_t s) {
    const int64_t n4 = n / 4;
    const int grid = static_cast<int>(std::min<int64_t>((n4 + 255) / 256, 8 * num_sms()));
    round_bf16_kernel<<<std::max(grid, 1), 256, 0, s>>>(reinterpret_cast<const float4*>(y), static_cast<uint2*>(out), n4);
    return cudaGetLastError();
}

cudaError_t launch_combine_partial(const Layout& L, float* y_partial, int ebeg, int eend, bool shared_here,
                                   uint8_t* ws, cudaStream_t s) {
    const int nv = L.d / 8;
    int parts = (4 * num_sms() + L.T - 1) / L.T;
    parts = std::max(1, std::min({parts, 8, nv / kCombineThreads}));
    combine_partial_kernel<<<dim3(L.T, parts), kCombineThreads, 0, s>>>(
        reinterpret_cast<const uint4*>(ws + L.y),
        (L.Is > 0 && shared_here) ? reinterpret_cast<const uint4*>(ws + L.y_sh) : nullptr,
        reinterpret_cast<const int*>(ws + L.row_of), reinterpret_cast<const int*>(ws + L.idx),
        reinterpret_cast<const float*>(ws + L.w), nv, L.k, ebeg, eend, reinterpret_cast<float4*>(y_partial));
    return cudaGetLastError();
}

cudaError_t launch_combine_next_norm(const Layout& L, void* out, const float* gain, float eps, void* resid,
                                     void* xn_next, uint8_t* ws, cudaStream_t s) {
    combine_next_norm_kernel<<<L.T, kNextThreads, 0, s>>>(
        reinterpret_cast<const uint4*>(ws + L.y), L.Is > 0 ? reinterpret_cast<const uint4*>(ws + L.y_sh) : nullptr,
        reinterpret_cast<const int*>(ws + L.row_of), reinterpret_cast<const float*>(ws + L.w), L.d / 8, L.k, gain, eps,
        L.d, static_cast<uint4*>(out), static_cast<uint4*>(resid), static_cast<uint4*>(xn_next));
    return cudaGetLastError();
}

cudaError_t launch_combine(const Layout& L, void* out, uint8_t* ws, cudaStream_t s) {
    // parts per token: enough CTAs for about four per SM, at most 8, each part >= 128 vectors
    const int nv = L.d / 8;
    int parts = (4 * num_sms() + L.T - 1) / L.T;
    parts = std::max(1, std::min({parts, 8, nv / kCombineThreads}));
    combine_kernel<<<dim3(L.T, parts), kCombineThreads, 0, s>>>(
        reinterpret_cast<const uint4*>(ws + L.y), L.Is > 0 ? reinterpret_cast<const uint4*>(ws + L.y_sh) : nullptr,
        reinterpret_cast<const int*>(ws + L.row_of), reinterpret_cast<const float*>(ws + L.w), L.d / 8, L.k,
        static_cast<uint4*>(out));
    return cudaGetLastError();
}

}  // namespace moe
