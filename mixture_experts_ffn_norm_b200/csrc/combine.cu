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

}  // namespace

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
