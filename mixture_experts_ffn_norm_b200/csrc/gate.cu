// Router selection.  The gate logits [T, E] come from the tensor-core GEMM (xn . Wg^T, float32
// accumulation).  The router's body is not on the pages ("MoE update" page, MoE.forward excerpt
// only shows `weights, indices = self.gate(x)`); this library reads it as: scores =
// sigmoid(logit + bias), the top_k scores win with the lower expert index first on equal
// scores, and the winners' scores are normalised to sum 1.
//
// topk_kernel: one warp per token, E <= 256 logits spread over the lanes; k+1 rounds of a
// warp-wide (value, index) argmax.  A token whose k-th and (k+1)-th float32 scores are closer
// than tau is appended to a device list.  recheck_kernel then recomputes every logit of those
// tokens in float64 (bf16 x bf16 products are exact) and re-decides the selection and weights,
// so the result only differs from exact arithmetic when the true margin is ~1e-15.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kTopkWarps = 8;

__device__ __forceinline__ bool better(float za, int ea, float zb, int eb) {
    return za > zb || (za == zb && ea < eb);
}

__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k, float tau,
            int* __restrict__ idx, float* __restrict__ wout, uint8_t* __restrict__ flag, int* __restrict__ flag_list,
            uint32_t* status) {
    __shared__ float selz[kTopkWarps][kMaxExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTopkWarps + warp;
    if (t >= T) return;
    float z[kMaxExperts / 32];
    uint32_t taken = 0;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) {
        const int e = lane + 32 * j;
        float v = -INFINITY;
        if (e < E) {
            v = logits[static_cast<size_t>(t) * E + e];
            if (bias) v = __fadd_rn(v, bias[e]);
            if (v != v) v = -INFINITY;
        }
        z[j] = v;
        if (e >= E) taken |= 1u << j;
    }
    const int rounds = k < E ? k + 1 : k;
    float znext = 0.0f;
    for (int rnd = 0; rnd < rounds; ++rnd) {
        float bz = -INFINITY;
        int be = 0x7FFFFFFF;
#pragma unroll
        for (int j = 0; j < kMaxExperts / 32; ++j) {
            const int e = lane + 32 * j;
            if (!((taken >> j) & 1u) && better(z[j], e, bz, be)) {
                bz = z[j];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float oz = __shfl_xor_sync(0xFFFFFFFFu, bz, off);
            const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
            if (better(oz, oe, bz, be)) {
                bz = oz;
                be = oe;
            }
        }
        if (rnd < k) {
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
            if (lane == 0) {
                idx[static_cast<size_t>(t) * k + rnd] = be;
                selz[warp][rnd] = bz;
            }
        } else {
            znext = bz;
        }
    }
    __syncwarp();
    if (lane == 0) {
        float sum = 0.0f;
        for (int j = 0; j < k; ++j) {
            const float s = 1.0f / (1.0f + expf(-selz[warp][j]));
            selz[warp][j] = s;
            sum += s;
        }
        for (int j = 0; j < k; ++j) wout[static_cast<size_t>(t) * k + j] = selz[warp][j] / sum;
        uint8_t f = 0;
        if (k < E) {
            const float snext = 1.0f / (1.0f + expf(-znext));
            if (!(selz[warp][k - 1] - snext >= tau)) {
                f = 1;
                const int slot = atomicAdd(reinterpret_cast<int*>(status + kStatusFlagCount), 1);
                flag_list[slot] = t;
            }
        }
        flag[t] = f;
    }
}

constexpr int kRecheckThreads = 256;

__global__ void __launch_bounds__(kRecheckThreads)
recheck_kernel(const uint16_t* __restrict__ xn, const uint16_t* __restrict__ gw, const float* __restrict__ bias,
               int d, int E, int k, const int* __restrict__ flag_list, const uint32_t* status,
               int* __restrict__ idx, float* __restrict__ wout) {
    extern __shared__ double xd[];               // d doubles: the token's normed input
    __shared__ double s64[kMaxExperts];
    __shared__ int taken[kMaxExperts];
    const int count = *reinterpret_cast<const volatile int*>(status + kStatusFlagCount);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = blockIdx.x; i < count; i += gridDim.x) {
        const int t = flag_list[i];
        for (int c = threadIdx.x; c < d; c += kRecheckThreads)
            xd[c] = static_cast<double>(__uint_as_float(static_cast<uint32_t>(xn[static_cast<size_t>(t) * d + c]) << 16));
        __syncthreads();
        for (int e = warp; e < E; e += kRecheckThreads / 32) {
            double acc = 0.0;
            const uint16_t* wr = gw + static_cast<size_t>(e) * d;
            for (int c = lane; c < d; c += 32)
                acc = fma(xd[c], static_cast<double>(__uint_as_float(static_cast<uint32_t>(wr[c]) << 16)), acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
            if (lane == 0) {
                const double zz = acc + (bias ? static_cast<double>(bias[e]) : 0.0);
                s64[e] = 1.0 / (1.0 + exp(-zz));
                taken[e] = 0;
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            double sum = 0.0;
            int sel[kMaxExperts];
            for (int j = 0; j < k; ++j) {
                int best = -1;
                for (int e = 0; e < E; ++e)
                    if (!taken[e] && (best < 0 || s64[e] > s64[best])) best = e;
                taken[best] = 1;
                sel[j] = best;
                sum += s64[best];
            }
            for (int j = 0; j < k; ++j) {
                idx[static_cast<size_t>(t) * k + j] = sel[j];
                wout[static_cast<size_t>(t) * k + j] = static_cast<float>(s64[sel[j]] / sum);
            }
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_topk(const Layout& L, const float* gate_bias, float tau, uint8_t* ws, cudaStream_t s) {
    const int grid = (L.T + kTopkWarps - 1) / kTopkWarps;
    topk_kernel<<<grid, kTopkWarps * 32, 0, s>>>(
        reinterpret_cast<const float*>(ws + L.logits), gate_bias, L.T, L.E, L.k, tau,
        reinterpret_cast<int*>(ws + L.idx), reinterpret_cast<float*>(ws + L.w), ws + L.flag,
        reinterpret_cast<int*>(ws + L.flag_list), reinterpret_cast<uint32_t*>(ws + L.status));
    return cudaGetLastError();
}

cudaError_t launch_recheck(const Layout& L, const void* gate_w, const float* gate_bias, uint8_t* ws,
                           cudaStream_t s) {
    const size_t smem = static_cast<size_t>(L.d) * sizeof(double);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(recheck_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int grid = std::min(L.T, 2 * num_sms());
    recheck_kernel<<<grid, kRecheckThreads, smem, s>>>(
        reinterpret_cast<const uint16_t*>(ws + L.xn), static_cast<const uint16_t*>(gate_w), gate_bias, L.d, L.E,
        L.k, reinterpret_cast<const int*>(ws + L.flag_list), reinterpret_cast<const uint32_t*>(ws + L.status),
        reinterpret_cast<int*>(ws + L.idx), reinterpret_cast<float*>(ws + L.w));
    return cudaGetLastError();
}

}  // namespace moe
