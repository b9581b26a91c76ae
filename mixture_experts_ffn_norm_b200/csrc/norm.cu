// ffn_norm: RMSNorm with the residual add fused in, plus the per-token 1x128 FP8 quant of the
// normed activations that the FP8 expert GEMMs consume.
//
// "MoE update" page, RMSNorm.forward excerpt: s = x.float() + residual.float();
// var = mean(s^2); s * rsqrt(var + eps); weight * s; the normed value and the new residual are
// cast back to x's dtype.  The mean is taken as the exact sum of the squares rounded to double
// (double-double accumulation: every float32 square is exact in double, the TwoSum error terms
// carry the rest), divided by d in double and rounded to float32, so the result does not depend
// on the reduction order.  rsqrt = IEEE sqrt then IEEE divide, and no multiply is contracted
// into an FMA, so every float32 step is the correctly rounded one.
//
// One CTA per token, 128 threads, 16-byte vector loads and stores, the row held in registers
// between the two passes.  Memory-bound: reads 4d bytes, writes 4d (+d + d/32).  d <= 8192.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(a));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(b));
    return lo | (hi << 16);
}

constexpr int kNormThreads = 128;
constexpr int kMaxVec = 8;          // 16-byte vectors per thread: d <= 128 * 8 * 8 = 8192

// a / b from y = the correctly rounded 1/b and one FMA-residual correction: the correctly rounded
// quotient (the same value as an IEEE divide), several times cheaper
__device__ __forceinline__ float div_by_rcp(float a, float b, float y) {
    const float q = a * y;
    return fmaf(fmaf(-q, b, a), y, q);
}

// One CTA per token.  Every 16-byte load of the row is issued before any arithmetic, the row stays
// in registers between the two passes (no shared-memory round trip), and the group quant uses one
// reciprocal per 128-column group.
__global__ void __launch_bounds__(kNormThreads)
norm_kernel(const uint4* __restrict__ x, const uint4* __restrict__ res, const float* __restrict__ gain,
            float eps, int d, int Tpad, uint4* __restrict__ res_out, uint4* __restrict__ xn,
            uint2* __restrict__ xq, float* __restrict__ xs) {
    __shared__ double red_hi[kNormThreads / 32], red_lo[kNormThreads / 32];
    __shared__ float rinv_sh;
    const int t = blockIdx.x;
    const int nv = d >> 3;
    const size_t row = static_cast<size_t>(t) * nv;

    uint4 xa[kMaxVec], ra[kMaxVec];
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
        const int v = threadIdx.x + kNormThreads * i;
        if (v < nv) {
            xa[i] = x[row + v];
            ra[i] = res ? res[row + v] : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    float s[kMaxVec][8];
    double hi = 0.0, lo = 0.0;
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
        const int v = threadIdx.x + kNormThreads * i;
        if (v >= nv) continue;
        const uint32_t xw[4] = {xa[i].x, xa[i].y, xa[i].z, xa[i].w};
        const uint32_t rw[4] = {ra[i].x, ra[i].y, ra[i].z, ra[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            s[i][2 * j] = res ? __fadd_rn(bf16_lo(xw[j]), bf16_lo(rw[j])) : bf16_lo(xw[j]);
            s[i][2 * j + 1] = res ? __fadd_rn(bf16_hi(xw[j]), bf16_hi(rw[j])) : bf16_hi(xw[j]);
        }
        if (res)
            res_out[row + v] = make_uint4(pack_bf16(s[i][0], s[i][1]), pack_bf16(s[i][2], s[i][3]),
                                          pack_bf16(s[i][4], s[i][5]), pack_bf16(s[i][6], s[i][7]));
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const double p = __dmul_rn(static_cast<double>(s[i][j]), static_cast<double>(s[i][j]));  // exact
            double sum, err;
            two_sum(hi, p, sum, err);
            hi = sum;
            lo = __dadd_rn(lo, err);
        }
    }
    // block reduction of the double-double partial sums
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
        for (int w = 1; w < kNormThreads / 32; ++w) dd_add(H, Lo, red_hi[w], red_lo[w]);
        const double ss = __dadd_rn(H, Lo);                                  // RN64 of the sum
        const float var = __double2float_rn(__ddiv_rn(ss, static_cast<double>(d)));
        const float v = __fadd_rn(var, eps);
        rinv_sh = __fdiv_rn(1.0f, __fsqrt_rn(v));
    }
    __syncthreads();
    const float rinv = rinv_sh;

#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
        const int v = threadIdx.x + kNormThreads * i;
        if (kNormThreads * i >= nv) break;                                   // uniform across the CTA
        const bool on = v < nv;
        float y[8];
        if (on) {
            const float4 g0 = reinterpret_cast<const float4*>(gain)[2 * v];
            const float4 g1 = reinterpret_cast<const float4*>(gain)[2 * v + 1];
            const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float tt = __fmul_rn(s[i][j], rinv);                   // x * rsqrt(var + eps)
                y[j] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(gv[j], tt)));  // (weight * x) -> bf16
            }
            xn[row + v] = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                                     pack_bf16(y[6], y[7]));
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) y[j] = 0.0f;
        }
        if (xq) {
            // 1x128 group = 16 consecutive vectors = 16 consecutive lanes of this warp (nv is a multiple
            // of 32, so a warp is entirely on or off)
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(y[j]));
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
            if (on) {
                const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                const float rsc = __frcp_rn(sc);
                uint32_t q[2] = {0u, 0u};
                if (amax > 0.0f) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t c = __nv_cvt_float_to_fp8(div_by_rcp(y[j], sc, rsc), __NV_SATFINITE, __NV_E4M3);
                        q[j >> 2] |= c << (8 * (j & 3));
                    }
                }
                xq[row + v] = make_uint2(q[0], q[1]);
                if ((v & 15) == 0) xs[static_cast<size_t>(v >> 4) * Tpad + t] = sc;
            }
        }
    }
}

}  // namespace

cudaError_t launch_norm(const Layout& L, const void* x, const void* residual, const float* g, float eps,
                        void* residual_out, uint8_t* ws, cudaStream_t s) {
    norm_kernel<<<L.T, kNormThreads, 0, s>>>(
        static_cast<const uint4*>(x), static_cast<const uint4*>(residual), g, eps, L.d, L.Tpad,
        static_cast<uint4*>(residual_out), reinterpret_cast<uint4*>(ws + L.xn),
        L.act8 ? reinterpret_cast<uint2*>(ws + L.xq) : nullptr,
        L.act8 ? reinterpret_cast<float*>(ws + L.xs) : nullptr);
    return cudaGetLastError();
}

}  // namespace moe
