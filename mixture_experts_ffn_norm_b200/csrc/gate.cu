// Router selection.  The gate logits [T, E] come from the tensor-core GEMM (xn . Wg^T, float32
// accumulation).  The router's body is not on the pages ("MoE update" page, MoE.forward excerpt
// only shows `weights, indices = self.gate(x)`); this library reads it as: scores =
// sigmoid(logit + bias), the top_k scores win with the lower expert index first on equal
// scores, and the winners' scores are normalised to sum 1.
//
// One warp per token.  The E <= 256 float32 logits (+ bias) are spread over the lanes and the
// top k are picked by k rounds of a warp-wide (value, lower index) argmax.  The logits GEMM
// promotes every 64-wide K stage into float32 registers, so a logit is off by ~1e-6; kCandDelta
// is far above that.  When another expert lies within kCandDelta of the k-th winner, the set
// S = {winners} U {those candidates} is re-evaluated in float64 (bf16 x bf16 products are exact in
// float64) and the top k is re-decided inside S: every expert outside S is provably below all k
// winners, so the selection is the exact one.  Such tokens are marked as re-decided and their
// weights come from float64 scores; the others take float64 sigmoids of their float32 logits.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kTopkWarps = 8;
constexpr int kMaxSplit = 16;   // K parts of the router-logits GEMM (the layout never makes more)
constexpr float kCandDelta = 2e-3f;   // logit units; far above the float32 logit error

__device__ __forceinline__ bool better(float za, int ea, float zb, int eb) {
    return za > zb || (za == zb && ea < eb);
}

__device__ __forceinline__ bool better64(double sa, int ea, double sb, int eb) {
    return sa > sb || (sa == sb && ea < eb);
}

constexpr int kDotBatch = 8;   // router rows per pass over the token's row

// float64 dot products of the token's normed row with up to kDotBatch router rows (ids in ex[0..nb),
// warp-uniform), by the whole warp: one pass over the row, every row's loads of a step in flight
// together.  bf16 x bf16 products are exact in float64; the sums are float64.
__device__ __forceinline__ void dot64_batch(const uint4* __restrict__ xr, const uint16_t* __restrict__ gw, int d,
                                            const int (&ex)[kDotBatch], int nb, int lane, double (&out)[kDotBatch]) {
    const int nv = d >> 3;
    double acc[kDotBatch];
#pragma unroll
    for (int i = 0; i < kDotBatch; ++i) acc[i] = 0.0;
    for (int v = lane; v < nv; v += 32) {
        const uint4 a = xr[v];
        uint4 b[kDotBatch];
#pragma unroll
        for (int i = 0; i < kDotBatch; ++i)
            if (i < nb) b[i] = reinterpret_cast<const uint4*>(gw + static_cast<size_t>(ex[i]) * d)[v];
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
        double ad[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            ad[2 * q] = static_cast<double>(__uint_as_float(aw[q] << 16));
            ad[2 * q + 1] = static_cast<double>(__uint_as_float(aw[q] & 0xFFFF0000u));
        }
#pragma unroll
        for (int i = 0; i < kDotBatch; ++i) {
            if (i >= nb) continue;
            const uint32_t bw[4] = {b[i].x, b[i].y, b[i].z, b[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[i] = fma(ad[2 * q], static_cast<double>(__uint_as_float(bw[q] << 16)), acc[i]);
                acc[i] = fma(ad[2 * q + 1], static_cast<double>(__uint_as_float(bw[q] & 0xFFFF0000u)), acc[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kDotBatch; ++i) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], off);
        out[i] = acc[i];
    }
}

__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(const float* __restrict__ logits, int ksplit, const float* __restrict__ bias, const uint16_t* __restrict__ xn,
            const uint16_t* __restrict__ gw, int T, int E, int k, int d, int* __restrict__ idx, float* __restrict__ wout,
            uint8_t* __restrict__ flag) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTopkWarps + warp;
    if (t >= T) return;
    constexpr int J = kMaxExperts / 32;
    float z[J];
    uint32_t taken = 0, valid = 0;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int e = lane + 32 * j;
        float v = -INFINITY;
        if (e < E) {
            if (ksplit == 1) {
                v = logits[static_cast<size_t>(t) * E + e];
            } else {
                // K parts of the logits GEMM: all loads first, then the sum in a fixed order
                float part[kMaxSplit];
#pragma unroll
                for (int sp = 0; sp < kMaxSplit; ++sp)
                    if (sp < ksplit) part[sp] = logits[(static_cast<size_t>(sp) * T + t) * E + e];
                v = part[0];
#pragma unroll
                for (int sp = 1; sp < kMaxSplit; ++sp)
                    if (sp < ksplit) v = __fadd_rn(v, part[sp]);
            }
            if (bias) v = __fadd_rn(v, bias[e]);
            if (v != v) v = -INFINITY;
            valid |= 1u << j;
        }
        z[j] = v;
    }
    // float32 top k
    float zk = 0.0f;
    for (int rnd = 0; rnd < k; ++rnd) {
        float bz = -INFINITY;
        int be = 0x7FFFFFFF;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int e = lane + 32 * j;
            if (((valid & ~taken) >> j) & 1u && better(z[j], e, bz, be)) {
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
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        zk = bz;
    }
    // candidates near the k-th winner
    uint32_t cand = 0;
#pragma unroll
    for (int j = 0; j < J; ++j)
        if (((valid & ~taken) >> j) & 1u && z[j] >= zk - kCandDelta) cand |= 1u << j;
    const bool redo = __any_sync(0xFFFFFFFFu, cand != 0);
    const uint32_t S = taken | cand;
    double s64[J];
    uint32_t fin = taken;
    if (redo) {
        // float64 scores of every member of S (each lane keeps its own experts' values), then the
        // top k inside S by float64 score, lower index first on equal scores
        const uint4* xr = reinterpret_cast<const uint4*>(xn + static_cast<size_t>(t) * d);
#pragma unroll
        for (int j = 0; j < J; ++j) s64[j] = -1.0;
        // walk the members of S in expert order, kDotBatch router rows per pass over the row
        int ex[kDotBatch];
        int nb = 0;
        for (int j = 0; j < J; ++j) {
            uint32_t m = __ballot_sync(0xFFFFFFFFu, (S >> j) & 1u);
            while (m) {
                const int src = __ffs(m) - 1;
                m &= m - 1;
                ex[nb++] = src + 32 * j;
                const bool last = !m && [&] {
                    for (int jj = j + 1; jj < J; ++jj)
                        if (__ballot_sync(0xFFFFFFFFu, (S >> jj) & 1u)) return false;
                    return true;
                }();
                if (nb == kDotBatch || last) {
                    double zz[kDotBatch];
                    dot64_batch(xr, gw, d, ex, nb, lane, zz);
#pragma unroll
                    for (int i = 0; i < kDotBatch; ++i) {
                        if (i >= nb) continue;
                        const int e = ex[i];
                        double z64 = zz[i];
                        if (bias) z64 += static_cast<double>(bias[e]);
                        const double sc = 1.0 / (1.0 + exp(-z64));
#pragma unroll
                        for (int jj = 0; jj < J; ++jj)
                            if (e == lane + 32 * jj) s64[jj] = sc;
                    }
                    nb = 0;
                }
            }
        }
        fin = 0u;
        for (int rnd = 0; rnd < k; ++rnd) {
            double bs = -2.0;
            int be = 0x7FFFFFFF;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int e = lane + 32 * j;
                if (((S & ~fin) >> j) & 1u && better64(s64[j], e, bs, be)) {
                    bs = s64[j];
                    be = e;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double os = __shfl_xor_sync(0xFFFFFFFFu, bs, off);
                const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
                if (better64(os, oe, bs, be)) {
                    bs = os;
                    be = oe;
                }
            }
            if ((be & 31) == lane) fin |= 1u << (be >> 5);
        }
    } else {
        // no expert near the boundary: the float32 winners are the top k; scores from the float32
        // logits (promoted per 64-wide K stage, so their error is ~1e-6)
#pragma unroll
        for (int j = 0; j < J; ++j) s64[j] = ((taken >> j) & 1u) ? 1.0 / (1.0 + exp(-static_cast<double>(z[j]))) : 0.0;
    }
    // weights = scores / their sum; slots in ascending expert order
    double sum = 0.0;
#pragma unroll
    for (int j = 0; j < J; ++j)
        if ((fin >> j) & 1u) sum += s64[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
    int slot = 0;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, (fin >> j) & 1u);
        if ((fin >> j) & 1u) {
            const int pos = slot + __popc(m & ((1u << lane) - 1u));
            idx[static_cast<size_t>(t) * k + pos] = lane + 32 * j;
            wout[static_cast<size_t>(t) * k + pos] = static_cast<float>(s64[j] / sum);
        }
        slot += __popc(m);
    }
    if (lane == 0) flag[t] = redo ? 1 : 0;
}

}  // namespace

cudaError_t launch_topk(const Layout& L, const void* gate_w, const float* gate_bias, uint8_t* ws, cudaStream_t s) {
    const int grid = (L.T + kTopkWarps - 1) / kTopkWarps;
    topk_kernel<<<grid, kTopkWarps * 32, 0, s>>>(
        reinterpret_cast<const float*>(ws + L.logits), L.ksplit, gate_bias, reinterpret_cast<const uint16_t*>(ws + L.xn),
        static_cast<const uint16_t*>(gate_w), L.T, L.E, L.k, L.d, reinterpret_cast<int*>(ws + L.idx),
        reinterpret_cast<float*>(ws + L.w), ws + L.flag);
    return cudaGetLastError();
}

}  // namespace moe
