// Router selection.  The gate logits [T, E] come from the tensor-core GEMM (xn . Wg^T, float32
// accumulation, possibly as K parts summed here in a fixed order).  The router's body is not on the
// pages ("MoE update" page, MoE.forward excerpt only shows `weights, indices = self.gate(x)`); this
// library reads it as: scores = sigmoid(logit + bias), the top_k scores win with the lower expert
// index first on equal scores, and the winners' scores are normalised to sum 1.
//
// Two kernels.  topk_kernel: one warp per token; the E <= 256 float32 logits are spread over the
// lanes and the top k are picked by k rounds of a warp-wide (value, lower index) argmax, winner r
// kept by lane r % 32.  The logits are off by ~1e-6; kCandDelta is far above that.  A token with
// no other expert within kCandDelta of the k-th winner is final: its weights are float64 sigmoids
// of the winners' float32 logits (one per lane, in parallel), normalised.  A token with such a
// candidate is listed for topk_redo_kernel, which re-evaluates S = {winners} U {candidates} in
// float64 (bf16 x bf16 products are exact in float64) with one CTA per listed token, the members'
// dot products spread over its warps, and re-decides the top k inside S: every expert outside S is
// provably below all k winners, so the selection is the exact one.  Slots are in selection order
// (descending score).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kTopkWarps = 8;
constexpr int kRedoWarps = 16;        // a listed token's candidates, one warp each (S rarely exceeds 16)
constexpr int kMaxSplit = 16;          // K parts of the router-logits GEMM (the layout never makes more)
constexpr float kCandDelta = 2e-3f;    // logit units; far above the float32 logit error
constexpr int J = kMaxExperts / 32;    // experts per lane
enum : int { kStatusRedoCount = 2 };   // status word counting the listed tokens (zeroed per forward)

__device__ __forceinline__ bool better(float za, int ea, float zb, int eb) {
    return za > zb || (za == zb && ea < eb);
}

__device__ __forceinline__ bool better64(double sa, int ea, double sb, int eb) {
    return sa > sb || (sa == sb && ea < eb);
}

__device__ __forceinline__ double sigmoid64(double z) { return 1.0 / (1.0 + exp(-z)); }

// float32 logit (+ bias) of expert e for token t; the K parts are summed in a fixed order
__device__ __forceinline__ float logit32(const float* __restrict__ logits, int ksplit, const float* __restrict__ bias,
                                         int T, int E, int t, int e) {
    float v;
    if (ksplit == 1) {
        v = logits[static_cast<size_t>(t) * E + e];
    } else {
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
    return v != v ? -INFINITY : v;
}

// the float32 top k of a token (warp-wide) and whether another expert lies within kCandDelta of
// the k-th winner; winner r's expert and logit end up in lane r % 32, register r / 32
struct Sel {
    float z[J];
    uint32_t taken, valid;
    int we[J];
    float wz[J];
};

__device__ __forceinline__ bool select32(const float* __restrict__ logits, int ksplit, const float* __restrict__ bias,
                                         int T, int E, int k, int t, int lane, Sel& s) {
    s.taken = s.valid = 0;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int e = lane + 32 * j;
        s.z[j] = -INFINITY;
        s.we[j] = 0;
        s.wz[j] = 0.0f;
        if (e < E) {
            s.z[j] = logit32(logits, ksplit, bias, T, E, t, e);
            s.valid |= 1u << j;
        }
    }
    float zk = 0.0f;
    for (int rnd = 0; rnd < k; ++rnd) {
        float bz = -INFINITY;
        int be = 0x7FFFFFFF;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int e = lane + 32 * j;
            if (((s.valid & ~s.taken) >> j) & 1u && better(s.z[j], e, bz, be)) {
                bz = s.z[j];
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
        if ((be & 31) == lane) s.taken |= 1u << (be >> 5);
#pragma unroll
        for (int q = 0; q < J; ++q)
            if (q == (rnd >> 5) && lane == (rnd & 31)) {
                s.we[q] = be;
                s.wz[q] = bz;
            }
        zk = bz;
    }
    uint32_t cand = 0;
#pragma unroll
    for (int j = 0; j < J; ++j)
        if (((s.valid & ~s.taken) >> j) & 1u && s.z[j] >= zk - kCandDelta) cand |= 1u << j;
    return __any_sync(0xFFFFFFFFu, cand != 0);
}

__global__ void __launch_bounds__(kTopkWarps * 32)
topk_kernel(const float* __restrict__ logits, int ksplit, const float* __restrict__ bias, int T, int E, int k,
            int* __restrict__ idx, float* __restrict__ wout, uint8_t* __restrict__ flag, int* __restrict__ redo_list,
            uint32_t* __restrict__ status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTopkWarps + warp;
    if (t >= T) return;
    Sel s;
    if (select32(logits, ksplit, bias, T, E, k, t, lane, s)) {
        // an expert near the boundary: decided in float64 by topk_redo_kernel
        if (lane == 0) {
            redo_list[atomicAdd(status + kStatusRedoCount, 1u)] = t;
            flag[t] = 1;
        }
        return;
    }
    // weights: float64 sigmoids of the winners' float32 logits, normalised
    double sc[J], part = 0.0;
#pragma unroll
    for (int q = 0; q < J; ++q) {
        sc[q] = 0.0;
        if (32 * q + lane < k) {
            sc[q] = sigmoid64(static_cast<double>(s.wz[q]));
            part += sc[q];
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, off);
#pragma unroll
    for (int q = 0; q < J; ++q) {
        const int r = 32 * q + lane;
        if (r < k) {
            idx[static_cast<size_t>(t) * k + r] = s.we[q];
            wout[static_cast<size_t>(t) * k + r] = static_cast<float>(sc[q] / part);
        }
    }
    if (lane == 0) flag[t] = 0;
}

// float64 dot product of the token's normed row with one router row, by one warp (two
// accumulators, the loads of two steps in flight)
__device__ __forceinline__ double dot64(const uint4* __restrict__ xr, const uint4* __restrict__ wr, int nv, int lane) {
    double acc0 = 0.0, acc1 = 0.0;
#pragma unroll 2
    for (int v = lane; v < nv; v += 64) {
        const uint4 a0 = xr[v], b0 = wr[v];
        const bool two = v + 32 < nv;
        const uint4 a1 = two ? xr[v + 32] : make_uint4(0u, 0u, 0u, 0u);
        const uint4 b1 = two ? wr[v + 32] : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t aw0[4] = {a0.x, a0.y, a0.z, a0.w}, bw0[4] = {b0.x, b0.y, b0.z, b0.w};
        const uint32_t aw1[4] = {a1.x, a1.y, a1.z, a1.w}, bw1[4] = {b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc0 = fma(static_cast<double>(__uint_as_float(aw0[i] << 16)), static_cast<double>(__uint_as_float(bw0[i] << 16)), acc0);
            acc0 = fma(static_cast<double>(__uint_as_float(aw0[i] & 0xFFFF0000u)),
                       static_cast<double>(__uint_as_float(bw0[i] & 0xFFFF0000u)), acc0);
            acc1 = fma(static_cast<double>(__uint_as_float(aw1[i] << 16)), static_cast<double>(__uint_as_float(bw1[i] << 16)), acc1);
            acc1 = fma(static_cast<double>(__uint_as_float(aw1[i] & 0xFFFF0000u)),
                       static_cast<double>(__uint_as_float(bw1[i] & 0xFFFF0000u)), acc1);
        }
    }
    double acc = acc0 + acc1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
    return acc;
}

// The listed tokens, one CTA each: warp 0 rebuilds S, every warp evaluates its share of S in
// float64, warp 0 re-decides the top k inside S and writes the token's slots.
__global__ void __launch_bounds__(kRedoWarps * 32)
topk_redo_kernel(const float* __restrict__ logits, int ksplit, const float* __restrict__ bias,
                 const uint16_t* __restrict__ xn, const uint16_t* __restrict__ gw, int T, int E, int k, int d,
                 int* __restrict__ idx, float* __restrict__ wout, const int* __restrict__ redo_list,
                 const uint32_t* __restrict__ status) {
    __shared__ int members[kMaxExperts];
    __shared__ double s64[kMaxExperts];
    __shared__ int nmem_sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int count = static_cast<int>(status[kStatusRedoCount]);
    for (int i = blockIdx.x; i < count; i += gridDim.x) {
        const int t = redo_list[i];
        if (warp == 0) {
            Sel s;
            select32(logits, ksplit, bias, T, E, k, t, lane, s);
            // S = winners and every expert within kCandDelta of the k-th winner, in expert order
            float zk = -INFINITY;
#pragma unroll
            for (int q = 0; q < J; ++q)
                if (32 * q + lane == k - 1) zk = s.wz[q];
            zk = __shfl_sync(0xFFFFFFFFu, zk, (k - 1) & 31);   // the k-th winner's logit
            int n = 0;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const bool in = ((s.taken >> j) & 1u) || (((s.valid & ~s.taken) >> j) & 1u && s.z[j] >= zk - kCandDelta);
                const uint32_t m = __ballot_sync(0xFFFFFFFFu, in);
                if (in) members[n + __popc(m & ((1u << lane) - 1u))] = lane + 32 * j;
                n += __popc(m);
            }
            if (lane == 0) nmem_sh = n;
        }
        __syncthreads();
        const int n = nmem_sh;
        const uint4* xr = reinterpret_cast<const uint4*>(xn + static_cast<size_t>(t) * d);
        for (int m = warp; m < n; m += kRedoWarps) {
            const int e = members[m];
            double z = dot64(xr, reinterpret_cast<const uint4*>(gw + static_cast<size_t>(e) * d), d >> 3, lane);
            if (bias) z += static_cast<double>(bias[e]);
            if (lane == 0) s64[m] = sigmoid64(z);
        }
        __syncthreads();
        if (warp == 0) {
            // top k inside S by float64 score, lower index first; lane l holds members l, l + 32, ...
            uint32_t fin = 0u;
            int we[J];
            double ws[J];
#pragma unroll
            for (int q = 0; q < J; ++q) {
                we[q] = 0;
                ws[q] = 0.0;
            }
            for (int rnd = 0; rnd < k; ++rnd) {
                double bs = -2.0;
                int be = 0x7FFFFFFF, bm = -1;
#pragma unroll
                for (int q = 0; q < J; ++q) {
                    const int m = lane + 32 * q;
                    if (m < n && !((fin >> q) & 1u) && better64(s64[m], members[m], bs, be)) {
                        bs = s64[m];
                        be = members[m];
                        bm = m;
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const double os = __shfl_xor_sync(0xFFFFFFFFu, bs, off);
                    const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
                    const int om = __shfl_xor_sync(0xFFFFFFFFu, bm, off);
                    if (better64(os, oe, bs, be)) {
                        bs = os;
                        be = oe;
                        bm = om;
                    }
                }
                if ((bm & 31) == lane) fin |= 1u << (bm >> 5);
#pragma unroll
                for (int q = 0; q < J; ++q)
                    if (q == (rnd >> 5) && lane == (rnd & 31)) {
                        we[q] = be;
                        ws[q] = bs;
                    }
            }
            double part = 0.0;
#pragma unroll
            for (int q = 0; q < J; ++q)
                if (32 * q + lane < k) part += ws[q];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, off);
#pragma unroll
            for (int q = 0; q < J; ++q) {
                const int r = 32 * q + lane;
                if (r < k) {
                    idx[static_cast<size_t>(t) * k + r] = we[q];
                    wout[static_cast<size_t>(t) * k + r] = static_cast<float>(ws[q] / part);
                }
            }
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_topk(const Layout& L, const void* gate_w, const float* gate_bias, uint8_t* ws, cudaStream_t s) {
    const int grid = (L.T + kTopkWarps - 1) / kTopkWarps;
    const float* logits = reinterpret_cast<const float*>(ws + L.logits);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
    topk_kernel<<<grid, kTopkWarps * 32, 0, s>>>(logits, L.ksplit, gate_bias, L.T, L.E, L.k,
                                                 reinterpret_cast<int*>(ws + L.idx), reinterpret_cast<float*>(ws + L.w),
                                                 ws + L.flag, reinterpret_cast<int*>(ws + L.redo), status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    topk_redo_kernel<<<std::min(L.T, 4 * num_sms()), kRedoWarps * 32, 0, s>>>(
        logits, L.ksplit, gate_bias, reinterpret_cast<const uint16_t*>(ws + L.xn), static_cast<const uint16_t*>(gate_w),
        L.T, L.E, L.k, L.d, reinterpret_cast<int*>(ws + L.idx), reinterpret_cast<float*>(ws + L.w),
        reinterpret_cast<const int*>(ws + L.redo), status);
    return cudaGetLastError();
}

}  // namespace moe
