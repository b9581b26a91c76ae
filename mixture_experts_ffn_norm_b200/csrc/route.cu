// Token permutation by expert, with no host synchronisation.
//
// The pages' loop ("MoE update" page, MoE.forward excerpt) counts tokens per expert with
// torch.bincount(...).tolist() -- a device-to-host copy -- and gathers each expert's
// (token, slot) pairs with torch.where.  Here the same grouping is built on the device:
//   hist    : per chunk of 2048 (token, slot) entries, a shared-memory histogram over experts;
//   scan    : per expert, exclusive prefix over chunks (stable order) and over experts of the
//             counts padded to the 128-row GEMM tile; the grouped GEMMs' tile tables;
//   scatter : every entry gets its row in the permuted order (token order inside an expert,
//             so the permutation is deterministic);
//   gather  : the permuted activation rows (FP8 codes or bf16) and their group scales are
//             copied next to each other so a TMA box of 128 rows is one expert's tile (one warp
//             per token reads its row once and writes its k copies).
// For an expert slice the scan gives only the experts in [ebeg, eend) GEMM tiles; every expert
// keeps its rows in the permutation.
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kRouteThreads = 256;
constexpr int kMaxTopkGather = 8;   // top-k slots the gather keeps in registers

__global__ void __launch_bounds__(kRouteThreads)
hist_kernel(const int* __restrict__ idx, int N, int E, int* __restrict__ chunk_hist, uint32_t* status) {
    __shared__ int h[kMaxExperts];
    for (int e = threadIdx.x; e < kMaxExperts; e += kRouteThreads) h[e] = 0;
    __syncthreads();
    const int c = blockIdx.x;
    const int end = min(N, (c + 1) * kRouteChunk);
    for (int i = c * kRouteChunk + threadIdx.x; i < end; i += kRouteThreads) {
        const int e = idx[i];
        if (e >= 0 && e < E) atomicAdd(&h[e], 1);
        else latch_error(status, kErrCheck, 0x100);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kRouteThreads) chunk_hist[static_cast<size_t>(c) * E + e] = h[e];
}

// block-wide exclusive scan of one int per thread (256 threads); returns the total in *total
__device__ int block_exclusive_scan(int v, int* sh, int* total) {
    const int tid = threadIdx.x;
    sh[tid] = v;
    __syncthreads();
    for (int off = 1; off < kRouteThreads; off <<= 1) {
        const int add = tid >= off ? sh[tid - off] : 0;
        __syncthreads();
        sh[tid] += add;
        __syncthreads();
    }
    const int incl = sh[tid];
    *total = sh[kRouteThreads - 1];
    __syncthreads();
    return incl - v;
}

__global__ void __launch_bounds__(kRouteThreads)
scan_kernel(int* __restrict__ chunk_hist, int nchunks, int E, int T, int has_shared, int ntu_r, int ntu_s,
            int ntd_r, int ntd_s, int* __restrict__ counts, int* __restrict__ offsets, int* __restrict__ row_base,
            int* __restrict__ row_count, int* __restrict__ ts_up, int* __restrict__ ts_down, int ebeg, int eend,
            int shared_here) {
    __shared__ int sh[kRouteThreads];
    const int e = threadIdx.x;
    int cnt = 0;
    if (e < E) {
        for (int c = 0; c < nchunks; ++c) {
            const int v = chunk_hist[static_cast<size_t>(c) * E + e];
            chunk_hist[static_cast<size_t>(c) * E + e] = cnt;   // exclusive base of chunk c
            cnt += v;
        }
    }
    const int mtiles = (cnt + kBM - 1) / kBM;
    // every expert keeps its rows; only the experts in [ebeg, eend) get GEMM tiles (an expert slice)
    const int mine = (e >= ebeg && e < eend) ? mtiles : 0;
    int tot_rows, tot_up, tot_down;
    const int off = block_exclusive_scan(mtiles * kBM, sh, &tot_rows);
    const int tu = block_exclusive_scan(mine * ntu_r, sh, &tot_up);
    const int td = block_exclusive_scan(mine * ntd_r, sh, &tot_down);
    if (e < E) {
        counts[e] = cnt;
        offsets[e] = off;
        row_base[e] = off;
        row_count[e] = cnt;
        ts_up[e] = tu;
        ts_down[e] = td;
    }
    if (e == 0) {
        offsets[E] = tot_rows;
        ts_up[E] = tot_up;
        ts_down[E] = tot_down;
        if (has_shared) {
            const int mt = (T + kBM - 1) / kBM;
            row_base[E] = 0;
            row_count[E] = T;
            ts_up[E + 1] = tot_up + (shared_here ? mt * ntu_s : 0);
            ts_down[E + 1] = tot_down + (shared_here ? mt * ntd_s : 0);
        }
    }
}

__global__ void __launch_bounds__(kRouteThreads)
scatter_kernel(const int* __restrict__ idx, int N, int E, int k, const int* __restrict__ chunk_base,
               const int* __restrict__ offsets, int* __restrict__ row_of, int* __restrict__ row_token) {
    __shared__ int run_base[kMaxExperts];
    __shared__ int wcnt[kRouteThreads / 32][kMaxExperts];
    const int c = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < kMaxExperts; e += kRouteThreads) {
        run_base[e] = e < E ? offsets[e] + chunk_base[static_cast<size_t>(c) * E + e] : 0;
#pragma unroll
        for (int w = 0; w < kRouteThreads / 32; ++w) wcnt[w][e] = 0;
    }
    __syncthreads();
    const int end = min(N, (c + 1) * kRouteChunk);
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int base = c * kRouteChunk; base < end; base += kRouteThreads) {
        const int i = base + threadIdx.x;
        const bool valid = i < end;
        int e = valid ? idx[i] : -1;
        if (e < 0 || e >= E) e = -1;
        const uint32_t m = __match_any_sync(0xFFFFFFFFu, e);
        const int lane_rank = __popc(m & lt_mask);
        const bool leader = (__ffs(m) - 1) == lane;
        if (e >= 0 && leader) wcnt[warp][e] = __popc(m);
        __syncthreads();
        if (e >= 0) {
            int rank = lane_rank;
            for (int w = 0; w < warp; ++w) rank += wcnt[w][e];
            const int pos = run_base[e] + rank;
            row_of[i] = pos;
            row_token[pos] = i / k;
        }
        __syncthreads();
        if (e >= 0 && leader) {
            atomicAdd(&run_base[e], __popc(m));
            wcnt[warp][e] = 0;
        }
        __syncthreads();
    }
}

// One warp per token: its activation row is read once and written to each of its k permuted rows
// (row_of), with its group scales.  Walking tokens rather than destination rows keeps the source
// row from being re-read k times -- with k rows' worth of writes streaming through L2 those re-reads
// would come back from DRAM.
__global__ void __launch_bounds__(kRouteThreads)
gather_kernel(const int* __restrict__ row_of, int T, int k, const uint4* __restrict__ src, int row_vecs,
              uint4* __restrict__ dst, const float* __restrict__ xs, int Tpad, float* __restrict__ as, int R, int KB) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int t = blockIdx.x * (kRouteThreads / 32) + warp; t < T; t += gridDim.x * (kRouteThreads / 32)) {
        int rows[kMaxTopkGather];
        const int kk = min(k, kMaxTopkGather);
#pragma unroll
        for (int j = 0; j < kMaxTopkGather; ++j) rows[j] = j < kk ? row_of[static_cast<size_t>(t) * k + j] : 0;
        const uint4* sr = src + static_cast<size_t>(t) * row_vecs;
#pragma unroll 2
        for (int v = lane; v < row_vecs; v += 32) {
            const uint4 val = sr[v];
#pragma unroll
            for (int j = 0; j < kMaxTopkGather; ++j)
                if (j < kk) dst[static_cast<size_t>(rows[j]) * row_vecs + v] = val;
            for (int j = kMaxTopkGather; j < k; ++j)          // wider top-k than the register list
                dst[static_cast<size_t>(row_of[static_cast<size_t>(t) * k + j]) * row_vecs + v] = val;
        }
        if (as)
            for (int kb = lane; kb < KB; kb += 32) {
                const float sc = xs[static_cast<size_t>(kb) * Tpad + t];
                for (int j = 0; j < k; ++j) as[static_cast<size_t>(kb) * R + row_of[static_cast<size_t>(t) * k + j]] = sc;
            }
    }
}

}  // namespace

cudaError_t launch_route(const Layout& L, int ntu_r, int ntu_s, int ntd_r, int ntd_s, uint8_t* ws, cudaStream_t s,
                         int ebeg, int eend, bool shared_here) {
    const int N = L.T * L.k;
    int* idx = reinterpret_cast<int*>(ws + L.idx);
    int* chunk = reinterpret_cast<int*>(ws + L.chunk_hist);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
    hist_kernel<<<L.nchunks, kRouteThreads, 0, s>>>(idx, N, L.E, chunk, status);
    scan_kernel<<<1, kRouteThreads, 0, s>>>(chunk, L.nchunks, L.E, L.T, L.Is > 0, ntu_r, ntu_s, ntd_r, ntd_s,
                                            reinterpret_cast<int*>(ws + L.counts), reinterpret_cast<int*>(ws + L.offsets),
                                            reinterpret_cast<int*>(ws + L.row_base),
                                            reinterpret_cast<int*>(ws + L.row_count), reinterpret_cast<int*>(ws + L.ts_up),
                                            reinterpret_cast<int*>(ws + L.ts_down), ebeg, eend, shared_here ? 1 : 0);
    scatter_kernel<<<L.nchunks, kRouteThreads, 0, s>>>(idx, N, L.E, L.k, chunk, reinterpret_cast<int*>(ws + L.offsets),
                                                       reinterpret_cast<int*>(ws + L.row_of),
                                                       reinterpret_cast<int*>(ws + L.row_token));
    const int row_bytes = L.act8 ? L.d : 2 * L.d;
    const int grid = 4 * num_sms();
    gather_kernel<<<grid, kRouteThreads, 0, s>>>(
        reinterpret_cast<const int*>(ws + L.row_of), L.T, L.k,
        reinterpret_cast<const uint4*>(ws + (L.act8 ? L.xq : L.xn)), row_bytes / 16,
        reinterpret_cast<uint4*>(ws + L.a_perm), L.act8 ? reinterpret_cast<const float*>(ws + L.xs) : nullptr,
        L.Tpad, L.act8 ? reinterpret_cast<float*>(ws + L.as_perm) : nullptr, L.R, L.KBd);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// moe_route_noalloc: the same counting / scan / permutation, for callers that cannot allocate.
//
// Its scratch -- the per-chunk histograms and the tile tables the scan also produces -- lives in
// one file-scope device array instead of a caller workspace.  The array exists once per device
// for the life of the process; every call on a device shares it.
// ------------------------------------------------------------------------------------------------
namespace {

constexpr int kNoAllocMaxEntries = 1 << 18;                               // T * k
constexpr int kNoAllocMaxChunks = kNoAllocMaxEntries / kRouteChunk;       // 128
constexpr int kNoAllocHist = kNoAllocMaxChunks * kMaxExperts;             // ints
constexpr int kNoAllocTables = 2 * (kMaxExperts + 1) + 2 * (kMaxExperts + 2);
constexpr int kNoAllocInts = kNoAllocHist + kNoAllocTables;                // 34,818 ints = 136 KiB

static __device__ __align__(256) int g_route_scratch[kNoAllocInts];

constexpr int kMaxDevices = 64;
int* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_route_scratch on the current device, looked up once per device.  In host
// code the array's name is only a host-side stand-in, so it must never be passed to a kernel.
cudaError_t scratch_for_current_device(int** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<int*>(p);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

}  // namespace moe

extern "C" moe_status_t moe_route_noalloc(const int32_t* idx, int32_t num_tokens, int32_t top_k, int32_t n_experts,
                                          int32_t* counts, int32_t* offsets, int32_t* row_of, int32_t* row_token,
                                          void* stream) {
    using namespace moe;
    if (!idx || !counts || !offsets || !row_of || !row_token) return MOE_ERR_INVALID_ARG;
    if (num_tokens < 1 || top_k < 1 || n_experts < 1 || n_experts > kMaxExperts || top_k > n_experts)
        return MOE_ERR_INVALID_ARG;
    const long long n = static_cast<long long>(num_tokens) * top_k;
    if (n > kNoAllocMaxEntries) return MOE_ERR_UNSUPPORTED;   // beyond the static scratch
    int* scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int N = static_cast<int>(n), E = n_experts;
    const int nchunks = (N + kRouteChunk - 1) / kRouteChunk;
    const long long rows = (n + static_cast<long long>(E) * (kBM - 1) + kBM - 1) / kBM * kBM;
    int* hist = scratch;
    int* row_base = scratch + kNoAllocHist;
    int* row_count = row_base + (kMaxExperts + 1);
    int* ts_up = row_count + (kMaxExperts + 1);
    int* ts_down = ts_up + (kMaxExperts + 2);
    // every histogram entry the scan reads is written by hist_kernel first, so nothing left in
    // the array by an earlier call is read; row_token's padding must read -1
    if (cudaMemsetAsync(row_token, 0xFF, static_cast<size_t>(rows) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    hist_kernel<<<nchunks, kRouteThreads, 0, s>>>(idx, N, E, hist, nullptr);
    scan_kernel<<<1, kRouteThreads, 0, s>>>(hist, nchunks, E, num_tokens, 0, 1, 1, 1, 1, counts, offsets, row_base,
                                            row_count, ts_up, ts_down, 0, E, 0);
    scatter_kernel<<<nchunks, kRouteThreads, 0, s>>>(idx, N, E, top_k, hist, offsets, row_of, row_token);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
