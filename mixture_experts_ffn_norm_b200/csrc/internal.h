// Internal declarations shared by the .cu files of libmoe: workspace layout, grouped-GEMM
// parameters and the host-side launchers of each kernel.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kBM = 128;          // rows of A per GEMM tile (tokens)
constexpr int kBN = 256;          // columns (weight rows) per GEMM tile
constexpr int kStageBytesA = kBM * 128;
constexpr int kStageBytesB = kBN * 128;
constexpr int kStages = 4;
constexpr int kGemmThreads = 384;  // warpgroup 0: warp 0 TMA, warp 1 MMA; warpgroups 1-2: epilogue
constexpr int kMaxExperts = 256;
constexpr int kRouteChunk = 2048;  // (token, slot) entries per block in the routing kernels

enum GemmMode : int { kModeLogits = 0, kModeUp = 1, kModeDown = 2 };

// Byte offsets of every region of the caller's workspace.
struct Layout {
    int T, d, I, E, k, Is, Tpad, R, KBd, KBi, KBs, nchunks;
    int ksplit;                 // K parts of the router-logits GEMM (float32 partials, summed by top-k)
    bool fp8, act8;
    bool dense;                 // E = 0: a dense block, the MLP held as the shared SwiGLU, no router
    size_t status, xn, xq, xs, logits, idx, w, flag, counts, offsets, row_base, row_count,
        ts_up, ts_down, chunk_hist, row_of, row_token, redo, a_perm, as_perm, h, hs, h_sh, hs_sh, y, y_sh, total;
};

bool make_layout(const moe_config_t& c, Layout& L);

// Parameters of the persistent grouped GEMM.  Groups 0..G-2 (or 0..G-1 without a shared expert)
// are routed experts whose rows sit at row_base[g] in the permuted A; the last group is the shared
// expert over all T tokens in token order.  Everything group-dependent is read on the device, so
// the host never learns the routing.
struct GemmParams {
    int G;                      // number of groups
    int has_shared;             // last group is the shared expert
    int single_rows;            // > 0: one shared-style group of this many rows, no device arrays
    const int* tile_start;      // [G + 1] cumulative tile counts
    const int* row_base;        // [G]
    const int* row_count;       // [G]
    int n_tiles_r, n_tiles_s;   // N tiles of a routed / the shared group
    int kb_r, kb_s;             // K stages of a routed / the shared group
    int b_rows_per_expert;      // rows of one routed expert in the B tensor
    // activation scales, transposed [K/128][ld] (FP8 only)
    const float* as_r; const float* as_s;
    int as_ld_r, as_ld_s;
    // weight block scales (FP8 only): routed [E][rows/128][cols/128], shared [rows/128][cols/128]
    const float* bs0_r; const float* bs1_r; const float* bs0_s; const float* bs1_s;
    int bs_cols_r, bs_cols_s, bs_rows_r;
    // outputs: row-major with row strides (elements) out_ld_*; output scales transposed [N/128][ld]
    void* out_r; void* out_s;
    int out_ld_r, out_ld_s;
    float* outs_r; float* outs_s;
    int outs_ld_r, outs_ld_s;
    int n_valid_cols;           // logits: columns actually stored (E)
    // split K (single-group launches only): part ks covers K stages [ks * kb_chunk, ...) and writes
    // its float32 partial tile at out + ks * split_stride bytes
    int ksplit, kb_chunk;
    size_t split_stride;
    uint32_t* status;
};

struct TensorMaps {
    CUtensorMap a_r, a_s, b0_r, b1_r, b0_s, b1_s;
    CUtensorMap o_r, o_s;   // FP8 epilogue outputs (h or y rows), written by TMA stores
};

// tensor-map encoding (driver entry point fetched at run time; no libcuda link)
bool encode_map_2d(CUtensorMap* map, const void* base, bool fp8, uint64_t inner, uint64_t rows);
// unswizzled map over a row-major [rows, inner] byte tensor loading [128 rows x 64 bytes] boxes
bool encode_raw_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows);
// unswizzled map for TMA stores of [32 rows x box_inner elements] boxes
bool encode_store_map_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t inner, uint64_t rows,
                         uint32_t box_inner);

cudaError_t launch_norm(const Layout& L, const void* x, const void* residual, const float* g, float eps,
                        void* residual_out, uint8_t* ws, cudaStream_t s);
// fp8: e4m3 weights with block scales; a16 (with fp8): bf16 activations, the weights widened in
// shared memory (the B maps then load raw 64-byte x 128-row e4m3 boxes, see encode_raw_map_2d)
cudaError_t launch_gemm(int mode, bool fp8, bool a16, const TensorMaps& maps, const GemmParams& p, int grid,
                        cudaStream_t s);
cudaError_t launch_topk(const Layout& L, const void* gate_w, const float* gate_bias, uint8_t* ws, cudaStream_t s);
cudaError_t launch_route(const Layout& L, int ntu_r, int ntu_s, int ntd_r, int ntd_s, uint8_t* ws,
                         cudaStream_t s, int ebeg, int eend, bool shared_here);
cudaError_t launch_combine(const Layout& L, void* out, uint8_t* ws, cudaStream_t s);
// expert slice: y_partial [T, d] float32 = sum over the token's slots routed to experts in
// [ebeg, eend) of w * y (+ the shared expert's row when it ran here); no rounding
cudaError_t launch_round_bf16(const float* y, void* out, int64_t n, cudaStream_t s);
cudaError_t launch_combine_partial(const Layout& L, float* y_partial, int ebeg, int eend, bool shared_here,
                                   uint8_t* ws, cudaStream_t s);
// the combine with the next block's RMSNorm: resid holds the block's new residual on entry and the
// next residual on exit; out (the MoE update) may be NULL
cudaError_t launch_combine_next_norm(const Layout& L, void* out, const float* gain, float eps, void* resid,
                                     void* xn_next, uint8_t* ws, cudaStream_t s);

int num_sms();

}  // namespace moe
