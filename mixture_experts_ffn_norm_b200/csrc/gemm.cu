// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by TMA.
//
// One kernel serves the three contractions of the layer:
//   kModeLogits : router logits  = xn [T, d] . Wg[E, d]^T                 (bf16, one group)
//   kModeUp     : SwiGLU up      g = a . W1_e^T, u = a . W3_e^T, h = silu(g) * u
//                 ("Gate projection" page, expert excerpt); w1 and w3 rows share one A tile:
//                 the B tile is [128 rows of W1 ; 128 rows of W3] and one 128x256 MMA covers both
//   kModeDown   : SwiGLU down    y = h . W2_e^T
// over groups = routed experts (rows permuted by expert) + the shared expert (all tokens).
//
// FP8 weights carry one float32 scale per 128x128 block ("Gate projection" page, Linear excerpt)
// and the activations one per 1x128 group, neither a power of two, so the tensor core's own block
// scaling does not apply.  Each 128-wide K block is therefore accumulated into its own TMEM buffer
// and promoted by the epilogue warps: acc += P_kb * (s_act[row, kb] * s_w[nblk, kb]) in float32
// registers.  Two TMEM buffers (2 x 256 columns) let the MMA of block kb+1 run while block kb is
// promoted.  bf16 operands simply accumulate the whole K in TMEM.  With FP8 weights and bf16
// activations (kA16) each stage's e4m3 weight tile is widened to bf16 in shared memory, the MMAs
// are bf16 and every 128-wide K block (two 64-wide stages) is promoted with its weight scale.
// The router-logits launch may split K into parts that write float32 partial tiles (few tokens).
//
// Warp roles (384 threads = 3 warpgroups, one CTA per SM, persistent over a device-side tile table):
//   warp 0      issues the TMA loads of A (128 x 128 B) and B (256 x 128 B) per stage (one elected lane)
//   warp 1      issues tcgen05.mma (M=128, N=256, K=32 bytes per instruction): the whole warp runs the
//               loop and waits, one elected lane issues
//   warps 2-3   kA16: widen the stage's e4m3 weight tile to bf16; otherwise idle (they only hand
//               their registers back)
//   warps 4..11 epilogue: warp w reads TMEM lanes 32*(w%4).., column half (w-4)/4
// Each promotion reads 64 TMEM columns per tcgen05.ld (two per K block per thread).
// The MMA thread and the epilogue poll their barriers (mbar_spin) rather than suspend in try_wait:
// the TMEM double buffer makes their handshake the critical path, and a suspended waiter wakes late.
// setmaxnreg moves registers from warpgroup 0 (56 each) to the two epilogue warpgroups (224 each):
// 128*56 + 256*224 = 64512 = 384 * 168, the launch budget.  The FP8 promotion keeps 128 float32
// accumulators per thread, loads 64 TMEM columns per wait, accumulates with packed fp32x2 FMAs and
// prefetches the next K block's scales while it waits.
// Tiles are taken m-fastest inside a group so concurrently running CTAs share the weight tile
// through L2.  Every wait is bounded (see ptx.cuh); on a timeout all roles leave their loops,
// in-flight TMA loads and MMAs are drained with bounded waits, and TMEM is freed.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kStageBytes = kStageBytesA + kStageBytesB;
// bf16-activation mode for FP8 weights: the weight tile of a 64-wide K stage arrives as e4m3 bytes
// (256 rows x 64 B) next to the stage and is widened to bf16 in the stage's B area
constexpr int kRawBytes = 256 * 64;
constexpr int kStagesA16 = 3;
constexpr int kStageBytesA16 = kStageBytes + kRawBytes;
constexpr int kOutStageBytes = 2048;                       // per epilogue warp: 32 rows x 64 bytes
constexpr int kSmemBytes = kStages * kStageBytes + 8 * kOutStageBytes + 1024;
constexpr int kSmemBytesA16 = kStagesA16 * kStageBytesA16 + 8 * kOutStageBytes + 1024;
constexpr uint32_t kTmemCols = 512;

struct Tile {
    int g, mt, nt, shared, a_row0, rows_valid, kb, b_row0;
    int kb0, ks;   // first K stage and K part (split-K launches; 0 otherwise)
};

__device__ __forceinline__ void decode_tile(int t, const int* ts, const int* rb, const int* rc, const GemmParams& p,
                                            int mode, Tile& ti) {
    int lo = 0, hi = p.G;   // largest g with ts[g] <= t (groups without tiles are skipped)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ts[mid] <= t) lo = mid;
        else hi = mid;
    }
    ti.g = lo;
    ti.shared = (p.single_rows > 0) || (p.has_shared && lo == p.G - 1);
    const int cnt = rc[lo];
    const int mtiles = (cnt + kBM - 1) / kBM;
    int local = t - ts[lo];
    ti.ks = 0;
    if (p.ksplit > 1) {                       // K part outermost, then N, then M
        const int per = mtiles * p.n_tiles_s;
        ti.ks = local / per;
        local -= ti.ks * per;
    }
    ti.nt = local / mtiles;
    ti.mt = local - ti.nt * mtiles;
    ti.a_row0 = rb[lo] + ti.mt * kBM;
    ti.rows_valid = min(kBM, cnt - ti.mt * kBM);
    const int kbt = ti.shared ? p.kb_s : p.kb_r;
    ti.kb0 = ti.ks * p.kb_chunk;
    ti.kb = p.ksplit > 1 ? min(p.kb_chunk, kbt - ti.kb0) : kbt;
    const int nrows = (mode == kModeUp) ? 128 : 256;
    ti.b_row0 = (ti.shared ? 0 : lo * p.b_rows_per_expert) + ti.nt * nrows;
}

// bounded wait without the abort check, for draining copies / MMAs already in flight
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(smem_u32(bar), parity))
        if (clock64() - t0 > kWaitCycles) return;
}

__device__ __forceinline__ float bf16r(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(a))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(b))) << 16);
}

// a / b given y = the correctly rounded 1/b: one product and one FMA-residual correction
// (Markstein), which yields the correctly rounded quotient -- exact quotients, such as the
// e4m3 rounding midpoints a group quantisation often lands on, come out exact.
__device__ __forceinline__ float div_by_rcp(float a, float b, float y) {
    const float q = a * y;
    return fmaf(fmaf(-q, b, a), y, q);
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    // silu(g) * u with the Linear outputs g, u in bf16 and the product rounded to bf16; silu in
    // float32: expf and a corrected division (1 + e >= 1, so the approximate reciprocal is safe)
    const float gb = bf16r(g), ub = bf16r(u);
    const float d = 1.0f + expf(-gb);
    // exp overflow (g below about -88): silu(g) rounds to zero; the correction step would form 0 * inf
    const float sg = d < INFINITY ? div_by_rcp(gb, d, rcp_approx(d)) : 0.0f;
    return bf16r(sg * ub);
}

// two e4m3 codes (low byte first) -> two bf16 (low half first); exact: every e4m3 value is a bf16 value
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<const uint32_t*>(&b);
}

// kFp8: the weights are e4m3 with 128x128 block scales.  kA16 (with kFp8): the activations stay bf16
// and each weight tile is widened to bf16 in shared memory by warps 2-3 before bf16 MMAs; otherwise
// FP8 weights meet 1x128-quantised FP8 activations in FP8 MMAs.
template <bool kFp8, int kMode, bool kA16>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tm_a_r, const __grid_constant__ CUtensorMap tm_a_s,
            const __grid_constant__ CUtensorMap tm_b0_r, const __grid_constant__ CUtensorMap tm_b1_r,
            const __grid_constant__ CUtensorMap tm_b0_s, const __grid_constant__ CUtensorMap tm_b1_s,
            const __grid_constant__ CUtensorMap tm_o_r, const __grid_constant__ CUtensorMap tm_o_s,
            const GemmParams p) {
    extern __shared__ uint8_t dyn_smem[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(8) uint64_t empty_bar[kStages];
    __shared__ __align__(8) uint64_t conv_bar[kStages];    // kA16: the stage's weight tile is widened
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ __align__(8) uint64_t xchg_bar;        // FP8 up: row maxima exchanged between the warpgroups
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ int ts_sh[kMaxExperts + 2];
    __shared__ int rb_sh[kMaxExperts + 1];
    __shared__ int rc_sh[kMaxExperts + 1];
    __shared__ float amax_sh[2][2][kBM];             // [tile parity][warpgroup][row]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool kAct8 = kFp8 && !kA16;               // FP8 activations, FP8 MMAs
    constexpr int NS = kA16 ? kStagesA16 : kStages;     // pipeline stages
    constexpr int SB = kA16 ? kStageBytesA16 : kStageBytes;
    constexpr int KX = kAct8 ? 128 : 64;                // K elements per stage
    static_assert(!kA16 || kFp8, "the bf16-activation mode is for FP8 weights");

    if (p.single_rows > 0) {
        if (threadIdx.x == 0) {
            ts_sh[0] = 0;
            ts_sh[1] = ((p.single_rows + kBM - 1) / kBM) * p.n_tiles_s * max(1, p.ksplit);
            rb_sh[0] = 0;
            rc_sh[0] = p.single_rows;
        }
    } else {
        for (int i = threadIdx.x; i <= p.G; i += blockDim.x) {
            ts_sh[i] = p.tile_start[i];
            if (i < p.G) {
                rb_sh[i] = p.row_base[i];
                rc_sh[i] = p.row_count[i];
            }
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
            mbar_init(&conv_bar[s], 64);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 8);
        }
        mbar_init(&drain_bar, 1);
        mbar_init(&xchg_bar, 256);
        abort_sh = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    const int total = ts_sh[p.G];

    if (warp < 4) {
      regs_dec<56>();
      if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        // whole warp in the loop (warp-uniform coordinates), the elected lane issues
        const bool leader = elect_one();
        if (leader) {
            prefetch_tensormap(&tm_a_r);
            prefetch_tensormap(&tm_a_s);
            prefetch_tensormap(&tm_b0_r);
            prefetch_tensormap(&tm_b1_r);
            prefetch_tensormap(&tm_b0_s);
            prefetch_tensormap(&tm_b1_s);
        }
        int stage = 0;
        uint32_t phase = 0, pend = 0, pend_par = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            Tile ti;
            decode_tile(t, ts_sh, rb_sh, rc_sh, p, kMode, ti);
            const CUtensorMap* ma = ti.shared ? &tm_a_s : &tm_a_r;
            const CUtensorMap* mb0 = ti.shared ? &tm_b0_s : &tm_b0_r;
            const CUtensorMap* mb1 = ti.shared ? &tm_b1_s : &tm_b1_r;
            const int b1_row = (kMode == kModeUp) ? ti.b_row0 : ti.b_row0 + 128;
            for (int kb = 0; kb < ti.kb; ++kb) {
                const bool got = mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_sh, p.status, 0x10);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    ok = false;
                    break;
                }
                if (leader) {
                    uint8_t* sa = smem + stage * SB;
                    uint8_t* sb = sa + (kA16 ? kStageBytes : kStageBytesA);   // kA16: the raw e4m3 area
                    mbar_arrive_expect_tx(&full_bar[stage], kA16 ? kStageBytesA + kRawBytes : kStageBytes);
                    const int kx = (ti.kb0 + kb) * KX;
                    tma_load_2d(sa, ma, &full_bar[stage], kx, ti.a_row0);
                    tma_load_2d(sb, mb0, &full_bar[stage], kx, ti.b_row0);
                    tma_load_2d(sb + (kA16 ? kRawBytes / 2 : 128 * 128), mb1, &full_bar[stage], kx, b1_row);
                }
                __syncwarp();
                pend |= 1u << stage;
                pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
                if (++stage == NS) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && leader)
            for (int s = 0; s < NS; ++s)
                if ((pend >> s) & 1u) drain_wait(&full_bar[s], (pend_par >> s) & 1u);
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop, so the descriptors are warp-uniform; the elected lane issues
        // the MMAs and the commits (a commit tracks the MMAs of the thread that issues it).
        constexpr uint32_t idesc = instr_desc(kAct8, kBM, kBN);
        constexpr bool kPromote = kFp8 || kMode == kModeLogits;
        // stages per promoted K block: FP8 weights carry one scale per 128 K, a bf16 stage is 64 wide
        constexpr int kPer = kA16 ? 2 : 1;
        const bool leader = elect_one();
        int stage = 0, abuf = 0;
        uint32_t phase = 0, aphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            Tile ti;
            decode_tile(t, ts_sh, rb_sh, rc_sh, p, kMode, ti);
            for (int kb = 0; kb < ti.kb; ++kb) {
                // the operands are normally resident long before the accumulator buffer is handed back,
                // so everything but the TMEM-empty wait is done first: the MMAs follow that wait directly
                if (!mbar_spin_warp(kA16 ? &conv_bar[stage] : &full_bar[stage], phase, &abort_sh, p.status, 0x21)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = smem_u32(smem + stage * SB);
                const uint64_t ad = smem_desc_sw128(sa);
                const uint64_t bd = smem_desc_sw128(sa + kStageBytesA);
                const uint32_t dt = tmem + static_cast<uint32_t>(abuf * kBN);
                const bool first = kPromote ? (kb % kPer == 0) : kb == 0;   // first stage into this buffer
                const bool last = kPromote ? (kb % kPer == kPer - 1) : kb == ti.kb - 1;
                if (first) {
                    if (!mbar_spin_warp(&tempty_bar[abuf], aphase ^ 1u, &abort_sh, p.status, 0x20)) {
                        ok = false;
                        break;
                    }
                }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma<kAct8>(dt, ad + 2 * ks, bd + 2 * ks, idesc, !first || ks > 0);
                    umma_commit(&empty_bar[stage]);
                    if (last) umma_commit(&tfull_bar[abuf]);
                }
                __syncwarp();
                if (last) {
                    abuf ^= 1;
                    if (abuf == 0) aphase ^= 1u;
                }
                if (++stage == NS) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (leader) {
            umma_commit(&drain_bar);
            drain_wait(&drain_bar, 0);
        }
        __syncwarp();
      } else if constexpr (kA16) {
        // ------------------------------------------------------------------ weight widening (kA16)
        // warps 2-3: the stage's e4m3 weight tile (256 rows x 64 B, as loaded) -> bf16 rows of 128 B in
        // the 128-byte-swizzled K-major layout the MMA reads (16-byte unit u of row n at unit u ^ (n % 8))
        const int ct = threadIdx.x - 64;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            Tile ti;
            decode_tile(t, ts_sh, rb_sh, rc_sh, p, kMode, ti);
            for (int kb = 0; kb < ti.kb; ++kb) {
                const bool got = mbar_wait(&full_bar[stage], phase, &abort_sh, p.status, 0x40);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    ok = false;
                    break;
                }
                const uint8_t* raw = smem + stage * SB + kStageBytes;
                uint8_t* bb = smem + stage * SB + kStageBytesA;
#pragma unroll 2
                for (int i = 0; i < kRawBytes / 16 / 64; ++i) {
                    const int u = i * 64 + ct;          // 16-byte unit of the raw tile: row u / 4, quarter u % 4
                    const int n = u >> 2, qd = u & 3;
                    const uint4 v = *reinterpret_cast<const uint4*>(raw + n * 64 + qd * 16);
                    const uint4 lo = make_uint4(e4m3x2_to_bf16x2(v.x), e4m3x2_to_bf16x2(v.x >> 16),
                                                e4m3x2_to_bf16x2(v.y), e4m3x2_to_bf16x2(v.y >> 16));
                    const uint4 hi = make_uint4(e4m3x2_to_bf16x2(v.z), e4m3x2_to_bf16x2(v.z >> 16),
                                                e4m3x2_to_bf16x2(v.w), e4m3x2_to_bf16x2(v.w >> 16));
                    uint8_t* row = bb + n * 128;
                    *reinterpret_cast<uint4*>(row + (((2 * qd) ^ (n & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(row + (((2 * qd + 1) ^ (n & 7)) << 4)) = hi;
                }
                fence_async_shared();   // the tensor core reads these bytes through the async proxy
                mbar_arrive(&conv_bar[stage]);
                if (++stage == NS) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
      }
    } else {
        regs_inc<224>();
        // ------------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int c = (warp - 4) >> 2;
        const int r = q * 32 + lane;
        uint8_t* ostage = smem + NS * SB + (warp - 4) * kOutStageBytes;
        const uint32_t tl = tmem + (static_cast<uint32_t>(q * 32) << 16);
        int abuf = 0;
        uint32_t aphase = 0, xpar = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            Tile ti;
            decode_tile(t, ts_sh, rb_sh, rc_sh, p, kMode, ti);
            const int grow = ti.a_row0 + r;
            const bool valid = r < ti.rows_valid;
            uint8_t* out = static_cast<uint8_t*>(ti.shared ? p.out_s : p.out_r);
            const size_t out_ld = static_cast<size_t>(ti.shared ? p.out_ld_s : p.out_ld_r);
            if constexpr (kFp8 || kMode == kModeLogits) {
                // promotion: every 128-wide K block arrives in its own TMEM buffer and is added into float32
                // registers (FP8 activations: scaled by s_act[row, kb] * s_w[blk, kb]; bf16 activations
                // with FP8 weights: by s_w[blk, kb]; logits: scale 1, one 64-wide stage per block)
                float2 acc[64];
#pragma unroll
                for (int j = 0; j < 64; ++j) acc[j] = make_float2(0.0f, 0.0f);
                constexpr bool kScaled = kFp8;
                const float* as = ti.shared ? p.as_s : p.as_r;
                const size_t as_ld = static_cast<size_t>(ti.shared ? p.as_ld_s : p.as_ld_r);
                const int bcols = ti.shared ? p.bs_cols_s : p.bs_cols_r;
                const int brow = (ti.shared ? 0 : ti.g * p.bs_rows_r) + (kMode == kModeUp ? ti.nt : 2 * ti.nt + c);
                const float* sc0 = kScaled ? (ti.shared ? p.bs0_s : p.bs0_r) + static_cast<size_t>(brow) * bcols : nullptr;
                const float* sc1 = kScaled ? (ti.shared ? p.bs1_s : p.bs1_r) + static_cast<size_t>(brow) * bcols : nullptr;
                // scales of K block 0; each iteration fetches the next block's before it waits
                float sa = 1.0f, w0 = 1.0f, w1 = 1.0f;
                if constexpr (kScaled) {
                    if constexpr (kAct8) sa = as[grow];
                    w0 = __ldg(sc0);
                    w1 = (kMode == kModeUp) ? __ldg(sc1) : 0.0f;
                }
                const int npb = kA16 ? ti.kb / 2 : ti.kb;   // promoted K blocks
                bool ok = true;
                for (int kb = 0; kb < npb; ++kb) {
                    const int kn = kb + 1 < npb ? kb + 1 : kb;
                    float sa_n = 1.0f, w0_n = 1.0f, w1_n = 1.0f;
                    if constexpr (kScaled) {
                        if constexpr (kAct8) sa_n = as[static_cast<size_t>(kn) * as_ld + grow];
                        w0_n = __ldg(sc0 + kn);
                        w1_n = (kMode == kModeUp) ? __ldg(sc1 + kn) : 0.0f;
                    }
                    if (!mbar_spin(&tfull_bar[abuf], aphase, &abort_sh, p.status, 0x30)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float f0 = sa * w0;
                    const float f1 = (kMode == kModeUp) ? sa * w1 : f0;
                    const float2 f0v = make_float2(f0, f0), f1v = make_float2(f1, f1);
                    const uint32_t base = tl + static_cast<uint32_t>(abuf * kBN);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        // UP: hh 0 = g columns (64c..), hh 1 = u columns (128+64c..); DOWN / logits: 128c + 64hh
                        const int col = (kMode == kModeUp) ? (hh ? 128 : 0) + 64 * c : 128 * c + 64 * hh;
                        uint32_t v[64];
                        tmem_ld64(base + col, v);
                        tmem_wait_ld();
                        if (kMode == kModeDown && hh == 1) {
                            // down GEMM: hand the buffer back before the last FMAs (measured faster there;
                            // the up GEMM's longer tiles do better releasing after them)
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&tempty_bar[abuf]);
                        }
                        const float2 fv = hh ? f1v : f0v;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            acc[hh * 32 + j] =
                                __ffma2_rn(make_float2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])), fv, acc[hh * 32 + j]);
                    }
                    if (kMode != kModeDown) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty_bar[abuf]);
                    }
                    abuf ^= 1;
                    if (abuf == 0) aphase ^= 1u;
                    sa = sa_n;
                    w0 = w0_n;
                    w1 = w1_n;
                }
                if (!ok) break;
                float* accf = reinterpret_cast<float*>(acc);
                if constexpr (kMode == kModeLogits) {
                    // router logits, float32, columns 128c .. 128c+127 that are < n_valid_cols
                    if (valid) {
                        float* dst = reinterpret_cast<float*>(out + static_cast<size_t>(ti.ks) * p.split_stride +
                                                              static_cast<size_t>(grow) * out_ld * 4) + 128 * c;
                        const int ncol = min(128, p.n_valid_cols - 128 * c);
                        if ((p.n_valid_cols & 3) == 0) {        // rows 16-byte aligned: vector stores
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (4 * i < ncol)
                                    reinterpret_cast<float4*>(dst)[i] =
                                        make_float4(accf[4 * i], accf[4 * i + 1], accf[4 * i + 2], accf[4 * i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 128; ++i)
                                if (i < ncol) dst[i] = accf[i];
                        }
                    }
                } else if constexpr (kMode == kModeUp && kA16) {
                    // h = bf16(silu(g) * u) for I-columns nt*128 + 64c + j, stored as bf16 (no quant)
                    if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(
                            out + (static_cast<size_t>(grow) * out_ld + ti.nt * 128 + 64 * c) * 2);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            float h[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) h[e] = silu_mul(accf[8 * i + e], accf[64 + 8 * i + e]);
                            dst[i] = make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]), pack2(h[4], h[5]), pack2(h[6], h[7]));
                        }
                    }
                } else if constexpr (kMode == kModeUp) {
                    // h = bf16(silu(g) * u) for I-columns nt*128 + 64c + j, then the 1x128 FP8 quant of h
                    float amax = 0.0f;
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        accf[j] = silu_mul(accf[j], accf[64 + j]);
                        amax = fmaxf(amax, fabsf(accf[j]));
                    }
                    // the row's other 64 columns belong to the other warpgroup: exchange the maxima through
                    // shared memory, double-buffered by tile, behind a bounded wait (a hardware barrier
                    // would wait forever for a warp that left after a timeout elsewhere)
                    amax_sh[xpar][c][r] = amax;
                    mbar_arrive(&xchg_bar);
                    mbar_spin(&xchg_bar, xpar, &abort_sh, p.status, 0x32);
                    amax = fmaxf(amax, amax_sh[xpar][c ^ 1][r]);
                    xpar ^= 1u;
                    const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                    const float rsc = __frcp_rn(sc);
                    // the row's 64 e4m3 codes -> this warp's staging rows -> one TMA store of 32 x 64 bytes
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        uint32_t word = 0;
                        if (amax > 0.0f) {
#pragma unroll
                            for (int b = 0; b < 4; ++b) {
                                const uint32_t code =
                                    __nv_cvt_float_to_fp8(div_by_rcp(accf[4 * i + b], sc, rsc), __NV_SATFINITE, __NV_E4M3);
                                word |= code << (8 * b);
                            }
                        }
                        w[i] = word;
                    }
                    if (lane == 0) bulk_wait_read();
                    __syncwarp();
                    uint4* srow = reinterpret_cast<uint4*>(ostage + lane * 64);
#pragma unroll
                    for (int i = 0; i < 4; ++i) srow[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                    fence_async_shared();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(ti.shared ? &tm_o_s : &tm_o_r, ostage, ti.nt * 128 + 64 * c, ti.a_row0 + q * 32);
                        bulk_commit();
                    }
                    if (valid && c == 0) {
                        float* os = ti.shared ? p.outs_s : p.outs_r;
                        const size_t os_ld = static_cast<size_t>(ti.shared ? p.outs_ld_s : p.outs_ld_r);
                        os[static_cast<size_t>(ti.nt) * os_ld + grow] = sc;
                    }
                } else {
                    // y rows (bf16): 8 chunks of 16 columns through the two 1 KB halves of this warp's
                    // staging rows, one TMA store of 32 x 16 bf16 each; a half is refilled as soon as the
                    // store two chunks back has read it, so the stores overlap the packing
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint8_t* half = ostage + (ch & 1) * (kOutStageBytes / 2);
                        if (lane == 0) bulk_wait_read_but1();
                        __syncwarp();
                        uint4* srow = reinterpret_cast<uint4*>(half + lane * 32);
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const float* a8 = accf + ch * 16 + 8 * i;
                            srow[i] = make_uint4(pack2(a8[0], a8[1]), pack2(a8[2], a8[3]), pack2(a8[4], a8[5]),
                                                 pack2(a8[6], a8[7]));
                        }
                        fence_async_shared();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(ti.shared ? &tm_o_s : &tm_o_r, half, ti.nt * 256 + 128 * c + 16 * ch,
                                         ti.a_row0 + q * 32);
                            bulk_commit();
                        }
                    }
                }
            } else {
                // bf16: the whole K accumulated in TMEM buffer abuf
                if (!mbar_spin(&tfull_bar[abuf], aphase, &abort_sh, p.status, 0x31)) break;
                tc_fence_after();
                const uint32_t base = tl + static_cast<uint32_t>(abuf * kBN);
                if constexpr (kMode == kModeUp) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t vg[32], vu[32];
                        tmem_ld32(base + 64 * c + 32 * hh, vg);
                        tmem_ld32(base + 128 + 64 * c + 32 * hh, vu);
                        tmem_wait_ld();
                        if (valid) {
                            uint4* dst = reinterpret_cast<uint4*>(
                                out + (static_cast<size_t>(grow) * out_ld + ti.nt * 128 + 64 * c + 32 * hh) * 2);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                float h[8];
#pragma unroll
                                for (int b = 0; b < 8; ++b)
                                    h[b] = silu_mul(__uint_as_float(vg[8 * i + b]), __uint_as_float(vu[8 * i + b]));
                                dst[i] = make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]), pack2(h[4], h[5]), pack2(h[6], h[7]));
                            }
                        }
                    }
                } else if constexpr (kMode == kModeDown) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t v[32];
                        tmem_ld32(base + 128 * c + 32 * ch, v);
                        tmem_wait_ld();
                        if (valid) {
                            uint4* dst = reinterpret_cast<uint4*>(
                                out + (static_cast<size_t>(grow) * out_ld + ti.nt * 256 + 128 * c + 32 * ch) * 2);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                dst[i] = make_uint4(pack2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                                                    pack2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                                                    pack2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                                                    pack2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty_bar[abuf]);
                abuf ^= 1;
                if (abuf == 0) aphase ^= 1u;
            }
        }
    }

    if (warp >= 4 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <bool kFp8, int kMode, bool kA16 = false>
cudaError_t launch_one(const TensorMaps& m, const GemmParams& p, int grid, cudaStream_t s) {
    constexpr int smem = kA16 ? kSmemBytesA16 : kSmemBytes;
    // the shared-memory opt-in is set once per device, so that a forward enqueued during stream
    // capture (a CUDA graph) makes no call besides the launch
    {
        static std::mutex mu;
        static bool done[64] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 64 || !done[dev]) {
            e = cudaFuncSetAttribute(gemm_kernel<kFp8, kMode, kA16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) done[dev] = true;
        }
    }
    gemm_kernel<kFp8, kMode, kA16><<<grid, kGemmThreads, smem, s>>>(m.a_r, m.a_s, m.b0_r, m.b1_r, m.b0_s, m.b1_s,
                                                                    m.o_r, m.o_s, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(int mode, bool fp8, bool a16, const TensorMaps& maps, const GemmParams& p, int grid,
                        cudaStream_t s) {
    if (fp8 && a16) {
        if (mode == kModeUp) return launch_one<true, kModeUp, true>(maps, p, grid, s);
        if (mode == kModeDown) return launch_one<true, kModeDown, true>(maps, p, grid, s);
        return cudaErrorInvalidValue;
    }
    if (fp8) {
        if (mode == kModeUp) return launch_one<true, kModeUp>(maps, p, grid, s);
        if (mode == kModeDown) return launch_one<true, kModeDown>(maps, p, grid, s);
        return cudaErrorInvalidValue;
    }
    if (mode == kModeUp) return launch_one<false, kModeUp>(maps, p, grid, s);
    if (mode == kModeDown) return launch_one<false, kModeDown>(maps, p, grid, s);
    return launch_one<false, kModeLogits>(maps, p, grid, s);
}

}  // namespace moe
