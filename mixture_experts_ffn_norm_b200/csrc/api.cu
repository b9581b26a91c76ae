// Host side of libmoe: argument checks, workspace layout, TMA tensor maps and the launch
// sequence of one forward pass.  Nothing here waits on the device except moe_get_status.
//
// Launch sequence (one stream, no host sync; every routing-dependent size is read on the device):
//   norm -> gate GEMM (logits; K split over CTAs for few tokens) -> top-k (float32 pass, then the
//   float64 re-decision of the listed near-tie tokens) -> hist -> scan -> scatter -> gather
//   -> grouped GEMM up (w1|w3 + SwiGLU) -> grouped GEMM down (w2) -> combine
// The combine has two variants: with the next block's RMSNorm fused in (moe_forward_next_norm)
// and the float32 partial of an expert slice (moe_forward_expert_slice).  A dense block
// (n_experts = 0) runs norm -> up -> down, the second GEMM writing the output.  Tensor maps are
// cached on the host (a map is a pure function of its arguments).
#include <algorithm>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Host-side cache of encoded tensor maps.  A map is a pure function of its arguments (address,
// type, extents, strides, box, swizzle), so the key is all of them and an entry never goes stale;
// a forward call then encodes only maps it has not seen.  Bounded: cleared when it grows large.
struct MapKey {
    const void* base;
    uint64_t d0, d1, stride;
    uint32_t b0, b1;
    int dtype, swizzle, promo;
    bool operator==(const MapKey& o) const {
        return base == o.base && d0 == o.d0 && d1 == o.d1 && stride == o.stride && b0 == o.b0 && b1 == o.b1 &&
               dtype == o.dtype && swizzle == o.swizzle && promo == o.promo;
    }
};
struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        uint64_t h = reinterpret_cast<uintptr_t>(k.base);
        for (uint64_t v : {k.d0, k.d1, k.stride, static_cast<uint64_t>(k.b0) << 32 | k.b1,
                           static_cast<uint64_t>(k.dtype) << 16 | static_cast<uint64_t>(k.swizzle) << 8 |
                               static_cast<uint64_t>(k.promo)})
            h = (h ^ v) * 0x100000001B3ull;
        return static_cast<size_t>(h ^ (h >> 29));
    }
};

bool encode_cached(CUtensorMap* map, CUtensorMapDataType dtype, void* base, uint64_t d0, uint64_t d1,
                   uint64_t stride, uint32_t b0, uint32_t b1, CUtensorMapSwizzle swizzle,
                   CUtensorMapL2promotion promo) {
    static std::mutex mu;
    static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
    const MapKey key{base, d0, d1, stride, b0, b1, static_cast<int>(dtype), static_cast<int>(swizzle),
                     static_cast<int>(promo)};
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) {
            *map = it->second;
            return true;
        }
    }
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {d0, d1};
    const cuuint64_t strides[1] = {stride};
    const cuuint32_t box[2] = {b0, b1};
    const cuuint32_t estr[2] = {1u, 1u};
    if (enc(map, dtype, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() >= 4096) cache.clear();
    cache.emplace(key, *map);
    return true;
}

}  // namespace

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// 2-D map over a row-major [rows, inner] tensor of 1-byte (fp8) or 2-byte (bf16) elements; box =
// 128 bytes x 128 rows, 128-byte swizzle, out-of-range rows read as zero.
bool encode_map_2d(CUtensorMap* map, const void* base, bool fp8, uint64_t inner, uint64_t rows) {
    return encode_cached(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         const_cast<void*>(base), inner, rows, inner * (fp8 ? 1u : 2u), fp8 ? 128u : 64u, 128u,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

bool encode_raw_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows) {
    return encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<void*>(base), inner, rows, inner, 64u, 128u,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

bool encode_store_map_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t inner, uint64_t rows,
                         uint32_t box_inner) {
    return encode_cached(map, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         const_cast<void*>(base), inner, rows, inner * static_cast<uint64_t>(elem_bytes), box_inner,
                         32u, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE);
}

bool make_layout(const moe_config_t& c, Layout& L) {
    if (c.num_tokens < 1 || c.dim < 256 || c.dim % 256 || c.dim > 8192 || c.inter_dim < 128 || c.inter_dim % 128)
        return false;
    if (c.n_experts == 0) {
        // dense block: no router, the MLP is the shared SwiGLU
        if (c.top_k != 0 || c.shared_inter < 128) return false;
    } else {
        if (c.n_experts < 1 || c.n_experts > kMaxExperts || (c.n_experts > 8 && c.n_experts % 8)) return false;
        if (c.top_k < 1 || c.top_k > c.n_experts) return false;
    }
    if (c.shared_inter < 0 || c.shared_inter % 128) return false;
    if (c.wtype != MOE_W_BF16 && c.wtype != MOE_W_FP8_E4M3_B128) return false;
    if (c.amode != MOE_ACT_FP8_1x128 && c.amode != MOE_ACT_BF16) return false;
    if (!(c.eps >= 0.0f)) return false;
    if (static_cast<long long>(c.num_tokens) * c.top_k > (1ll << 30)) return false;
    L.T = c.num_tokens;
    L.d = c.dim;
    L.I = c.inter_dim;
    L.E = c.n_experts;
    L.k = c.top_k;
    L.Is = c.shared_inter;
    L.fp8 = c.wtype == MOE_W_FP8_E4M3_B128;
    L.dense = c.n_experts == 0;
    L.act8 = L.fp8 && c.amode == MOE_ACT_FP8_1x128;
    L.Tpad = static_cast<int>(align_up(L.T, kBM));
    L.R = static_cast<int>(align_up(static_cast<size_t>(L.T) * L.k + static_cast<size_t>(L.E) * (kBM - 1), kBM));
    L.KBd = L.d / 128;
    L.KBi = L.I / 128;
    L.KBs = L.Is / 128;
    L.nchunks = (L.T * L.k + kRouteChunk - 1) / kRouteChunk;
    const size_t ab = L.act8 ? 1 : 2;   // bytes per activation element fed to the expert GEMMs
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes, 1024);
        return at;
    };
    L.status = take(kStatusWords * 4);
    L.xn = take(static_cast<size_t>(L.T) * L.d * 2);
    L.xq = take(L.act8 ? static_cast<size_t>(L.T) * L.d : 0);
    L.xs = take(L.act8 ? static_cast<size_t>(L.KBd) * L.Tpad * 4 : 0);
    // few tokens leave the router GEMM with few tiles: split its K so that more SMs stream it
    {
        const int tiles = (L.T + kBM - 1) / kBM;
        L.ksplit = tiles >= 64 ? 1 : std::min({16, 128 / tiles, L.d / 64});
    }
    L.logits = take(static_cast<size_t>(L.T) * L.E * 4 * L.ksplit);
    L.idx = take(static_cast<size_t>(L.T) * L.k * 4);
    L.w = take(static_cast<size_t>(L.T) * L.k * 4);
    L.flag = take(L.T);
    L.redo = take(static_cast<size_t>(L.T) * 4);     // tokens listed for the float64 re-decision
    L.counts = take(static_cast<size_t>(L.E) * 4);
    L.offsets = take(static_cast<size_t>(L.E + 1) * 4);
    L.row_base = take(static_cast<size_t>(L.E + 1) * 4);
    L.row_count = take(static_cast<size_t>(L.E + 1) * 4);
    L.ts_up = take(static_cast<size_t>(L.E + 2) * 4);
    L.ts_down = take(static_cast<size_t>(L.E + 2) * 4);
    L.chunk_hist = take(static_cast<size_t>(L.nchunks) * L.E * 4);
    L.row_of = take(static_cast<size_t>(L.T) * L.k * 4);
    L.row_token = take(static_cast<size_t>(L.R) * 4);
    L.a_perm = take(static_cast<size_t>(L.R) * L.d * ab);
    L.as_perm = take(L.act8 ? static_cast<size_t>(L.KBd) * L.R * 4 : 0);
    L.h = take(static_cast<size_t>(L.R) * L.I * ab);
    L.hs = take(L.act8 ? static_cast<size_t>(L.KBi) * L.R * 4 : 0);
    L.h_sh = take(static_cast<size_t>(L.Tpad) * L.Is * ab);
    L.hs_sh = take(L.act8 ? static_cast<size_t>(L.KBs) * L.Tpad * 4 : 0);
    L.y = take(static_cast<size_t>(L.R) * L.d * 2);
    L.y_sh = take(L.dense ? 0 : static_cast<size_t>(L.T) * L.d * 2);   // dense: the MLP writes out directly
    L.total = o;
    return true;
}

}  // namespace moe

using namespace moe;

namespace {

moe_status_t check_config(const moe_config_t* cfg, Layout& L) {
    if (!cfg || !make_layout(*cfg, L)) return MOE_ERR_INVALID_ARG;
    if (cfg->wtype == MOE_W_BF16 && cfg->amode != MOE_ACT_BF16) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

#define MOE_TRY(expr)                          \
    do {                                       \
        if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

}  // namespace

extern "C" size_t moe_workspace_bytes(const moe_config_t* cfg) {
    Layout L;
    if (check_config(cfg, L) != MOE_OK) return 0;
    return L.total;
}

extern "C" int32_t moe_launches_per_forward(const moe_config_t* cfg) {
    Layout L;
    if (check_config(cfg, L) != MOE_OK) return 0;
    return L.dense ? 3 : 11;   // norm, gate GEMM, top-k (2), hist, scan, scatter, gather, up, down, combine
}

// A dense block's MLP ("MoE update" page, Block excerpt: MLP(dim, inter_dim) in the first blocks):
// the two GEMMs of the SwiGLU over all T tokens as one group, the second writing the bf16 output
// rows straight into `out` (there is nothing to combine).
static cudaError_t dense_mlp(const Layout& L, const moe_weights_t* w, uint8_t* ws, void* out, int sms,
                             cudaStream_t s, int part) {
    const bool fp8 = L.fp8, act8 = L.act8, a16 = fp8 && !act8;
    auto bmap = [&](CUtensorMap* mp, const void* base, uint64_t inner, uint64_t rows) {
        return a16 ? encode_raw_map_2d(mp, base, inner, rows) : encode_map_2d(mp, base, fp8, inner, rows);
    };
    const int mtiles = (L.T + kBM - 1) / kBM;
    if (part == 0) {   // h = silu(xn W1^T) * (xn W3^T)
        TensorMaps m;
        bool ok = encode_map_2d(&m.a_s, ws + (act8 ? L.xq : L.xn), act8, L.d, L.T) &&
                  bmap(&m.b0_s, w->sw1, L.d, L.Is) && bmap(&m.b1_s, w->sw3, L.d, L.Is);
        if (act8) ok = ok && encode_store_map_2d(&m.o_s, ws + L.h_sh, 1, L.Is, L.Tpad, 64);
        else m.o_s = m.a_s;
        if (!ok) return cudaErrorInvalidValue;
        m.a_r = m.a_s, m.b0_r = m.b0_s, m.b1_r = m.b1_s, m.o_r = m.o_s;
        GemmParams p{};
        p.G = 1;
        p.single_rows = L.T;
        p.n_tiles_s = L.Is / 128;
        p.kb_s = act8 ? L.d / 128 : L.d / 64;
        p.as_s = reinterpret_cast<const float*>(ws + L.xs);
        p.as_ld_s = L.Tpad;
        p.bs0_s = w->ss1;
        p.bs1_s = w->ss3;
        p.bs_cols_s = L.d / 128;
        p.out_s = ws + L.h_sh;
        p.out_ld_s = L.Is;
        p.outs_s = reinterpret_cast<float*>(ws + L.hs_sh);
        p.outs_ld_s = L.Tpad;
        p.status = reinterpret_cast<uint32_t*>(ws + L.status);
        return launch_gemm(kModeUp, fp8, a16, m, p, std::min(mtiles * p.n_tiles_s, sms), s);
    }
    {   // out = h W2^T
        TensorMaps m;
        bool ok = encode_map_2d(&m.a_s, ws + L.h_sh, act8, L.Is, L.Tpad) && bmap(&m.b0_s, w->sw2, L.Is, L.d);
        if (fp8) ok = ok && encode_store_map_2d(&m.o_s, out, 2, L.d, L.T, 16);
        else m.o_s = m.a_s;
        if (!ok) return cudaErrorInvalidValue;
        m.b1_s = m.b0_s;
        m.a_r = m.a_s, m.b0_r = m.b0_s, m.b1_r = m.b0_s, m.o_r = m.o_s;
        GemmParams p{};
        p.G = 1;
        p.single_rows = L.T;
        p.n_tiles_s = L.d / 256;
        p.kb_s = act8 ? L.Is / 128 : L.Is / 64;
        p.as_s = reinterpret_cast<const float*>(ws + L.hs_sh);
        p.as_ld_s = L.Tpad;
        p.bs0_s = p.bs1_s = w->ss2;
        p.bs_cols_s = L.Is / 128;
        p.out_s = out;
        p.out_ld_s = L.d;
        p.status = reinterpret_cast<uint32_t*>(ws + L.status);
        return launch_gemm(kModeDown, fp8, a16, m, p, std::min(mtiles * p.n_tiles_s, sms), s);
    }
}

static moe_status_t forward_impl(const moe_config_t* cfg, const void* x, const void* residual,
                                 const float* norm_w, const void* gate_w, const float* gate_bias,
                                 const moe_weights_t* w, void* out, void* residual_out, void* workspace,
                                 size_t workspace_bytes, void* stream_, void* const* events, int n_events,
                                 const float* next_norm_w = nullptr, void* next_xn = nullptr,
                                 float* y_partial = nullptr, int ebeg = 0, int eend = -1, bool shared_here = true) {
    Layout L;
    moe_status_t st = check_config(cfg, L);
    if (st != MOE_OK) return st;
    const bool slice = y_partial != nullptr;   // expert slice: float32 partial of experts [ebeg, eend)
    if (eend < 0) eend = L.E;
    if (slice && (L.dense || next_xn)) return MOE_ERR_UNSUPPORTED;
    if (slice && (ebeg < 0 || ebeg > eend || eend > L.E || !aligned16(y_partial) || y_partial == x ||
                  y_partial == residual || y_partial == residual_out))
        return MOE_ERR_INVALID_ARG;
    const bool next = next_xn != nullptr;   // the next block's attn_norm fused into the combine
    if (next && L.dense) return MOE_ERR_UNSUPPORTED;
    if (next && (!next_norm_w || !residual || !residual_out)) return MOE_ERR_INVALID_ARG;
    if (next && (next_xn == x || next_xn == residual || next_xn == out || next_xn == residual_out ||
                 !aligned16(next_xn) || !aligned16(next_norm_w)))
        return MOE_ERR_INVALID_ARG;
    if (!x || !norm_w || !w || (!out && !next && !slice)) return MOE_ERR_INVALID_ARG;
    if (residual && !residual_out) return MOE_ERR_INVALID_ARG;
    if (!L.dense) {
        if (!gate_w || !w->w1 || !w->w3 || !w->w2) return MOE_ERR_INVALID_ARG;
        if (L.fp8 && (!w->s1 || !w->s3 || !w->s2)) return MOE_ERR_INVALID_ARG;
    }
    if (L.Is > 0) {
        if (!w->sw1 || !w->sw3 || !w->sw2) return MOE_ERR_INVALID_ARG;
        if (L.fp8 && (!w->ss1 || !w->ss3 || !w->ss2)) return MOE_ERR_INVALID_ARG;
    }
    const void* ptrs[] = {x, residual, norm_w, gate_w, gate_bias, w->w1, w->w3, w->w2, w->sw1, w->sw3, w->sw2,
                          out, residual_out};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    if ((out && (out == x || out == residual)) || (residual_out && (residual_out == x || residual_out == out)))
        return MOE_ERR_INVALID_ARG;

    cudaStream_t s = static_cast<cudaStream_t>(stream_);
    auto mark = [&](int i) {
        return (events && i < n_events && events[i]) ? cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s)
                                                     : cudaSuccess;
    };
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int sms = num_sms();
    const bool fp8 = L.fp8;
    const bool act8 = L.act8;           // FP8 activations into the expert GEMMs
    const bool a16 = fp8 && !act8;      // FP8 weights widened to bf16 next to bf16 activations

    MOE_TRY(cudaMemsetAsync(ws + L.status, 0, kStatusWords * 4, s));
    MOE_TRY(cudaMemsetAsync(ws + L.row_token, 0xFF, static_cast<size_t>(L.R) * 4, s));
    MOE_TRY(mark(0));

    // 1. ffn_norm (+ FP8 activation quant)
    MOE_TRY(launch_norm(L, x, residual, norm_w, cfg->eps, residual_out, ws, s));
    MOE_TRY(mark(1));
    if (L.dense) {
        MOE_TRY(mark(2));
        MOE_TRY(mark(3));
        MOE_TRY(mark(4));
        MOE_TRY(dense_mlp(L, w, ws, out, sms, s, 0));
        MOE_TRY(mark(5));
        MOE_TRY(dense_mlp(L, w, ws, out, sms, s, 1));
        MOE_TRY(mark(6));
        MOE_TRY(mark(7));
        return MOE_OK;
    }

    // 2. router logits on the tensor cores: xn [T, d] x Wg [E, d]^T
    {
        TensorMaps m;
        if (!encode_map_2d(&m.a_s, ws + L.xn, false, L.d, L.T) || !encode_map_2d(&m.b0_s, gate_w, false, L.d, L.E))
            return MOE_ERR_CUDA;
        m.a_r = m.a_s;
        m.b1_s = m.b0_s;
        m.b0_r = m.b0_s;
        m.b1_r = m.b0_s;
        m.o_r = m.a_s;
        m.o_s = m.a_s;
        GemmParams p{};
        p.G = 1;
        p.single_rows = L.T;
        p.n_tiles_s = 1;
        p.kb_s = L.d / 64;
        p.ksplit = L.ksplit;
        p.kb_chunk = (p.kb_s + L.ksplit - 1) / L.ksplit;
        p.split_stride = static_cast<size_t>(L.T) * L.E * 4;
        p.out_s = ws + L.logits;
        p.out_ld_s = L.E;
        p.n_valid_cols = L.E;
        p.status = reinterpret_cast<uint32_t*>(ws + L.status);
        const int tiles = (L.T + kBM - 1) / kBM * L.ksplit;
        MOE_TRY(launch_gemm(kModeLogits, false, false, m, p, std::min(tiles, sms), s));
    }
    MOE_TRY(mark(2));
    // 3. top-k, re-decided in float64 near the boundary
    MOE_TRY(launch_topk(L, gate_w, gate_bias, ws, s));
    MOE_TRY(mark(3));

    // 4. permutation by expert
    const int ntu_r = L.I / 128, ntu_s = L.Is / 128, ntd = L.d / 256;
    MOE_TRY(launch_route(L, ntu_r, ntu_s, ntd, ntd, ws, s, ebeg, eend, shared_here));
    MOE_TRY(mark(4));

    const int G = L.E + (L.Is > 0 ? 1 : 0);
    const int max_tiles_up = (L.R / kBM) * ntu_r + (L.Is > 0 ? (L.Tpad / kBM) * ntu_s : 0);
    const int max_tiles_down = (L.R / kBM) * ntd + (L.Is > 0 ? (L.Tpad / kBM) * ntd : 0);

    // 5. grouped GEMM up: h = silu(a W1^T) * (a W3^T)
    {
        TensorMaps m;
        auto bmap = [&](CUtensorMap* mp, const void* base, uint64_t inner, uint64_t rows) {
            return a16 ? encode_raw_map_2d(mp, base, inner, rows) : encode_map_2d(mp, base, fp8, inner, rows);
        };
        bool ok = encode_map_2d(&m.a_r, ws + L.a_perm, act8, L.d, L.R) &&
                  encode_map_2d(&m.a_s, ws + (act8 ? L.xq : L.xn), act8, L.d, L.T) &&
                  bmap(&m.b0_r, w->w1, L.d, static_cast<uint64_t>(L.E) * L.I) &&
                  bmap(&m.b1_r, w->w3, L.d, static_cast<uint64_t>(L.E) * L.I);
        if (L.Is > 0)
            ok = ok && bmap(&m.b0_s, w->sw1, L.d, L.Is) && bmap(&m.b1_s, w->sw3, L.d, L.Is);
        else
            m.b0_s = m.b0_r, m.b1_s = m.b1_r;
        if (act8) {
            ok = ok && encode_store_map_2d(&m.o_r, ws + L.h, 1, L.I, L.R, 64);
            if (L.Is > 0) ok = ok && encode_store_map_2d(&m.o_s, ws + L.h_sh, 1, L.Is, L.Tpad, 64);
            else m.o_s = m.o_r;
        } else {
            m.o_r = m.a_r, m.o_s = m.a_r;
        }
        if (!ok) return MOE_ERR_CUDA;
        GemmParams p{};
        p.G = G;
        p.has_shared = L.Is > 0;
        p.tile_start = reinterpret_cast<const int*>(ws + L.ts_up);
        p.row_base = reinterpret_cast<const int*>(ws + L.row_base);
        p.row_count = reinterpret_cast<const int*>(ws + L.row_count);
        p.n_tiles_r = ntu_r;
        p.n_tiles_s = ntu_s;
        p.kb_r = p.kb_s = act8 ? L.d / 128 : L.d / 64;
        p.b_rows_per_expert = L.I;
        p.as_r = reinterpret_cast<const float*>(ws + L.as_perm);
        p.as_s = reinterpret_cast<const float*>(ws + L.xs);
        p.as_ld_r = L.R;
        p.as_ld_s = L.Tpad;
        p.bs0_r = w->s1;
        p.bs1_r = w->s3;
        p.bs0_s = w->ss1;
        p.bs1_s = w->ss3;
        p.bs_cols_r = p.bs_cols_s = L.d / 128;
        p.bs_rows_r = L.I / 128;
        p.out_r = ws + L.h;
        p.out_s = ws + L.h_sh;
        p.out_ld_r = L.I;
        p.out_ld_s = L.Is;
        p.outs_r = reinterpret_cast<float*>(ws + L.hs);
        p.outs_s = reinterpret_cast<float*>(ws + L.hs_sh);
        p.outs_ld_r = L.R;
        p.outs_ld_s = L.Tpad;
        p.status = reinterpret_cast<uint32_t*>(ws + L.status);
        MOE_TRY(launch_gemm(kModeUp, fp8, a16, m, p, std::min(max_tiles_up, sms), s));
    }
    MOE_TRY(mark(5));
    // 6. grouped GEMM down: y = h W2^T
    {
        TensorMaps m;
        auto bmap = [&](CUtensorMap* mp, const void* base, uint64_t inner, uint64_t rows) {
            return a16 ? encode_raw_map_2d(mp, base, inner, rows) : encode_map_2d(mp, base, fp8, inner, rows);
        };
        bool ok = encode_map_2d(&m.a_r, ws + L.h, act8, L.I, L.R) &&
                  bmap(&m.b0_r, w->w2, L.I, static_cast<uint64_t>(L.E) * L.d);
        m.b1_r = m.b0_r;
        if (L.Is > 0) {
            ok = ok && encode_map_2d(&m.a_s, ws + L.h_sh, act8, L.Is, L.Tpad) &&
                 bmap(&m.b0_s, w->sw2, L.Is, L.d);
            m.b1_s = m.b0_s;
        } else {
            m.a_s = m.a_r, m.b0_s = m.b0_r, m.b1_s = m.b0_r;
        }
        if (fp8) {
            ok = ok && encode_store_map_2d(&m.o_r, ws + L.y, 2, L.d, L.R, 16);
            if (L.Is > 0) ok = ok && encode_store_map_2d(&m.o_s, ws + L.y_sh, 2, L.d, L.T, 16);
            else m.o_s = m.o_r;
        } else {
            m.o_r = m.a_r, m.o_s = m.a_r;
        }
        if (!ok) return MOE_ERR_CUDA;
        GemmParams p{};
        p.G = G;
        p.has_shared = L.Is > 0;
        p.tile_start = reinterpret_cast<const int*>(ws + L.ts_down);
        p.row_base = reinterpret_cast<const int*>(ws + L.row_base);
        p.row_count = reinterpret_cast<const int*>(ws + L.row_count);
        p.n_tiles_r = p.n_tiles_s = ntd;
        p.kb_r = act8 ? L.I / 128 : L.I / 64;
        p.kb_s = act8 ? L.Is / 128 : L.Is / 64;
        p.b_rows_per_expert = L.d;
        p.as_r = reinterpret_cast<const float*>(ws + L.hs);
        p.as_s = reinterpret_cast<const float*>(ws + L.hs_sh);
        p.as_ld_r = L.R;
        p.as_ld_s = L.Tpad;
        p.bs0_r = p.bs1_r = w->s2;
        p.bs0_s = p.bs1_s = w->ss2;
        p.bs_cols_r = L.I / 128;
        p.bs_cols_s = L.Is / 128;
        p.bs_rows_r = L.d / 128;
        p.out_r = ws + L.y;
        p.out_s = ws + L.y_sh;
        p.out_ld_r = p.out_ld_s = L.d;
        p.status = reinterpret_cast<uint32_t*>(ws + L.status);
        MOE_TRY(launch_gemm(kModeDown, fp8, a16, m, p, std::min(max_tiles_down, sms), s));
    }
    MOE_TRY(mark(6));
    // 7. weighted combine + shared add -> out
    if (slice)
        MOE_TRY(launch_combine_partial(L, y_partial, ebeg, eend, shared_here, ws, s));
    else if (next)
        MOE_TRY(launch_combine_next_norm(L, out, next_norm_w, cfg->eps, residual_out, next_xn, ws, s));
    else
        MOE_TRY(launch_combine(L, out, ws, s));
    MOE_TRY(mark(7));
    return MOE_OK;
}

extern "C" moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const void* residual,
                                    const float* norm_w, const void* gate_w, const float* gate_bias,
                                    const moe_weights_t* w, void* out, void* residual_out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
    return forward_impl(cfg, x, residual, norm_w, gate_w, gate_bias, w, out, residual_out, workspace,
                        workspace_bytes, stream, nullptr, 0);
}

extern "C" moe_status_t moe_forward_next_norm(const moe_config_t* cfg, const void* x, const void* residual,
                                              const float* norm_w, const void* gate_w, const float* gate_bias,
                                              const moe_weights_t* w, const float* next_norm_w, void* out,
                                              void* next_xn, void* next_residual, void* workspace,
                                              size_t workspace_bytes, void* stream) {
    if (!next_xn) return MOE_ERR_INVALID_ARG;
    return forward_impl(cfg, x, residual, norm_w, gate_w, gate_bias, w, out, next_residual, workspace,
                        workspace_bytes, stream, nullptr, 0, next_norm_w, next_xn);
}

extern "C" moe_status_t moe_forward_expert_slice(const moe_config_t* cfg, const void* x, const void* residual,
                                                 const float* norm_w, const void* gate_w, const float* gate_bias,
                                                 const moe_weights_t* w, int32_t expert_begin, int32_t expert_end,
                                                 int32_t with_shared, float* y_partial, void* residual_out,
                                                 void* workspace, size_t workspace_bytes, void* stream) {
    if (!y_partial) return MOE_ERR_INVALID_ARG;
    return forward_impl(cfg, x, residual, norm_w, gate_w, gate_bias, w, nullptr, residual_out, workspace,
                        workspace_bytes, stream, nullptr, 0, nullptr, nullptr, y_partial, expert_begin, expert_end,
                        with_shared != 0);
}

extern "C" moe_status_t moe_round_bf16(const float* y, void* out, int64_t n, void* stream) {
    if (!y || !out || n < 0 || (n & 3) || !aligned16(y) || (reinterpret_cast<uintptr_t>(out) & 7u))
        return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    MOE_TRY(launch_round_bf16(y, out, n, static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

extern "C" moe_status_t moe_forward_traced(const moe_config_t* cfg, const void* x, const void* residual,
                                           const float* norm_w, const void* gate_w, const float* gate_bias,
                                           const moe_weights_t* w, void* out, void* residual_out, void* workspace,
                                           size_t workspace_bytes, void* stream, void* const* events,
                                           int32_t n_events) {
    return forward_impl(cfg, x, residual, norm_w, gate_w, gate_bias, w, out, residual_out, workspace,
                        workspace_bytes, stream, events, n_events);
}

extern "C" moe_status_t moe_get_status(const void* workspace, void* stream) {
    if (!workspace) return MOE_ERR_INVALID_ARG;
    uint32_t st[2] = {0, 0};
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(st, workspace, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (st[0] == kErrTimeout) return MOE_ERR_DEVICE_TIMEOUT;
    if (st[0] != 0) return MOE_ERR_DEVICE_CHECK;
    return MOE_OK;
}

extern "C" moe_status_t moe_debug_routing(const moe_config_t* cfg, const void* workspace, int32_t* idx,
                                          float* weights, int32_t* counts, uint8_t* near_tie, void* stream) {
    Layout L;
    moe_status_t st = check_config(cfg, L);
    if (st != MOE_OK) return st;
    if (L.dense) return MOE_ERR_INVALID_ARG;   // a dense block has no routing
    if (!workspace) return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint8_t* ws = static_cast<const uint8_t*>(workspace);
    const size_t tk = static_cast<size_t>(L.T) * L.k;
    if (idx) MOE_TRY(cudaMemcpyAsync(idx, ws + L.idx, tk * 4, cudaMemcpyDeviceToDevice, s));
    if (weights) MOE_TRY(cudaMemcpyAsync(weights, ws + L.w, tk * 4, cudaMemcpyDeviceToDevice, s));
    if (counts) MOE_TRY(cudaMemcpyAsync(counts, ws + L.counts, static_cast<size_t>(L.E) * 4, cudaMemcpyDeviceToDevice, s));
    if (near_tie) MOE_TRY(cudaMemcpyAsync(near_tie, ws + L.flag, L.T, cudaMemcpyDeviceToDevice, s));
    return MOE_OK;
}

extern "C" moe_status_t moe_debug_norm(const moe_config_t* cfg, const void* workspace, void* xn, void* xq,
                                       float* xs, void* stream) {
    Layout L;
    moe_status_t st = check_config(cfg, L);
    if (st != MOE_OK) return st;
    if (!workspace) return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint8_t* ws = static_cast<const uint8_t*>(workspace);
    const size_t td = static_cast<size_t>(L.T) * L.d;
    if (xn) MOE_TRY(cudaMemcpyAsync(xn, ws + L.xn, td * 2, cudaMemcpyDeviceToDevice, s));
    if ((xq || xs) && !L.act8) return MOE_ERR_INVALID_ARG;
    if (xq) MOE_TRY(cudaMemcpyAsync(xq, ws + L.xq, td, cudaMemcpyDeviceToDevice, s));
    if (xs)
        MOE_TRY(cudaMemcpy2DAsync(xs, static_cast<size_t>(L.T) * 4, ws + L.xs, static_cast<size_t>(L.Tpad) * 4,
                                  static_cast<size_t>(L.T) * 4, L.KBd, cudaMemcpyDeviceToDevice, s));
    return MOE_OK;
}

extern "C" const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA call or kernel launch failed";
        case MOE_ERR_DEVICE_TIMEOUT: return "a device-side bounded wait gave up";
        case MOE_ERR_DEVICE_CHECK: return "a device-side check failed";
    }
    return "unknown status";
}
