// Host side of libsa: argument validation, TMA descriptors and launches for the C-ABI
// declared in include/sa.h.  All kernels live in the headers included below (one
// translation unit, so the device error word is shared by every kernel).
#include <math.h>
#include <mutex>
#include <string.h>

#include "k_attn_bwd.cuh"
#include "k_attn_prep.cuh"
#include "k_attn_tc.cuh"
#include "k_attn_tcg.cuh"
#include "k_budget.cuh"
#include "k_pool.cuh"
#include "k_scores_tc.cuh"
#include "k_select.cuh"
#include "k_sga.cuh"

// Fixed scratch of sa_select_topk_noalloc: one block of score rows (2 Mi floats = 8 MiB).
constexpr long long kNoallocScratchFloats = 1ll << 21;
// 64 rows of the longest row any selection accepts (SEL_MAX_NT) fit, so SEL_MAX_NT is the
// binding limit of the no-allocation call.
static_assert(kNoallocScratchFloats >= 64ll * SEL_MAX_NT, "scratch must hold 64 rows of SEL_MAX_NT scores");
static __device__ __align__(256) float g_sa_noalloc_scores[kNoallocScratchFloats];

namespace {

constexpr int kTcSlots = 2;
constexpr int kTcStages = 2;       // per slot, sparse calls: the mask operands take the third stage's room
constexpr int kTcStagesDense = 3;  // per slot, dense calls: one partial tile per head, masked in the softmax
constexpr int kMaxDevices = 64;

struct Geo {
    int64_t bh, S, N, d, T, n_sink, tpf, nt, L;
    bool bf16;
    float scale;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sa_status geo_of(const sa_shape* s, Geo* g) {
    if (!s) return SA_ERR_INVALID_ARG;
    if (s->bh < 1 || s->frames < 1 || s->tokens < 1 || s->head_dim < 1 || s->tile < 1 || s->n_sink < 0 ||
        s->n_sink >= s->tokens)
        return SA_ERR_INVALID_ARG;
    if (s->dtype != SA_F32 && s->dtype != SA_BF16) return SA_ERR_INVALID_ARG;
    if (!(s->softmax_scale >= 0.0f) || isinf(s->softmax_scale)) return SA_ERR_INVALID_ARG;
    g->bh = s->bh;
    g->S = s->frames;
    g->N = s->tokens;
    g->d = s->head_dim;
    g->T = s->tile;
    g->n_sink = s->n_sink;
    g->tpf = (s->tokens + s->tile - 1) / s->tile;
    g->nt = g->S * g->tpf;
    g->L = g->S * g->N;
    g->bf16 = s->dtype == SA_BF16;
    g->scale = s->softmax_scale > 0.0f ? s->softmax_scale : (float)(1.0 / sqrt((double)s->head_dim));
    if (g->bh * g->L >= (int64_t(1) << 31) || g->nt >= (int64_t(1) << 31)) return SA_ERR_UNSUPPORTED;
    if (s->head_dim != 64) return SA_ERR_UNSUPPORTED;
    if (s->tile != 64 && s->tile != 128) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

int64_t candidate_slots(const Geo& g) {
    int64_t n = 0;
    for (int64_t slot = 0; slot < g.tpf; ++slot) {
        const int64_t n0 = slot * g.T;
        const int64_t nq = std::min<int64_t>(g.T, g.N - n0);
        if (nq > std::max<int64_t>(0, g.n_sink - n0)) ++n;
    }
    return n;
}

int64_t max_kept_of(const Geo& g, int64_t k) {
    const int64_t c = (g.S - 1) * candidate_slots(g);
    return g.tpf + std::min(k, c);
}

sa_status launch_status() {
    const cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    return SA_OK;
}

// ---- per-device one-time kernel attributes
std::mutex g_attr_mu;
bool g_attr_done[kMaxDevices];
bool g_tc_regs_ok[kMaxDevices];
int g_sm_count[kMaxDevices];  // SMs per device, read once with the attributes

sa_status ensure_attributes() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_attr_mu);
    if (g_attr_done[dev]) return SA_OK;
    bool ok = true;
    ok &= cudaFuncSetAttribute(attn_tc_kernel<kTcSlots, kTcStages, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_tc_kernel<kTcSlots, kTcStages, true, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_tc_kernel<kTcSlots, kTcStagesDense, false, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_tcg_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)tcg::Cfg<false>::smem_bytes()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_tcg_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)tcg::Cfg<true>::smem_bytes()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)bw::QLay::smem_bytes()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)bw::KVLay::smem_bytes()) == cudaSuccess;
    ok &= cudaFuncSetAttribute(score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)stc::kSmemBytes) == cudaSuccess;
    ok &= cudaFuncSetAttribute(head_stat_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, BUDGET_SMEM) ==
          cudaSuccess;
    ok &= cudaFuncSetAttribute(select_topk_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SEL_SMEM_BUDGET) == cudaSuccess;
    ok &= cudaFuncSetAttribute(select_topk_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)select_block_smem_bytes(SEL_MAX_NT)) == cudaSuccess;
    // The tensor-core kernel moves registers between its warpgroups (setmaxnreg); that is only
    // satisfiable if the block is launched with at least the registers the split hands out.
    cudaFuncAttributes fa, fa_lm, fa_d;
    ok &= cudaFuncGetAttributes(&fa, attn_tc_kernel<kTcSlots, kTcStages, false, true>) == cudaSuccess;
    ok &= cudaFuncGetAttributes(&fa_lm, attn_tc_kernel<kTcSlots, kTcStages, true, true>) == cudaSuccess;
    ok &= cudaFuncGetAttributes(&fa_d, attn_tc_kernel<kTcSlots, kTcStagesDense, false, false>) == cudaSuccess;
    using Lay = TcLayout<kTcSlots, kTcStages, true>;
    using LayD = TcLayout<kTcSlots, kTcStagesDense, false>;
    if (!ok) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    g_tc_regs_ok[dev] = (uint32_t)fa.numRegs * (uint32_t)Lay::kThreads >= Lay::kRegsNeeded &&
                        (uint32_t)fa_lm.numRegs * (uint32_t)Lay::kThreads >= Lay::kRegsNeeded &&
                        (uint32_t)fa_d.numRegs * (uint32_t)LayD::kThreads >= LayD::kRegsNeeded;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    g_sm_count[dev] = sms;
    g_attr_done[dev] = true;
    return SA_OK;
}

// ---- fixed scratch for sa_select_topk_noalloc: one block of score rows (8 MiB), part of the
// library image on every device that loads it; its device address is looked up once per device.
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kMaxDevices];

sa_status noalloc_scratch(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_sa_noalloc_scores) != cudaSuccess || !p) {
            cudaGetLastError();
            return SA_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return SA_OK;
}

// ---- TMA descriptor encoding through the driver entry point (no link-time libcuda)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::mutex g_enc_mu;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encoder() {
    std::lock_guard<std::mutex> lk(g_enc_mu);
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        else
            cudaGetLastError();
    }
    return g_encode;
}

// [rows][cols] bf16 matrix with (box_cols x box_rows) boxes and the 128-byte swizzle
// (box_cols * 2 bytes must be 128).
bool encode_bf16_2d(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, uint32_t box_cols,
                    uint32_t box_rows) {
    EncodeTiledFn enc = encoder();
    if (!enc || rows < 1 || cols < 1) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows][64] matrix of bf16 or f32 read in boxes of 128 bytes x box_rows (128-byte swizzle).
bool encode_rows_e(CUtensorMap* m, const void* base, int64_t rows, bool bf16, uint32_t box_rows) {
    EncodeTiledFn enc = encoder();
    if (!enc || rows < 1) return false;
    const cuuint64_t elem = bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {64, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {64 * elem};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / elem), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows][64] bf16 matrix read in 128-row boxes (Q, K, sink keys, landmark keys).
bool encode_rows_bf16(CUtensorMap* m, const void* base, int64_t rows) {
    return encode_bf16_2d(m, base, 64, rows, 64, 128);
}

// Transposed V tiles: [tiles * 64][128] bf16 read as two 64 x 64 boxes per tile.
bool encode_vt_tiles(CUtensorMap* m, const void* base, int64_t tiles) {
    return encode_bf16_2d(m, base, 128, tiles * 64, 64, 64);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of the tensor-core attention call (all offsets 256-byte aligned):
//   vt   transposed V tiles of every key tile [bh][n_vtiles][64][128] bf16
//   svt  transposed V tiles of the sink segment [bh][n_sink_tiles][64][128]
//   lk   landmark key table [bh][ntp][64] bf16, lvt its transposed value tiles, lbias [ntp] f32
struct AttnWs {
    int64_t n_vtiles, n_sink_tiles, n_lm_chunks, ntp;
    size_t vt, svt, lk, lvt, lbias, total;
};
// Lk: key rows per head in dense mode (g.L, or the length of a compacted key sequence).
AttnWs attn_ws(const Geo& g, bool dense, bool landmark, int64_t Lk = -1) {
    AttnWs w;
    constexpr size_t kTile = 64 * 128 * 2;
    if (Lk < 0) Lk = g.L;
    w.ntp = (g.nt + 127) / 128 * 128;
    w.n_vtiles = dense ? (Lk + 127) / 128 : g.nt;
    w.n_sink_tiles = dense ? 0 : (g.S * g.n_sink + 127) / 128;
    w.n_lm_chunks = (!dense && landmark) ? w.ntp / 128 : 0;
    size_t off = 0;
    w.vt = off;
    off += align256((size_t)g.bh * w.n_vtiles * kTile);
    w.svt = off;
    off += align256((size_t)g.bh * w.n_sink_tiles * kTile);
    w.lk = off;
    off += (!dense && landmark) ? align256((size_t)g.bh * w.ntp * 64 * 2) : 0;
    w.lvt = off;
    off += align256((size_t)g.bh * w.n_lm_chunks * kTile);
    w.lbias = off;
    off += (!dense && landmark) ? align256((size_t)w.ntp * 4) : 0;
    w.total = off;
    return w;
}

bool use_tc(const Geo& g) { return g.bf16 && g.T == 128 && g.d == 64; }

// The 64-key tensor-core kernel (k_attn_tcg.cuh) takes every other supported shape: f32 with
// tile 64 or 128, bf16 with tile 64.
//   vt   transposed V items [bh][n_vt][64][64] E, n_vt = nt * tile / 64 (dense: ceil(Lk / 64))
//   svt  transposed sink V items [bh][n_sink_items][64][64] E
//   lk   landmark keys [bh][ntp][64] E, lvt their transposed values [bh][ntp/64][64][64] E,
//   lbias [ntp] f32 (ntp = nt rounded up to 64)
//   f32 only: Q, K and the sink keys rounded to tf32 (q32 [bh][L][64], k32 [bh][Lk][64],
//   sk32 [bh][S*n_sink][64])
struct TcgWs {
    int64_t sub, n_vt, n_sink_items, n_lm_items, ntp, elem;
    size_t vt, svt, lk, lvt, lbias, q32, k32, sk32, total;
};
TcgWs tcg_ws(const Geo& g, bool dense, bool landmark, int64_t Lk = -1) {
    TcgWs w;
    if (Lk < 0) Lk = g.L;
    w.elem = g.bf16 ? 2 : 4;
    w.sub = g.T / 64;
    w.ntp = (g.nt + 63) / 64 * 64;
    w.n_vt = dense ? (Lk + 63) / 64 : g.nt * w.sub;
    w.n_sink_items = dense ? 0 : (g.S * g.n_sink + 63) / 64;
    w.n_lm_items = (!dense && landmark) ? w.ntp / 64 : 0;
    const size_t item = (size_t)64 * 64 * w.elem;
    size_t off = 0;
    w.vt = off;
    off += align256((size_t)g.bh * w.n_vt * item);
    w.svt = off;
    off += align256((size_t)g.bh * w.n_sink_items * item);
    w.lk = off;
    off += w.n_lm_items ? align256((size_t)g.bh * w.ntp * 64 * w.elem) : 0;
    w.lvt = off;
    off += align256((size_t)g.bh * w.n_lm_items * item);
    w.lbias = off;
    off += w.n_lm_items ? align256((size_t)w.ntp * 4) : 0;
    const bool f32 = !g.bf16;
    w.q32 = off;
    off += f32 ? align256((size_t)g.bh * g.L * 64 * 4) : 0;
    w.k32 = off;
    off += f32 ? align256((size_t)g.bh * Lk * 64 * 4) : 0;
    w.sk32 = off;
    off += (f32 && !dense) ? align256((size_t)g.bh * g.S * g.n_sink * 64 * 4) : 0;
    w.total = off;
    return w;
}

size_t select_rows_per_block(const Geo& g) {
    // one block of score rows stays in L2 (about 48 MB), at least 64 rows
    int64_t r = (48ll << 20) / (g.nt * 4);
    r = std::max<int64_t>(64, r / 64 * 64);
    return (size_t)std::min<int64_t>(r, g.nt);
}

sa_status attn_common(const Geo& g, const void* q, const void* k, const void* v, const int32_t* kept_idx,
                      const int32_t* kept_cnt, int32_t max_kept, const void* sink_k, const void* sink_v,
                      int32_t landmark, const float* k_pool, const float* v_pool, const int32_t* k_cnt,
                      void* ws, size_t ws_bytes, void* o, float* lse, bool dense, cudaStream_t stream,
                      int64_t Lk = -1) {
    sa_status st = ensure_attributes();
    if (st != SA_OK) return st;
    if (Lk < 0) Lk = g.L;
    if (use_tc(g)) {
        TcArgs a;
        memset(&a, 0, sizeof(a));
        const AttnWs w = attn_ws(g, dense, landmark != 0, Lk);
        if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
        uint8_t* base = static_cast<uint8_t*>(ws);
        const int64_t n_sink_rows = g.S * g.n_sink;
        bool ok = encode_rows_bf16(&a.tm_q, q, g.bh * g.L) && encode_rows_bf16(&a.tm_k, k, g.bh * Lk) &&
                  encode_vt_tiles(&a.tm_vt, base + w.vt, g.bh * w.n_vtiles);
        if (w.n_sink_tiles > 0)
            ok = ok && encode_rows_bf16(&a.tm_sk, sink_k, g.bh * n_sink_rows) &&
                 encode_vt_tiles(&a.tm_svt, base + w.svt, g.bh * w.n_sink_tiles);
        else
            a.tm_sk = a.tm_k, a.tm_svt = a.tm_vt;
        if (w.n_lm_chunks > 0) {
            ok = ok && encode_rows_bf16(&a.tm_lk, base + w.lk, g.bh * w.ntp) &&
                 encode_vt_tiles(&a.tm_lvt, base + w.lvt, g.bh * w.n_lm_chunks);
            a.lbias2 = reinterpret_cast<const float*>(base + w.lbias);
        } else {
            a.tm_lk = a.tm_k, a.tm_lvt = a.tm_vt;
        }
        if (!ok) return SA_ERR_CUDA;
        // operand preparation: transposed V tiles (and the landmark tables)
        {
            VtArgs t;
            t.src = static_cast<const __nv_bfloat16*>(v);
            t.dst = reinterpret_cast<__nv_bfloat16*>(base + w.vt);
            t.tiles_per_head = (int32_t)w.n_vtiles;
            t.frame_mode = dense ? 0 : 1;
            t.tokens = (int32_t)g.N;
            t.tpf = (int32_t)g.tpf;
            t.L = (int32_t)g.L;
            t.rows_per_head = (int32_t)Lk;
            if (w.n_vtiles > 2147483647 || g.bh > 65535) return SA_ERR_UNSUPPORTED;
            vtile_transpose_kernel<<<dim3((unsigned)w.n_vtiles, (unsigned)g.bh), 256, 0, stream>>>(t);
            if ((st = launch_status()) != SA_OK) return st;
            if (w.n_sink_tiles > 0) {
                t.src = static_cast<const __nv_bfloat16*>(sink_v);
                t.dst = reinterpret_cast<__nv_bfloat16*>(base + w.svt);
                t.tiles_per_head = (int32_t)w.n_sink_tiles;
                t.frame_mode = 0;
                t.rows_per_head = (int32_t)n_sink_rows;
                vtile_transpose_kernel<<<dim3((unsigned)w.n_sink_tiles, (unsigned)g.bh), 256, 0, stream>>>(t);
                if ((st = launch_status()) != SA_OK) return st;
            }
        }
        if (w.n_lm_chunks > 0) {
            const int64_t n4 = g.bh * w.ntp * 16;
            const int blocks = (int)std::min<int64_t>((n4 + 255) / 256, 148 * 32);
            landmark_prep_kernel<<<blocks, 256, 0, stream>>>(
                k_pool, v_pool, k_cnt, reinterpret_cast<__nv_bfloat16*>(base + w.lk),
                reinterpret_cast<__nv_bfloat16*>(base + w.lvt), reinterpret_cast<float*>(base + w.lbias),
                (int32_t)g.bh, (int32_t)g.nt, (int32_t)w.ntp);
            if ((st = launch_status()) != SA_OK) return st;
        }
        a.kept_idx = kept_idx;
        a.kept_cnt = kept_cnt;
        a.o = static_cast<__nv_bfloat16*>(o);
        a.lse = lse;
        a.max_kept = max_kept;
        a.frames = (int32_t)g.S;
        a.tokens = (int32_t)g.N;
        a.n_sink = (int32_t)g.n_sink;
        a.tpf = (int32_t)g.tpf;
        a.nt = (int32_t)g.nt;
        a.L = (int32_t)g.L;
        a.Lk = (int32_t)Lk;
        a.ntp = (int32_t)w.ntp;
        a.n_vtiles = (int32_t)w.n_vtiles;
        a.n_sink_rows = (int32_t)n_sink_rows;
        a.n_sink_tiles = (int32_t)w.n_sink_tiles;
        a.n_lm_chunks = (int32_t)w.n_lm_chunks;
        a.dense = dense ? 1 : 0;
        a.landmark = w.n_lm_chunks > 0 ? 1 : 0;
        a.q_per_head = dense ? (int32_t)((g.L + 127) / 128) : (int32_t)g.nt;
        a.total_items = (int32_t)(g.bh * a.q_per_head);
        a.scale_log2 = (float)((double)g.scale * 1.4426950408889634);
        using Lay = TcLayout<kTcSlots, kTcStages, true>;
        using LayD = TcLayout<kTcSlots, kTcStagesDense, false>;
        {
            int dev = 0;
            if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
            if (!g_tc_regs_ok[dev]) return SA_ERR_UNSUPPORTED;
        }
        // exact division by tpf with a multiply-high (tpf > 1; one tile per frame needs none),
        // checked for every tile index; the dense modes never divide
        a.tpf_magic = 0;
        if (!dense && g.tpf > 1) {
            a.tpf_magic = (uint32_t)((0x100000000ull + (uint64_t)g.tpf - 1) / (uint64_t)g.tpf);
            for (int64_t j = 0; j < g.nt; ++j)
                if ((int64_t)(((uint64_t)j * a.tpf_magic) >> 32) != j / g.tpf) return SA_ERR_UNSUPPORTED;
        }
        const size_t smem = dense ? LayD::smem_bytes() : Lay::smem_bytes();
        if (smem > 227 * 1024) return SA_ERR_UNSUPPORTED;
        const int grid = (a.total_items + kTcSlots - 1) / kTcSlots;
        if (dense)
            attn_tc_kernel<kTcSlots, kTcStagesDense, false, false><<<grid, Lay::kThreads, smem, stream>>>(a);
        else if (a.landmark)
            attn_tc_kernel<kTcSlots, kTcStages, true, true><<<grid, Lay::kThreads, smem, stream>>>(a);
        else
            attn_tc_kernel<kTcSlots, kTcStages, false, true><<<grid, Lay::kThreads, smem, stream>>>(a);
        return launch_status();
    }
    {
        // 64-key tensor-core kernel: f32 (tf32 products) or bf16 with tile 64
        const TcgWs w = tcg_ws(g, dense, landmark != 0, Lk);
        if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
        uint8_t* base = static_cast<uint8_t*>(ws);
        TcgArgs a;
        memset(&a, 0, sizeof(a));
        const int64_t n_sink_rows = g.S * g.n_sink;
        if (!g.bf16) {  // f32: the product operands rounded to tf32 once per call
            auto round = [&](const void* src, size_t off, int64_t n) {
                const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
                round_tf32_kernel<<<std::max(1, blocks), 256, 0, stream>>>(static_cast<const float*>(src),
                                                                           reinterpret_cast<float*>(base + off), n);
            };
            round(q, w.q32, g.bh * g.L * 64);
            round(k, w.k32, g.bh * Lk * 64);
            if (!dense && n_sink_rows > 0) round(sink_k, w.sk32, g.bh * n_sink_rows * 64);
            if ((st = launch_status()) != SA_OK) return st;
            q = base + w.q32;
            k = base + w.k32;
            if (!dense && n_sink_rows > 0) sink_k = base + w.sk32;
        }
        bool ok = encode_rows_e(&a.tm_q, q, g.bh * g.L, g.bf16, 128) && encode_rows_e(&a.tm_k, k, g.bh * Lk, g.bf16, 64) &&
                  encode_rows_e(&a.tm_vt, base + w.vt, g.bh * w.n_vt * 64, g.bf16, 64);
        if (w.n_sink_items > 0)
            ok = ok && encode_rows_e(&a.tm_sk, sink_k, g.bh * n_sink_rows, g.bf16, 64) &&
                 encode_rows_e(&a.tm_svt, base + w.svt, g.bh * w.n_sink_items * 64, g.bf16, 64);
        else
            a.tm_sk = a.tm_k, a.tm_svt = a.tm_vt;
        if (w.n_lm_items > 0) {
            ok = ok && encode_rows_e(&a.tm_lk, base + w.lk, g.bh * w.ntp, g.bf16, 64) &&
                 encode_rows_e(&a.tm_lvt, base + w.lvt, g.bh * w.n_lm_items * 64, g.bf16, 64);
            a.lbias2 = reinterpret_cast<const float*>(base + w.lbias);
        } else {
            a.tm_lk = a.tm_k, a.tm_lvt = a.tm_vt;
        }
        if (!ok) return SA_ERR_CUDA;
        if (w.n_vt > 2147483647 || g.bh > 65535) return SA_ERR_UNSUPPORTED;
        Vt64Args t;
        t.src = v;
        t.dst = base + w.vt;
        t.items_per_head = (int32_t)w.n_vt;
        t.frame_mode = dense ? 0 : 1;
        t.tokens = (int32_t)g.N;
        t.tpf = (int32_t)g.tpf;
        t.tile = (int32_t)g.T;
        t.sub = (int32_t)w.sub;
        t.L = (int32_t)g.L;
        t.rows_per_head = (int32_t)Lk;
        auto vt_launch = [&](const Vt64Args& x, int64_t items) {
            if (g.bf16)
                vtile64_transpose_kernel<__nv_bfloat16><<<dim3((unsigned)items, (unsigned)g.bh), 256, 0, stream>>>(x);
            else
                vtile64_transpose_kernel<float><<<dim3((unsigned)items, (unsigned)g.bh), 256, 0, stream>>>(x);
        };
        vt_launch(t, w.n_vt);
        if ((st = launch_status()) != SA_OK) return st;
        if (w.n_sink_items > 0) {
            t.src = sink_v;
            t.dst = base + w.svt;
            t.items_per_head = (int32_t)w.n_sink_items;
            t.frame_mode = 0;
            t.rows_per_head = (int32_t)n_sink_rows;
            vt_launch(t, w.n_sink_items);
            if ((st = launch_status()) != SA_OK) return st;
        }
        if (w.n_lm_items > 0) {
            const int64_t n1 = g.bh * w.ntp * 64;
            const int blocks = (int)std::min<int64_t>((n1 + 255) / 256, 148 * 32);
            if (g.bf16)
                landmark64_prep_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
                    k_pool, v_pool, k_cnt, reinterpret_cast<__nv_bfloat16*>(base + w.lk),
                    reinterpret_cast<__nv_bfloat16*>(base + w.lvt), reinterpret_cast<float*>(base + w.lbias),
                    (int32_t)g.bh, (int32_t)g.nt, (int32_t)w.ntp);
            else
                landmark64_prep_kernel<float><<<blocks, 256, 0, stream>>>(
                    k_pool, v_pool, k_cnt, reinterpret_cast<float*>(base + w.lk), reinterpret_cast<float*>(base + w.lvt),
                    reinterpret_cast<float*>(base + w.lbias), (int32_t)g.bh, (int32_t)g.nt, (int32_t)w.ntp);
            if ((st = launch_status()) != SA_OK) return st;
        }
        a.kept_idx = kept_idx;
        a.kept_cnt = kept_cnt;
        a.o = o;
        a.lse = lse;
        a.max_kept = max_kept;
        a.frames = (int32_t)g.S;
        a.tokens = (int32_t)g.N;
        a.tile = (int32_t)g.T;
        a.n_sink = (int32_t)g.n_sink;
        a.tpf = (int32_t)g.tpf;
        a.nt = (int32_t)g.nt;
        a.L = (int32_t)g.L;
        a.ntp = (int32_t)w.ntp;
        a.sub = (int32_t)w.sub;
        a.n_vt = (int32_t)w.n_vt;
        a.n_sink_rows = (int32_t)n_sink_rows;
        a.n_sink_items = (int32_t)w.n_sink_items;
        a.n_lm_items = (int32_t)w.n_lm_items;
        a.dense = dense ? 1 : 0;
        a.landmark = w.n_lm_items > 0 ? 1 : 0;
        a.q_per_head = dense ? (int32_t)((g.L + g.T - 1) / g.T) : (int32_t)g.nt;
        a.total_items = (int32_t)(g.bh * a.q_per_head);
        a.scale_log2 = (float)((double)g.scale * 1.4426950408889634);
        if (dense && Lk != g.L) return SA_ERR_UNSUPPORTED;  // compacted keys: bf16 tile-128 only
        const int grid = (a.total_items + 1) / 2;
        if (g.bf16) {
            using C = tcg::Cfg<false>;
            attn_tcg_kernel<false><<<grid, C::kThreads, C::smem_bytes(), stream>>>(a);
        } else {
            using C = tcg::Cfg<true>;
            attn_tcg_kernel<true><<<grid, C::kThreads, C::smem_bytes(), stream>>>(a);
        }
        return launch_status();
    }
}

}  // namespace

extern "C" {

int32_t sa_num_tiles(const sa_shape* shape) {
    Geo g;
    if (geo_of(shape, &g) == SA_ERR_INVALID_ARG) return -1;
    return (int32_t)g.nt;
}

int32_t sa_max_kept(const sa_shape* shape, int32_t k) {
    Geo g;
    if (k < 0 || geo_of(shape, &g) == SA_ERR_INVALID_ARG) return -1;
    return (int32_t)max_kept_of(g, k);
}

const char* sa_status_string(sa_status s) {
    switch (s) {
        case SA_OK: return "ok";
        case SA_ERR_INVALID_ARG: return "invalid argument";
        case SA_ERR_UNSUPPORTED: return "unsupported shape or type";
        case SA_ERR_CUDA: return "CUDA error";
        case SA_ERR_TIMEOUT: return "device wait timed out";
        case SA_ERR_BAD_LIST: return "kept list entry out of range";
        case SA_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

sa_status sa_check_device_error(sa_stream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    int code = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&code, g_sa_error, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_sa_error, &zero, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    return (sa_status)code;
}

sa_status sa_set_wait_limit_ns(int64_t limit_ns) {
    if (limit_ns <= 0) return SA_ERR_INVALID_ARG;
    const unsigned long long v = (unsigned long long)limit_ns;
    if (cudaMemcpyToSymbol(g_sa_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    return SA_OK;
}

sa_status sa_test_withhold_query_load(int32_t enable) {
    const int v = enable ? 1 : 0;
    if (cudaMemcpyToSymbol(g_sa_test_withhold, &v, sizeof(v)) != cudaSuccess) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    return SA_OK;
}

sa_status sa_tile_pool(const sa_shape* shape, const void* q, const void* k, const void* v_or_null,
                       float* q_pool, float* k_pool, float* v_pool_or_null, int32_t* k_cnt, void* sink_k_or_null,
                       void* sink_v_or_null, sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    if (!q || !k || !q_pool || !k_pool || !k_cnt) return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_pool) || !aligned16(k_pool) || !aligned16(k_cnt))
        return SA_ERR_INVALID_ARG;
    const bool with_v = v_or_null && v_pool_or_null;
    if ((v_or_null && !aligned16(v_or_null)) || (v_pool_or_null && !aligned16(v_pool_or_null)))
        return SA_ERR_INVALID_ARG;
    if (g.n_sink > 0) {
        if (!sink_k_or_null || !aligned16(sink_k_or_null)) return SA_ERR_INVALID_ARG;
        if (v_or_null && (!sink_v_or_null || !aligned16(sink_v_or_null))) return SA_ERR_INVALID_ARG;
    }
    PoolArgs a;
    a.q = q;
    a.k = k;
    a.v = v_or_null;
    a.q_pool = q_pool;
    a.k_pool = k_pool;
    a.v_pool = with_v ? v_pool_or_null : nullptr;
    a.k_cnt = k_cnt;
    a.sink_k = g.n_sink > 0 ? sink_k_or_null : nullptr;
    a.sink_v = (g.n_sink > 0 && v_or_null) ? sink_v_or_null : nullptr;
    a.bh = (int32_t)g.bh;
    a.frames = (int32_t)g.S;
    a.tokens = (int32_t)g.N;
    a.tile = (int32_t)g.T;
    a.n_sink = (int32_t)g.n_sink;
    a.tpf = (int32_t)g.tpf;
    a.nt = (int32_t)g.nt;
    const int64_t warps = g.bh * g.nt;
    const int64_t blocks = (warps + 7) / 8;
    if (blocks >= (int64_t(1) << 31) || g.bh > 65535 || g.nt >= (int64_t(1) << 31)) return SA_ERR_UNSUPPORTED;
    if (g.bf16)
        pool_tiles_bf16_kernel<<<dim3((unsigned)g.nt, (unsigned)g.bh), 128, 0, stream>>>(a);
    else
        pool_tiles_f32_kernel<<<(unsigned)blocks, 256, 0, stream>>>(a);
    return launch_status();
}

// Step 2 on the tensor cores (k_scores_tc.cuh): the pooled tables' tensor maps are encoded once
// per call; each launch then covers rows [i0, i0 + rows) of heads h0 .. h0 + gz - 1.
struct ScoreTcLaunch {
    ScoreTcArgs a;
    int32_t sms;  // SMs of the current device
};

static bool score_tc_prepare(ScoreTcLaunch* L, const Geo& g, const float* q_pool, const float* k_pool, float* out,
                             int64_t ldo) {
    memset(&L->a, 0, sizeof(L->a));
    int dev = 0;  // ensure_attributes() has run: the SM count is known
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices || g_sm_count[dev] < 1) return false;
    L->sms = g_sm_count[dev];
    if (!encode_rows_e(&L->a.tm_q, q_pool, g.bh * g.nt, false, 128) ||
        !encode_rows_e(&L->a.tm_k, k_pool, g.bh * g.nt, false, 128))
        return false;
    L->a.out = out;
    L->a.ldo = ldo;
    L->a.nt = (int32_t)g.nt;
    L->a.n_chunks = (int32_t)((g.nt + 127) / 128);
    L->a.vec_out = (ldo % 4 == 0 && aligned16(out)) ? 1 : 0;
    return true;
}

static sa_status score_tc_launch(ScoreTcLaunch* L, int64_t h0, int64_t i0, int64_t rows, int64_t gz,
                                 cudaStream_t stream) {
    ScoreTcArgs& a = L->a;
    a.h0 = (int32_t)h0;
    a.i0 = (int32_t)i0;
    a.rows = (int32_t)rows;
    const int64_t gy = (rows + 127) / 128;
    if (gy > 65535 || gz > 65535 || gy < 1 || gz < 1) return SA_ERR_UNSUPPORTED;
    // One CTA per SM at a time (211 KB of shared memory): with fewer row tiles than SMs the chunks
    // of a row tile are split so that the grid is one wave of at most one CTA per SM; otherwise
    // every CTA takes whole row tiles.
    const int64_t sms = L->sms;
    const int64_t tiles = gy * gz;
    const int64_t per_tile = tiles >= sms ? 1 : sms / tiles;
    a.chunks_per_cta = (int32_t)((a.n_chunks + per_tile - 1) / per_tile);
    const int64_t gx = (a.n_chunks + a.chunks_per_cta - 1) / a.chunks_per_cta;
    score_tc_kernel<<<dim3((unsigned)gx, (unsigned)gy, (unsigned)gz), 384, stc::kSmemBytes, stream>>>(a);
    return launch_status();
}

sa_status sa_tile_scores(const sa_shape* shape, const float* q_pool, const float* k_pool, float* scores,
                         sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    if (!q_pool || !k_pool || !scores || !aligned16(q_pool) || !aligned16(k_pool) || !aligned16(scores))
        return SA_ERR_INVALID_ARG;
    if (g.bh > 65535) return SA_ERR_UNSUPPORTED;
    if ((st = ensure_attributes()) != SA_OK) return st;
    ScoreTcLaunch L;
    if (!score_tc_prepare(&L, g, q_pool, k_pool, scores, g.nt)) return SA_ERR_CUDA;
    return score_tc_launch(&L, 0, 0, g.nt, g.bh, stream);
}

size_t sa_select_workspace_size(const sa_shape* shape, int32_t streamed) {
    Geo g;
    if (geo_of(shape, &g) != SA_OK) return 0;
    if (!streamed) return 0;
    return select_rows_per_block(g) * (size_t)g.nt * 4;
}

// Short rows: one warp per row, as many rows per CTA as fit in shared memory; long rows:
// one 256-thread CTA per row.
static void launch_select(const SelectArgs& a, unsigned gy, cudaStream_t stream) {
    if (a.nt <= SEL_WARP_MAX_NT) {
        const int w = select_warps(a.nt);
        const unsigned gx = (unsigned)((a.rows + w - 1) / w);
        select_topk_warp_kernel<<<dim3(gx, gy), 32 * w, select_smem_bytes(a.nt), stream>>>(a);
    } else {
        select_topk_block_kernel<<<dim3((unsigned)a.rows, gy), SEL_BLOCK_THREADS, select_block_smem_bytes(a.nt),
                                   stream>>>(a);
    }
}

// Shared by sa_select_topk (k_head == nullptr: every head keeps k) and
// sa_select_topk_per_head (head h keeps k_head[h] <= k).
static sa_status select_impl(const sa_shape* shape, const float* scores_or_null, const float* q_pool,
                             const float* k_pool, int32_t k, const int32_t* k_head, int32_t* kept_idx,
                             int32_t* kept_cnt, int32_t max_kept, void* workspace_or_null, size_t workspace_bytes,
                             sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    if (k < 0 || !kept_idx || !kept_cnt || !aligned16(kept_idx) || !aligned16(kept_cnt)) return SA_ERR_INVALID_ARG;
    if (max_kept < max_kept_of(g, k)) return SA_ERR_INVALID_ARG;
    if (g.nt > SEL_MAX_NT) return SA_ERR_UNSUPPORTED;
    if (scores_or_null) {
        if (!aligned16(scores_or_null)) return SA_ERR_INVALID_ARG;
        if (g.bh > 65535) return SA_ERR_UNSUPPORTED;
    } else {
        if (!q_pool || !k_pool || !aligned16(q_pool) || !aligned16(k_pool)) return SA_ERR_INVALID_ARG;
        const size_t need = sa_select_workspace_size(shape, 1);
        if (!workspace_or_null || workspace_bytes < need || !aligned16(workspace_or_null)) return SA_ERR_WORKSPACE;
    }
    if ((st = ensure_attributes()) != SA_OK) return st;
    SelectArgs a;
    a.kept_idx = kept_idx;
    a.kept_cnt = kept_cnt;
    a.nt = (int32_t)g.nt;
    a.tpf = (int32_t)g.tpf;
    a.tile = (int32_t)g.T;
    a.tokens = (int32_t)g.N;
    a.n_sink = (int32_t)g.n_sink;
    a.k = k;
    a.max_kept = max_kept;
    a.k_head = k_head;
    a.k_max = k;
    if (scores_or_null) {
        a.scores = scores_or_null;
        a.lds = g.nt;
        a.h0 = 0;
        a.i0 = 0;
        a.rows = (int32_t)g.nt;
        launch_select(a, (unsigned)g.bh, stream);
        return launch_status();
    }
    // streamed: score one L2-resident block of rows at a time, then select from it (a single
    // persistent launch that takes score tiles and row selections from one work counter was
    // measured slower: 23.9 ms against 17.9 ms at 1024 frames)
    const int64_t R = (int64_t)select_rows_per_block(g);
    float* blk = static_cast<float*>(workspace_or_null);
    ScoreTcLaunch L;
    if (!score_tc_prepare(&L, g, q_pool, k_pool, blk, g.nt)) return SA_ERR_CUDA;
    for (int64_t h = 0; h < g.bh; ++h) {
        for (int64_t i0 = 0; i0 < g.nt; i0 += R) {
            const int64_t rows = std::min<int64_t>(R, g.nt - i0);
            if ((st = score_tc_launch(&L, h, i0, rows, 1, stream)) != SA_OK) return st;
            a.scores = blk;
            a.lds = g.nt;
            a.h0 = (int32_t)h;
            a.i0 = (int32_t)i0;
            a.rows = (int32_t)rows;
            launch_select(a, 1u, stream);
            if ((st = launch_status()) != SA_OK) return st;
        }
    }
    return SA_OK;
}

sa_status sa_select_topk(const sa_shape* shape, const float* scores_or_null, const float* q_pool,
                         const float* k_pool, int32_t k, int32_t* kept_idx, int32_t* kept_cnt, int32_t max_kept,
                         void* workspace_or_null, size_t workspace_bytes, sa_stream_t stream) {
    return select_impl(shape, scores_or_null, q_pool, k_pool, k, nullptr, kept_idx, kept_cnt, max_kept,
                       workspace_or_null, workspace_bytes, stream);
}

sa_status sa_select_topk_per_head(const sa_shape* shape, const float* scores_or_null, const float* q_pool,
                                  const float* k_pool, const int32_t* k_per_head, int32_t k_max, int32_t* kept_idx,
                                  int32_t* kept_cnt, int32_t max_kept, void* workspace_or_null,
                                  size_t workspace_bytes, sa_stream_t stream) {
    if (!k_per_head || (reinterpret_cast<uintptr_t>(k_per_head) & 3u) || k_max < 0) return SA_ERR_INVALID_ARG;
    return select_impl(shape, scores_or_null, q_pool, k_pool, k_max, k_per_head, kept_idx, kept_cnt, max_kept,
                       workspace_or_null, workspace_bytes, stream);
}

sa_status sa_select_topk_noalloc(const sa_shape* shape, const float* q_pool, const float* k_pool, int32_t k,
                                 int32_t* kept_idx, int32_t* kept_cnt, int32_t max_kept, sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    if (k < 0 || !kept_idx || !kept_cnt || !aligned16(kept_idx) || !aligned16(kept_cnt)) return SA_ERR_INVALID_ARG;
    if (!q_pool || !k_pool || !aligned16(q_pool) || !aligned16(k_pool)) return SA_ERR_INVALID_ARG;
    if (max_kept < max_kept_of(g, k)) return SA_ERR_INVALID_ARG;
    // the fixed scratch must hold at least 64 whole score rows
    if (g.nt > SEL_MAX_NT || g.nt * 64 > kNoallocScratchFloats) return SA_ERR_UNSUPPORTED;
    if ((st = ensure_attributes()) != SA_OK) return st;
    float* blk = nullptr;
    if ((st = noalloc_scratch(&blk)) != SA_OK) return st;
    const int64_t R = std::min<int64_t>(g.nt, (kNoallocScratchFloats / g.nt) / 64 * 64);
    SelectArgs a;
    a.kept_idx = kept_idx;
    a.kept_cnt = kept_cnt;
    a.nt = (int32_t)g.nt;
    a.tpf = (int32_t)g.tpf;
    a.tile = (int32_t)g.T;
    a.tokens = (int32_t)g.N;
    a.n_sink = (int32_t)g.n_sink;
    a.k = k;
    a.max_kept = max_kept;
    a.k_head = nullptr;
    a.k_max = k;
    ScoreTcLaunch L;
    if (!score_tc_prepare(&L, g, q_pool, k_pool, blk, g.nt)) return SA_ERR_CUDA;
    for (int64_t h = 0; h < g.bh; ++h) {
        for (int64_t i0 = 0; i0 < g.nt; i0 += R) {
            const int64_t rows = std::min<int64_t>(R, g.nt - i0);
            if ((st = score_tc_launch(&L, h, i0, rows, 1, stream)) != SA_OK) return st;
            a.scores = blk;
            a.lds = g.nt;
            a.h0 = (int32_t)h;
            a.i0 = (int32_t)i0;
            a.rows = (int32_t)rows;
            launch_select(a, 1u, stream);
            if ((st = launch_status()) != SA_OK) return st;
        }
    }
    return SA_OK;
}

size_t sa_head_budget_workspace_size(const sa_shape* shape) {
    Geo g;
    if (geo_of(shape, &g) != SA_OK) return 0;
    return (size_t)g.bh * (size_t)g.nt * 4;
}

sa_status sa_head_budgets(const sa_shape* shape, const float* q_pool, const float* k_pool, float temperature,
                          float beta, int32_t k_lo, int32_t k_hi, int32_t* k_per_head, float* perplexity_or_null,
                          void* workspace, size_t workspace_bytes, sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    if (!q_pool || !k_pool || !aligned16(q_pool) || !aligned16(k_pool)) return SA_ERR_INVALID_ARG;
    if (!k_per_head || (reinterpret_cast<uintptr_t>(k_per_head) & 3u)) return SA_ERR_INVALID_ARG;
    if (perplexity_or_null && (reinterpret_cast<uintptr_t>(perplexity_or_null) & 3u)) return SA_ERR_INVALID_ARG;
    if (!(temperature > 0.0f) || isinf(temperature) || !(beta >= 0.0f) || isinf(beta)) return SA_ERR_INVALID_ARG;
    if (k_lo < 0 || k_hi < k_lo) return SA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < sa_head_budget_workspace_size(shape) || !aligned16(workspace))
        return SA_ERR_WORKSPACE;
    if (g.bh > 65535 || (g.nt + 127) / 128 > 2147483647ll) return SA_ERR_UNSUPPORTED;
    if ((st = ensure_attributes()) != SA_OK) return st;
    BudgetArgs a;
    a.q_pool = q_pool;
    a.k_pool = k_pool;
    a.row_perp = static_cast<float*>(workspace);
    a.k_per_head = k_per_head;
    a.perp_out = perplexity_or_null;
    a.nt = (int32_t)g.nt;
    a.tpf = (int32_t)g.tpf;
    a.tile = (int32_t)g.T;
    a.tokens = (int32_t)g.N;
    a.n_sink = (int32_t)g.n_sink;
    a.temperature = temperature;
    a.beta = beta;
    a.k_lo = k_lo;
    a.k_hi = k_hi;
    head_stat_kernel<<<dim3((unsigned)((g.nt + 127) / 128), (unsigned)g.bh), 256, BUDGET_SMEM, stream>>>(a);
    if ((st = launch_status()) != SA_OK) return st;
    head_budget_kernel<<<(unsigned)g.bh, 256, 0, stream>>>(a);
    return launch_status();
}

size_t sa_sparse_attn_workspace_size(const sa_shape* shape, int32_t landmark) {
    Geo g;
    if (geo_of(shape, &g) != SA_OK) return 0;
    if (!use_tc(g)) return tcg_ws(g, false, landmark != 0).total;
    return attn_ws(g, false, landmark != 0).total;
}

size_t sa_dense_attn_workspace_size(const sa_shape* shape) {
    Geo g;
    if (geo_of(shape, &g) != SA_OK) return 0;
    if (!use_tc(g)) return tcg_ws(g, true, false).total;
    return attn_ws(g, true, false).total;
}

sa_status sa_sparse_attn_fwd(const sa_shape* shape, const void* q, const void* k, const void* v,
                             const int32_t* kept_idx, const int32_t* kept_cnt, int32_t max_kept,
                             const void* sink_k_or_null, const void* sink_v_or_null, int32_t landmark,
                             const float* k_pool_or_null, const float* v_pool_or_null,
                             const int32_t* k_cnt_or_null, void* workspace_or_null, size_t workspace_bytes,
                             void* o, float* lse_or_null, sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    if (!q || !k || !v || !kept_idx || !kept_cnt || !o) return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kept_idx) || !aligned16(kept_cnt) ||
        !aligned16(o) || (lse_or_null && !aligned16(lse_or_null)))
        return SA_ERR_INVALID_ARG;
    if (max_kept < 1 || max_kept > g.nt) return SA_ERR_INVALID_ARG;
    if (g.n_sink > 0 && (!sink_k_or_null || !sink_v_or_null || !aligned16(sink_k_or_null) ||
                         !aligned16(sink_v_or_null)))
        return SA_ERR_INVALID_ARG;
    if (landmark) {
        if (!k_pool_or_null || !v_pool_or_null || !k_cnt_or_null || !aligned16(k_pool_or_null) ||
            !aligned16(v_pool_or_null) || !aligned16(k_cnt_or_null))
            return SA_ERR_INVALID_ARG;
    }
    const size_t need = sa_sparse_attn_workspace_size(shape, landmark);
    if (need && (!workspace_or_null || workspace_bytes < need || !aligned16(workspace_or_null)))
        return SA_ERR_WORKSPACE;
    return attn_common(g, q, k, v, kept_idx, kept_cnt, max_kept, sink_k_or_null, sink_v_or_null, landmark ? 1 : 0,
                       k_pool_or_null, v_pool_or_null, k_cnt_or_null, workspace_or_null, workspace_bytes, o,
                       lse_or_null, false, stream);
}

sa_status sa_dense_attn_fwd(const sa_shape* shape, const void* q, const void* k, const void* v,
                            void* workspace_or_null, size_t workspace_bytes, void* o, float* lse_or_null,
                            sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    if (!q || !k || !v || !o) return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse_or_null && !aligned16(lse_or_null)))
        return SA_ERR_INVALID_ARG;
    const size_t need = sa_dense_attn_workspace_size(shape);
    if (need && (!workspace_or_null || workspace_bytes < need || !aligned16(workspace_or_null)))
        return SA_ERR_WORKSPACE;
    return attn_common(g, q, k, v, nullptr, nullptr, 0, nullptr, nullptr, 0, nullptr, nullptr, nullptr,
                       workspace_or_null, workspace_bytes, o, lse_or_null, true, stream);
}

}  // extern "C"

// ------------------------------------------------------------------ subsampled global attention

struct SgaWs {
    SgaGeo sg;
    int64_t Lk, n_disc;
    size_t ksub, vsub, part, sums, lse, attn, attn_bytes, total;
};

static sa_status sga_plan(const Geo& g, int32_t grid_h, int32_t grid_w, int32_t s_h, int32_t s_w, SgaWs* w) {
    if (grid_h < 1 || grid_w < 1 || s_h < 1 || s_w < 1) return SA_ERR_INVALID_ARG;
    if ((int64_t)g.n_sink + (int64_t)grid_h * grid_w != g.N) return SA_ERR_INVALID_ARG;
    SgaGeo& sg = w->sg;
    sg.frames = (int32_t)g.S;
    sg.tokens = (int32_t)g.N;
    sg.n_special = (int32_t)g.n_sink;
    sg.grid_h = grid_h;
    sg.grid_w = grid_w;
    sg.s_h = s_h;
    sg.s_w = s_w;
    sg.kh = (grid_h + s_h - 1) / s_h;
    sg.kw = (grid_w + s_w - 1) / s_w;
    sg.kpf = sg.n_special + sg.kh * sg.kw;
    w->Lk = g.S * sg.kpf;
    w->n_disc = g.S * ((int64_t)grid_h * grid_w - (int64_t)sg.kh * sg.kw);
    size_t off = 0;
    w->ksub = off;
    off += align256((size_t)g.bh * w->Lk * 128);
    w->vsub = off;
    off += align256((size_t)g.bh * w->Lk * 128);
    w->part = off;
    off += align256((size_t)g.bh * g.S * SGA_SPLIT * 128 * 4);
    w->sums = off;
    off += align256((size_t)g.bh * 128 * 4);
    w->lse = off;
    off += align256((size_t)g.bh * g.L * 4);
    w->attn = off;
    w->attn_bytes = attn_ws(g, true, false, w->Lk).total;
    off += align256(w->attn_bytes);
    w->total = off;
    return SA_OK;
}

extern "C" {

size_t sa_sga_workspace_size(const sa_shape* shape, int32_t grid_h, int32_t grid_w, int32_t s_h, int32_t s_w) {
    Geo g;
    SgaWs w;
    if (geo_of(shape, &g) != SA_OK || !use_tc(g)) return 0;
    if (sga_plan(g, grid_h, grid_w, s_h, s_w, &w) != SA_OK) return 0;
    return w.total;
}

sa_status sa_sga_fwd(const sa_shape* shape, int32_t grid_h, int32_t grid_w, int32_t s_h, int32_t s_w, const void* q,
                     const void* k, const void* v, void* workspace, size_t workspace_bytes, void* o, float* lse_or_null,
                     sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    if (!q || !k || !v || !o) return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse_or_null && !aligned16(lse_or_null)))
        return SA_ERR_INVALID_ARG;
    SgaWs w;
    if ((st = sga_plan(g, grid_h, grid_w, s_h, s_w, &w)) != SA_OK) return st;
    if (!use_tc(g)) return SA_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return SA_ERR_WORKSPACE;
    if (g.bh > 65535 || g.S > 2147483647 || w.Lk > 2147483647 || g.bh * g.L > (1ll << 40)) return SA_ERR_UNSUPPORTED;
    if ((st = ensure_attributes()) != SA_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    SgaGatherArgs ga;
    ga.k = static_cast<const uint32_t*>(k);
    ga.v = static_cast<const uint32_t*>(v);
    ga.ksub = reinterpret_cast<uint32_t*>(base + w.ksub);
    ga.vsub = reinterpret_cast<uint32_t*>(base + w.vsub);
    ga.part = reinterpret_cast<float*>(base + w.part);
    ga.L = (int32_t)g.L;
    ga.Lk = (int32_t)w.Lk;
    ga.g = w.sg;
    sga_gather_kernel<<<dim3((unsigned)g.S, SGA_SPLIT, (unsigned)g.bh), 256, 0, stream>>>(ga);
    if ((st = launch_status()) != SA_OK) return st;
    float* sums = reinterpret_cast<float*>(base + w.sums);
    sga_sum_kernel<<<(unsigned)g.bh, 128, 0, stream>>>(ga.part, sums, (int32_t)(g.S * SGA_SPLIT));
    if ((st = launch_status()) != SA_OK) return st;
    float* lse_att = reinterpret_cast<float*>(base + w.lse);
    st = attn_common(g, q, ga.ksub, ga.vsub, nullptr, nullptr, 0, nullptr, nullptr, 0, nullptr, nullptr, nullptr,
                     base + w.attn, w.attn_bytes, o, lse_att, true, stream, w.Lk);
    if (st != SA_OK) return st;
    SgaCombineArgs ca;
    ca.q = static_cast<const uint32_t*>(q);
    ca.k = static_cast<const uint32_t*>(k);
    ca.v = static_cast<const uint32_t*>(v);
    ca.o = static_cast<uint32_t*>(o);
    ca.lse_in = lse_att;
    ca.lse_out = lse_or_null;
    ca.sums = sums;
    ca.rows = g.bh * g.L;
    ca.L = (int32_t)g.L;
    ca.n_disc = (int32_t)w.n_disc;
    ca.scale = g.scale;
    ca.g = w.sg;
    sga_combine_kernel<<<(unsigned)((ca.rows + 8 * SGA_ROWS_PER_WARP - 1) / (8 * SGA_ROWS_PER_WARP)), 256, 0,
                         stream>>>(ca);
    return launch_status();
}

}  // extern "C"

// ------------------------------------------------------------------ backward of the sparse attention

namespace {

// Workspace of the backward (offsets 256-byte aligned):
//   lse2t, dt   per query tile row: LSE in base 2 and rowsum(dO*O)      f32 [bh][nt][128] each
//   qt, dot, kt transposed tiles of Q, dO (query tiles) and K (key tiles) bf16 [bh][nt][64][128]
//   skt         transposed sink K tiles                                   bf16 [bh][n_sink_tiles][64][128]
//   lk, lv      landmark K / V rows, lkt transposed landmark K chunks,
//               lvt scratch of the landmark table writer, lbias [ntp]     (landmark mode)
//   bits        listed-tile bitmap of every query tile                    u32 [bh][nt][ntp/32] (landmark)
//   rev_cnt, fill, rev, units, n_units   reverse lists and the dK/dV work units
//   dk32, dv32  fp32 accumulators [bh][L][64]; dkbar, dvbar landmark gradients [bh][ntp][64]
struct BwdWs {
    int64_t ntp, n_sink_tiles, n_lm_chunks, words, units_cap;
    size_t lse2t, dt, qt, dot, kt, skt, lk, lv, lkt, lvt, lbias, bits, rev_cnt, fill, rev, units, n_units, dk32,
        dv32, dkbar, dvbar, total;
};

BwdWs bwd_ws(const Geo& g, int64_t max_kept, bool landmark) {
    BwdWs w;
    constexpr size_t kTile = 64 * 128 * 2;
    w.ntp = (g.nt + 127) / 128 * 128;
    w.n_sink_tiles = (g.S * g.n_sink + 127) / 128;
    w.n_lm_chunks = landmark ? w.ntp / 128 : 0;
    w.words = w.ntp / 32;
    const int64_t chunks_q = (g.nt + kBwdChunk - 1) / kBwdChunk;
    const int64_t M = g.bh * g.nt;
    w.units_cap = g.bh * (w.n_sink_tiles + w.n_lm_chunks) * chunks_q + (M * max_kept) / kBwdChunk + M + 1;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align256(bytes);
        return at;
    };
    w.lse2t = take((size_t)M * 128 * 4);
    w.dt = take((size_t)M * 128 * 4);
    w.qt = take((size_t)M * kTile);
    w.dot = take((size_t)M * kTile);
    w.kt = take((size_t)M * kTile);
    w.skt = take((size_t)g.bh * w.n_sink_tiles * kTile);
    w.lk = take(landmark ? (size_t)g.bh * w.ntp * 128 : 0);
    w.lv = take(landmark ? (size_t)g.bh * w.ntp * 128 : 0);
    w.lkt = take((size_t)g.bh * w.n_lm_chunks * kTile);
    w.lvt = take((size_t)g.bh * w.n_lm_chunks * kTile);
    w.lbias = take(landmark ? (size_t)w.ntp * 4 : 0);
    w.bits = take(landmark ? (size_t)M * w.words * 4 : 0);
    w.rev_cnt = take((size_t)M * 4);
    w.fill = take((size_t)M * 4);
    w.rev = take((size_t)M * max_kept * 4);
    w.units = take((size_t)w.units_cap * 16);
    w.n_units = take(16);
    w.dk32 = take((size_t)g.bh * g.L * 64 * 4);
    w.dv32 = take((size_t)g.bh * g.L * 64 * 4);
    w.dkbar = take(landmark ? (size_t)g.bh * w.ntp * 64 * 4 : 0);
    w.dvbar = take(landmark ? (size_t)g.bh * w.ntp * 64 * 4 : 0);
    w.total = off;
    return w;
}

sa_status transpose_tiles(const void* src, void* dst, int64_t tiles_per_head, bool frame_mode, const Geo& g,
                          int64_t rows_per_head, cudaStream_t stream) {
    if (tiles_per_head < 1) return SA_OK;
    VtArgs t;
    t.src = static_cast<const __nv_bfloat16*>(src);
    t.dst = static_cast<__nv_bfloat16*>(dst);
    t.tiles_per_head = (int32_t)tiles_per_head;
    t.frame_mode = frame_mode ? 1 : 0;
    t.tokens = (int32_t)g.N;
    t.tpf = (int32_t)g.tpf;
    t.L = (int32_t)g.L;
    t.rows_per_head = (int32_t)rows_per_head;
    vtile_transpose_kernel<<<dim3((unsigned)tiles_per_head, (unsigned)g.bh), 256, 0, stream>>>(t);
    return launch_status();
}

}  // namespace

extern "C" {

size_t sa_sparse_attn_bwd_workspace_size(const sa_shape* shape, int32_t max_kept, int32_t landmark) {
    Geo g;
    if (geo_of(shape, &g) != SA_OK || !use_tc(g)) return 0;
    if (max_kept < 1 || max_kept > g.nt) return 0;
    return bwd_ws(g, max_kept, landmark != 0).total;
}

sa_status sa_sparse_attn_bwd(const sa_shape* shape, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* d_o, const int32_t* kept_idx, const int32_t* kept_cnt,
                             int32_t max_kept, const void* sink_k_or_null, const void* sink_v_or_null,
                             int32_t landmark, const float* k_pool_or_null, const float* v_pool_or_null,
                             const int32_t* k_cnt_or_null, void* workspace, size_t workspace_bytes, void* dq, void* dk,
                             void* dv, sa_stream_t stream) {
    Geo g;
    sa_status st = geo_of(shape, &g);
    if (st != SA_OK) return st;
    const void* must[] = {q, k, v, o, lse, d_o, kept_idx, kept_cnt, dq, dk, dv};
    for (const void* p : must)
        if (!p || !aligned16(p)) return SA_ERR_INVALID_ARG;
    if (max_kept < 1 || max_kept > g.nt) return SA_ERR_INVALID_ARG;
    if (g.n_sink > 0 && (!sink_k_or_null || !sink_v_or_null || !aligned16(sink_k_or_null) ||
                         !aligned16(sink_v_or_null)))
        return SA_ERR_INVALID_ARG;
    if (landmark && (!k_pool_or_null || !v_pool_or_null || !k_cnt_or_null || !aligned16(k_pool_or_null) ||
                     !aligned16(v_pool_or_null) || !aligned16(k_cnt_or_null)))
        return SA_ERR_INVALID_ARG;
    if (!use_tc(g)) return SA_ERR_UNSUPPORTED;
    const bool lm = landmark != 0;
    const BwdWs w = bwd_ws(g, max_kept, lm);
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return SA_ERR_WORKSPACE;
    if (g.bh > 65535 || g.bh * g.nt * max_kept >= (1ll << 31) || w.units_cap >= (1ll << 31) ||
        g.nt >= (1 << 24) || g.bh * g.nt * 64 >= (1ll << 31))
        return SA_ERR_UNSUPPORTED;
    if ((st = ensure_attributes()) != SA_OK) return st;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return SA_ERR_CUDA;
    }
    uint8_t* base = static_cast<uint8_t*>(workspace);
    const int64_t M = g.bh * g.nt;
    const int64_t n_sink_rows = g.S * g.n_sink;

    BwdArgs a;
    memset(&a, 0, sizeof(a));
    TcArgs& t = a.geo;
    bool ok = encode_rows_bf16(&t.tm_q, q, g.bh * g.L) && encode_rows_bf16(&t.tm_k, k, g.bh * g.L) &&
              encode_vt_tiles(&t.tm_vt, base + w.kt, M) && encode_rows_bf16(&a.tm_do, d_o, g.bh * g.L) &&
              encode_rows_bf16(&a.tm_v, v, g.bh * g.L) && encode_vt_tiles(&a.tm_qt, base + w.qt, M) &&
              encode_vt_tiles(&a.tm_dot, base + w.dot, M);
    if (w.n_sink_tiles > 0)
        ok = ok && encode_rows_bf16(&t.tm_sk, sink_k_or_null, g.bh * n_sink_rows) &&
             encode_rows_bf16(&a.tm_sv, sink_v_or_null, g.bh * n_sink_rows) &&
             encode_vt_tiles(&t.tm_svt, base + w.skt, g.bh * w.n_sink_tiles);
    else
        t.tm_sk = t.tm_k, a.tm_sv = a.tm_v, t.tm_svt = t.tm_vt;
    if (lm)
        ok = ok && encode_rows_bf16(&t.tm_lk, base + w.lk, g.bh * w.ntp) &&
             encode_rows_bf16(&a.tm_lv, base + w.lv, g.bh * w.ntp) &&
             encode_vt_tiles(&t.tm_lvt, base + w.lkt, g.bh * w.n_lm_chunks);
    else
        t.tm_lk = t.tm_k, a.tm_lv = a.tm_v, t.tm_lvt = t.tm_vt;
    if (!ok) return SA_ERR_CUDA;

    // ---- per-row terms and transposed operand tiles
    {
        const int64_t rows = M * 128;
        bwd_rows_kernel<<<(unsigned)((rows + 31) / 32), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(d_o), lse,
            reinterpret_cast<float*>(base + w.lse2t), reinterpret_cast<float*>(base + w.dt), (int32_t)g.bh,
            (int32_t)g.nt, (int32_t)g.tpf, (int32_t)g.N, (int32_t)g.L);
        if ((st = launch_status()) != SA_OK) return st;
    }
    if ((st = transpose_tiles(q, base + w.qt, g.nt, true, g, g.L, stream)) != SA_OK) return st;
    if ((st = transpose_tiles(d_o, base + w.dot, g.nt, true, g, g.L, stream)) != SA_OK) return st;
    if ((st = transpose_tiles(k, base + w.kt, g.nt, true, g, g.L, stream)) != SA_OK) return st;
    if (w.n_sink_tiles > 0 &&
        (st = transpose_tiles(sink_k_or_null, base + w.skt, w.n_sink_tiles, false, g, n_sink_rows, stream)) != SA_OK)
        return st;
    if (lm) {
        const int64_t n4 = g.bh * w.ntp * 16;
        const int blocks = (int)std::min<int64_t>((n4 + 255) / 256, 148 * 32);
        float* lbias = reinterpret_cast<float*>(base + w.lbias);
        __nv_bfloat16* lvt = reinterpret_cast<__nv_bfloat16*>(base + w.lvt);
        landmark_prep_kernel<<<blocks, 256, 0, stream>>>(k_pool_or_null, v_pool_or_null, k_cnt_or_null,
                                                         reinterpret_cast<__nv_bfloat16*>(base + w.lk), lvt, lbias,
                                                         (int32_t)g.bh, (int32_t)g.nt, (int32_t)w.ntp);
        if ((st = launch_status()) != SA_OK) return st;
        landmark_prep_kernel<<<blocks, 256, 0, stream>>>(v_pool_or_null, v_pool_or_null, k_cnt_or_null,
                                                         reinterpret_cast<__nv_bfloat16*>(base + w.lv), lvt, lbias,
                                                         (int32_t)g.bh, (int32_t)g.nt, (int32_t)w.ntp);
        if ((st = launch_status()) != SA_OK) return st;
        if ((st = transpose_tiles(base + w.lk, base + w.lkt, w.n_lm_chunks, false, g, w.ntp, stream)) != SA_OK)
            return st;
        if (cudaMemsetAsync(base + w.bits, 0, (size_t)M * w.words * 4, stream) != cudaSuccess) return SA_ERR_CUDA;
    }

    // ---- reverse lists and the dK/dV work units
    int32_t* rev_cnt = reinterpret_cast<int32_t*>(base + w.rev_cnt);
    int32_t* fill = reinterpret_cast<int32_t*>(base + w.fill);
    if (cudaMemsetAsync(rev_cnt, 0, (size_t)M * 4, stream) != cudaSuccess) return SA_ERR_CUDA;
    {
        const int64_t total = M * max_kept;
        const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, (int64_t)sms * 16));
        bwd_scan_lists_kernel<<<blocks, 256, 0, stream>>>(kept_idx, kept_cnt, max_kept, (int32_t)g.bh, (int32_t)g.nt,
                                                          (int32_t)w.words,
                                                          lm ? reinterpret_cast<uint32_t*>(base + w.bits) : nullptr,
                                                          rev_cnt);
        if ((st = launch_status()) != SA_OK) return st;
        bwd_plan_kernel<<<1, 1024, 0, stream>>>(rev_cnt, fill, reinterpret_cast<int4*>(base + w.units),
                                                reinterpret_cast<int32_t*>(base + w.n_units), (int32_t)g.bh,
                                                (int32_t)g.nt, (int32_t)w.n_sink_tiles, (int32_t)w.n_lm_chunks,
                                                (int64_t)w.units_cap);
        if ((st = launch_status()) != SA_OK) return st;
        bwd_fill_lists_kernel<<<blocks, 256, 0, stream>>>(kept_idx, kept_cnt, max_kept, (int32_t)g.bh, (int32_t)g.nt,
                                                          fill, reinterpret_cast<int32_t*>(base + w.rev));
        if ((st = launch_status()) != SA_OK) return st;
    }
    if (cudaMemsetAsync(base + w.dk32, 0, (size_t)g.bh * g.L * 64 * 4, stream) != cudaSuccess ||
        cudaMemsetAsync(base + w.dv32, 0, (size_t)g.bh * g.L * 64 * 4, stream) != cudaSuccess)
        return SA_ERR_CUDA;
    if (lm && (cudaMemsetAsync(base + w.dkbar, 0, (size_t)g.bh * w.ntp * 64 * 4, stream) != cudaSuccess ||
               cudaMemsetAsync(base + w.dvbar, 0, (size_t)g.bh * w.ntp * 64 * 4, stream) != cudaSuccess))
        return SA_ERR_CUDA;

    // ---- the two tensor-core kernels
    t.kept_idx = kept_idx;
    t.kept_cnt = kept_cnt;
    t.lbias2 = lm ? reinterpret_cast<const float*>(base + w.lbias) : nullptr;
    t.max_kept = max_kept;
    t.frames = (int32_t)g.S;
    t.tokens = (int32_t)g.N;
    t.n_sink = (int32_t)g.n_sink;
    t.tpf = (int32_t)g.tpf;
    t.nt = (int32_t)g.nt;
    t.L = (int32_t)g.L;
    t.Lk = (int32_t)g.L;
    t.ntp = (int32_t)w.ntp;
    t.n_vtiles = (int32_t)g.nt;
    t.n_sink_rows = (int32_t)n_sink_rows;
    t.n_sink_tiles = (int32_t)w.n_sink_tiles;
    t.n_lm_chunks = (int32_t)w.n_lm_chunks;
    t.dense = 0;
    t.landmark = lm ? 1 : 0;
    t.q_per_head = (int32_t)g.nt;
    t.total_items = (int32_t)M;
    t.scale_log2 = (float)((double)g.scale * 1.4426950408889634);
    t.tpf_magic = 0;
    if (g.tpf > 1) {
        t.tpf_magic = (uint32_t)((0x100000000ull + (uint64_t)g.tpf - 1) / (uint64_t)g.tpf);
        for (int64_t j = 0; j < g.nt; ++j)
            if ((int64_t)(((uint64_t)j * t.tpf_magic) >> 32) != j / g.tpf) return SA_ERR_UNSUPPORTED;
    }
    a.lse2t = reinterpret_cast<const float*>(base + w.lse2t);
    a.dt = reinterpret_cast<const float*>(base + w.dt);
    a.listed_bits = lm ? reinterpret_cast<const uint32_t*>(base + w.bits) : nullptr;
    a.units = reinterpret_cast<const int4*>(base + w.units);
    a.n_units = reinterpret_cast<const int32_t*>(base + w.n_units);
    a.rev = reinterpret_cast<const int32_t*>(base + w.rev);
    a.dq = static_cast<__nv_bfloat16*>(dq);
    a.dk32 = reinterpret_cast<float*>(base + w.dk32);
    a.dv32 = reinterpret_cast<float*>(base + w.dv32);
    a.dkbar = lm ? reinterpret_cast<float*>(base + w.dkbar) : nullptr;
    a.dvbar = lm ? reinterpret_cast<float*>(base + w.dvbar) : nullptr;
    a.scale = g.scale;
    attn_bwd_dq_kernel<<<(unsigned)M, bw::kThreads, bw::QLay::smem_bytes(), stream>>>(a);
    if ((st = launch_status()) != SA_OK) return st;
    const int grid = (int)std::min<int64_t>(sms, w.units_cap);
    attn_bwd_dkv_kernel<<<grid, bw::kThreads, bw::KVLay::smem_bytes(), stream>>>(a);
    if ((st = launch_status()) != SA_OK) return st;
    {
        const int64_t total = g.bh * g.L * 8;
        const int blocks = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sms * 32);
        bwd_finalize_kernel<<<blocks, 256, 0, stream>>>(
            reinterpret_cast<const float*>(base + w.dk32), reinterpret_cast<const float*>(base + w.dv32),
            lm ? reinterpret_cast<const float*>(base + w.dkbar) : nullptr,
            lm ? reinterpret_cast<const float*>(base + w.dvbar) : nullptr, static_cast<__nv_bfloat16*>(dk),
            static_cast<__nv_bfloat16*>(dv), (int32_t)g.bh, (int32_t)g.L, (int32_t)g.N, (int32_t)g.tpf,
            (int32_t)g.n_sink, (int32_t)w.ntp);
        if ((st = launch_status()) != SA_OK) return st;
    }
    return SA_OK;
}

}  // extern "C"
