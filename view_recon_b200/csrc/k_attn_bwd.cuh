// Backward of the block-sparse attention (step 4) on the 5th-generation tensor cores: bf16,
// d = 64, tile = 128.  For post-conversion training of a sparse backbone ("Zebra3D",
// abstract: tile-sparse attention with landmark summaries of the unselected tiles).
//
// The kept lists are constants of the call (selection is piecewise constant), so the
// gradients are those of softmax attention over each query tile's attended set:
//   P = exp(scale q.k + b - LSE),  D_r = rowsum(dO_r * O_r),  dS = P * (dO V^T - D)
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO
// with the landmark of an unselected tile j standing for the mean of its c_j non-sink rows:
// its gradient reaches each of those rows divided by c_j.
//
// Two kernels share nothing but their operands:
//   attn_bwd_dq_kernel   one CTA per query tile (like the forward): walks the tile's item list
//                        (listed tiles, sink chunks, landmark chunks) and accumulates
//                          S = Q K^T, dP = dO V^T      (SS, both operands K-major)
//                          dQ += dS K                  (TS: dS from TMEM, K^T tile K-major)
//                        dQ is written once, in bf16, with no atomics.
//   attn_bwd_dkv_kernel  persistent, one CTA per SM, over "units": a key item (a key tile, a
//                        sink chunk or a landmark chunk) and a run of at most kBwdChunk query
//                        tiles that attend it (the reverse of the kept lists, built on the
//                        device).  Per pair it recomputes, transposed (thread = key row),
//                          S^T = K Q^T, dP^T = V dO^T  (SS)
//                          dV += P^T dO,  dK += dS^T Q (TS: P^T / dS^T from TMEM, dO^T / Q^T
//                                                       tiles K-major)
//                        and adds the unit's dK, dV rows to fp32 accumulators (float4 atomics;
//                        a key item split over several units, and every sink row, receives
//                        several contributions).
// Warp roles of both kernels (640 threads, one CTA per SM): warp 0 and warp 2 the TMA producers
// of the two operand rings, warp 1 the tcgen05.mma issuer (it also owns the TMEM allocation),
// warp 3 idle, warpgroups 1-4 the elementwise work (32 of the 128 columns each; a thread owns one
// row of the 128-row tile).
// Every operand is staged K-major in shared memory by TMA (128-byte swizzle); the transposed
// tiles (Q^T, dO^T, K^T) are written once per call by the transpose kernel of the forward.
// Every wait is bounded (g_sa_wait_limit_ns) and drains what the role has in flight.
#pragma once
#include "k_attn_tc.cuh"

constexpr int kBwdChunk = 32;  // query tiles per dK/dV unit at most

struct __align__(64) BwdArgs {
    // Item geometry and maps shared with the forward's list walk: tm_q = Q rows, tm_k = K rows,
    // tm_vt = transposed K tiles, tm_sk = sink K rows, tm_svt = transposed sink K tiles,
    // tm_lk = landmark K rows, tm_lvt = transposed landmark K chunks.
    TcArgs geo;
    CUtensorMap tm_do, tm_v, tm_sv, tm_lv;  // dO rows, V rows, sink V rows, landmark V rows
    CUtensorMap tm_qt, tm_dot;              // transposed query tiles of Q and dO [bh*nt*64][128]
    const float* lse2t;                     // [bh][nt][128] -LSE*log2(e) per query tile row, -inf past the tile
    const float* dt;                        // [bh][nt][128] -rowsum(dO*O), 0 past the tile
    const uint32_t* listed_bits;            // [bh][nt][ntp/32] bit j: tile j is listed (landmark mode)
    const int4* units;                      // {h, kind << 24 | item, first, end}
    const int32_t* n_units;
    const int32_t* rev;                     // query tiles of each key tile, grouped by key tile
    __nv_bfloat16* dq;                      // [bh][L][64]
    float* dk32;                            // [bh][L][64] accumulators
    float* dv32;
    float* dkbar;                           // [bh][ntp][64] landmark gradients
    float* dvbar;
    float scale;
};

namespace bw {

constexpr int kT = tc::kTileBytes;
constexpr int kThreads = 640;   // warps 0-3 control, warpgroups 1-4 the elementwise work
constexpr int kCompute = 512;

// Operands come through two rings per kernel, each with its own producer warp: the row tiles
// read by the S / dP products (released as soon as those complete; in the dK/dV kernel also
// once every elementwise thread has read the per-row terms that ride with them) and the
// transposed tiles read by the gradient products (released after them), so that the next
// tiles' copies start early and their latency stays off the tensor pipe's path.
struct QLay {
    static constexpr int RS = 4, TS = 3;
    static constexpr int kQ = 0, kDO = kT;
    static constexpr int kRows = 2 * kT, kRowStage = 2 * kT;  // [RS] K rows, V rows
    static constexpr int kTr = kRows + RS * kRowStage, kTrStage = kT;  // [TS] K^T
    static constexpr int kBars = kTr + TS * kTrStage;
    static constexpr int kNumBars = 1 + 2 * RS + 2 * TS + 5;
    static constexpr int kMisc = kBars + 8 * kNumBars;
    static constexpr int kEnd = kMisc + 16;
    static constexpr uint32_t colS = 0, colDP = 128, colDS = 256, colDQ = 320;
    static size_t smem_bytes() { return 1024 + kEnd; }
};

struct KVLay {
    static constexpr int RS = 3, TS = 2;
    static constexpr int kK = 0, kV = kT;
    static constexpr int kRows = 2 * kT, kRowStage = 2 * kT + 1024;  // [RS] Q rows, dO rows, -lse2[128], -D[128]
    static constexpr int kTr = kRows + RS * kRowStage, kTrStage = 2 * kT;  // [TS] Q^T, dO^T
    static constexpr int kBars = kTr + TS * kTrStage;
    static constexpr int kNumBars = 2 * RS + 2 * TS + 9;
    static constexpr int kMisc = kBars + 8 * kNumBars;
    static constexpr int kEnd = kMisc + 16;
    static constexpr uint32_t colS = 0, colDP = 128, colP = 256, colDS = 320, colDV = 384, colDK = 448;
    static size_t smem_bytes() { return 1024 + kEnd; }
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Query tile i of head h: first row in the [bh*L][64] row maps and valid rows.
__device__ __forceinline__ void query_tile(const TcArgs& g, int h, int i, int32_t* qrow, int* nq) {
    const int f = g.tpf == 1 ? i : (int)__umulhi((uint32_t)i, g.tpf_magic);
    const int slot = i - f * g.tpf;
    *qrow = h * g.L + f * g.tokens + slot * 128;
    *nq = min(128, g.tokens - slot * 128);
}

}  // namespace bw

// ------------------------------------------------------------------------------ dQ

__global__ void __launch_bounds__(640, 1) attn_bwd_dq_kernel(const __grid_constant__ BwdArgs a) {
    using Lay = bw::QLay;
    constexpr int RS = Lay::RS, TS = Lay::TS;
    constexpr int kT = bw::kT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = bw::align1024(smem_raw);
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* sQ = smem + Lay::kQ;
    uint8_t* sDO = smem + Lay::kDO;
    uint8_t* sRows = smem + Lay::kRows;
    uint8_t* sTr = smem + Lay::kTr;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBars);
    uint64_t* q_full = bars;
    uint64_t* rows_full = bars + 1;
    uint64_t* rows_empty = rows_full + RS;
    uint64_t* t_full = rows_empty + RS;
    uint64_t* t_empty = t_full + TS;
    uint64_t* sd_full = t_empty + TS;
    uint64_t* sd_free = sd_full + 1;
    uint64_t* ds_full = sd_free + 1;
    uint64_t* dq_done = ds_full + 1;
    uint64_t* drain_bar = dq_done + 1;
    const TcArgs& g = a.geo;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < RS; ++s) {
            mbar_init(&rows_full[s], 1);
            mbar_init(&rows_empty[s], 1);
        }
        for (int s = 0; s < TS; ++s) {
            mbar_init(&t_full[s], 1);
            mbar_init(&t_empty[s], 1);
        }
        mbar_init(sd_full, 1);
        mbar_init(sd_free, bw::kCompute);
        mbar_init(ds_full, bw::kCompute);
        mbar_init(dq_done, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    const tc::Slot sl = tc::make_slot(g, blockIdx.x);
    const int n_items = sl.n_items;

    if (warp == 0 || warp == 2) {
        // ------------------------------------------------------------------ TMA producers
        // warp 0: Q, dO, then K and V rows of every item; warp 2: the transposed K tiles
        const bool rows = warp == 0;
        const int depth = rows ? RS : TS;
        uint64_t* full = rows ? rows_full : t_full;
        uint64_t* empty = rows ? rows_empty : t_empty;
        const bool leader = tc::elect_one();
        uint32_t issued_mask = 0, phase_mask = 0;
        bool ok = true;
        const bool withhold = g_sa_test_withhold != 0 && blockIdx.x == 0;  // failure-path test facility
        if (rows && n_items > 0 && leader && !withhold) {
            mbar_arrive_expect_tx(q_full, 2 * kT);
            tma_load_2d(sQ, &g.tm_q, q_full, 0, sl.qrow);
            tma_load_2d(sDO, &a.tm_do, q_full, 0, sl.qrow);
        }
        for (int n = 0; n < n_items; ++n) {
            const uint32_t s = n % depth, ph = (n / depth) & 1u;
            if (!mbar_wait_warp(&empty[s], ph ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (leader) {
                const tc::Item it = tc::get_item(g, sl, n);
                if (rows) {
                    const CUtensorMap* mk = it.kind == 1 ? &g.tm_sk : (it.kind == 2 ? &g.tm_lk : &g.tm_k);
                    const CUtensorMap* mv = it.kind == 1 ? &a.tm_sv : (it.kind == 2 ? &a.tm_lv : &a.tm_v);
                    uint8_t* d = sRows + s * Lay::kRowStage;
                    mbar_arrive_expect_tx(&full[s], 2 * kT);
                    tma_load_2d(d, mk, &full[s], 0, it.krow);
                    tma_load_2d(d + kT, mv, &full[s], 0, it.krow);
                } else {
                    const CUtensorMap* mt = it.kind == 1 ? &g.tm_svt : (it.kind == 2 ? &g.tm_lvt : &g.tm_vt);
                    uint8_t* d = sTr + s * Lay::kTrStage;
                    mbar_arrive_expect_tx(&full[s], kT);
                    tma_load_2d(d, mt, &full[s], 0, it.vrow);
                    tma_load_2d(d + kT / 2, mt, &full[s], 64, it.vrow);
                }
            }
            issued_mask |= 1u << s;
            phase_mask = (phase_mask & ~(1u << s)) | (ph << s);
        }
        if (!ok) {
            for (int s = 0; s < depth; ++s)
                if ((issued_mask >> s) & 1u) tc::drain_wait(&full[s], (phase_mask >> s) & 1u);
            if (rows && n_items > 0 && !withhold) tc::drain_wait(q_full, 0);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        const bool leader = tc::elect_one();
        bool ok = n_items == 0 || mbar_wait_warp(q_full, 0, abort_flag);
        bool any_mma = false;
        tc_fence_after();
        const uint64_t dq_desc = smem_desc_sw128(smem_u32(sQ), 16, 1024);
        const uint64_t ddo = smem_desc_sw128(smem_u32(sDO), 16, 1024);
        const uint64_t dk0 = smem_desc_sw128(smem_u32(sRows), 16, 1024);
        const uint64_t dv0 = smem_desc_sw128(smem_u32(sRows + kT), 16, 1024);
        const uint64_t dt0 = smem_desc_sw128(smem_u32(sTr), 16, 1024);
        constexpr uint64_t kRowStep = (uint64_t)Lay::kRowStage >> 4;
        constexpr uint64_t kTrStep = (uint64_t)Lay::kTrStage >> 4;
        for (int n = 0; n <= n_items && ok; ++n) {
            if (n < n_items) {
                const uint32_t s = n % RS, ph = (n / RS) & 1u;
                if (!mbar_wait_warp(&rows_full[s], ph, abort_flag)) { ok = false; break; }
                if (n > 0 && !mbar_wait_warp(sd_free, (n - 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_ss(tmem + Lay::colS, dq_desc + 2 * kk, dk0 + s * kRowStep + 2 * kk, tc::kIdescS, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_ss(tmem + Lay::colDP, ddo + 2 * kk, dv0 + s * kRowStep + 2 * kk, tc::kIdescS, kk > 0);
                    umma_commit(sd_full);
                    umma_commit(&rows_empty[s]);
                }
                __syncwarp();
                any_mma = true;
            }
            if (n >= 1) {
                const int m = n - 1;
                const uint32_t s = m % TS, ph = (m / TS) & 1u;
                if (!mbar_wait_warp(ds_full, m & 1, abort_flag)) { ok = false; break; }
                if (!mbar_wait_warp(&t_full[s], ph, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
                    const uint64_t dt = dt0 + s * kTrStep;
                    // K^T is two 64-key swizzle atoms of 8 KB; a K=16 step is 32 bytes
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ts(tmem + Lay::colDQ, tmem + Lay::colDS + 8 * kk,
                                dt + (uint64_t)((kk >> 2) * (8192 >> 4) + (kk & 3) * 2), tc::kIdescPV,
                                (m > 0 || kk > 0));
                    umma_commit(&t_empty[s]);
                    umma_commit(dq_done);
                }
                __syncwarp();
            }
        }
        if (any_mma) {
            if (leader) umma_commit(drain_bar);
            __syncwarp();
            tc::drain_wait(drain_bar, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ dS (thread = query row)
        const int hc = (warp - 4) >> 2;  // key columns [32 hc, 32 hc + 32)
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + Lay::colS + lane_off + hc * 32;
        const uint32_t tDP = tmem + Lay::colDP + lane_off + hc * 32;
        const uint32_t tDS = tmem + Lay::colDS + lane_off + hc * 16;
        const uint32_t tDQ = tmem + Lay::colDQ + lane_off + hc * 16;
        float nlse2 = -INFINITY, ndrow = 0.0f;  // -LSE (base 2) and -D of this row
        if (sl.active) {
            const int64_t ti = ((int64_t)sl.h * g.nt + sl.i) * 128 + r;
            nlse2 = __ldg(a.lse2t + ti);
            ndrow = __ldg(a.dt + ti);
        }
        const float2 scale2 = make_float2(g.scale_log2, g.scale_log2);
        const float2 nl2 = make_float2(nlse2, nlse2);
        const float2 nd2 = make_float2(ndrow, ndrow);
        bool ok = true;
        int lm_ptr = 0;
        for (int n = 0; n < n_items; ++n) {
            const int j_cur = n < sl.cnt ? __ldg(sl.list + n) : 0;
            const tc::Item it = tc::get_item_j(g, sl, n, j_cur);
            if (it.kind < 0 && threadIdx.x == 128) sa_flag_error(SA_ERR_BAD_LIST);
            // validity of this warpgroup's 32 key columns [32 hc, 32 hc + 32): the tile's valid rows,
            // or for a landmark chunk the tiles the list does not hold
            uint32_t vmask;
            if (it.kind == 2) {
                const int c_lo = it.chunk * 128, w_lo = c_lo + 32 * hc;
                uint32_t listed = 0u;
                while (lm_ptr < sl.cnt) {
                    const int j = __ldg(sl.list + lm_ptr);
                    if (j >= c_lo + 128) break;
                    if (j >= w_lo && j < w_lo + 32) listed |= 1u << (j - w_lo);
                    ++lm_ptr;
                }
                vmask = ~listed;
            } else {
                const int lo = max(0, it.lo - 32 * hc), hi = min(32, it.hi - 32 * hc);
                vmask = hi <= lo ? 0u : ((hi - lo == 32 ? 0xFFFFFFFFu : ((1u << (hi - lo)) - 1u)) << lo);
            }
            if (!mbar_wait_warp(sd_full, n & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[32], dp[32];
            tmem_ld_32x32b_x32(tS, sv);
            tmem_ld_32x32b_x32(tDP, dp);
            tmem_ld_wait(sv);
            reg_fence(dp);
            tc_fence_before();
            mbar_arrive(sd_free);  // the next item's products may overwrite S and dP now
            uint32_t pk[16];
            if (it.kind != 2 && vmask == 0xFFFFFFFFu) {
                // whole tile attended: no mask, no bias
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * u]), __uint_as_float(sv[2 * u + 1])),
                                                scale2, nl2);
                    float2 p;
                    p.x = ex2_approx(x.x);
                    p.y = ex2_approx(x.y);
                    const float2 d = __fmul2_rn(
                        p, __fadd2_rn(make_float2(__uint_as_float(dp[2 * u]), __uint_as_float(dp[2 * u + 1])), nd2));
                    pk[u] = pack_bf16x2(d.x, d.y);
                }
            } else {
                // partial tile, sink chunk tail, landmark chunk (per-column bias) or skipped entry
                const float2* b2p = it.kind == 2
                    ? reinterpret_cast<const float2*>(g.lbias2 + it.chunk * 128 + 32 * hc) : nullptr;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const float2 nb = b2p ? __fadd2_rn(nl2, __ldg(b2p + u)) : nl2;
                    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[2 * u]), __uint_as_float(sv[2 * u + 1])),
                                                scale2, nb);
                    float2 p;
                    p.x = ((vmask >> (2 * u)) & 1u) ? ex2_approx(x.x) : 0.0f;
                    p.y = ((vmask >> (2 * u + 1)) & 1u) ? ex2_approx(x.y) : 0.0f;
                    const float2 d = __fmul2_rn(
                        p, __fadd2_rn(make_float2(__uint_as_float(dp[2 * u]), __uint_as_float(dp[2 * u + 1])), nd2));
                    pk[u] = pack_bf16x2(d.x, d.y);
                }
            }
            if (n > 0) {
                if (!mbar_wait_warp(dq_done, (n - 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
            }
            tmem_st_32x32b_x16(tDS, pk);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(ds_full);
        }
        if (ok && n_items > 0 && mbar_wait_warp(dq_done, (n_items - 1) & 1, abort_flag)) {
            tc_fence_after();
            uint32_t acc[16];
            tmem_ld_32x32b_x16(tDQ, acc);
            tmem_ld_wait16(acc);
            if (r < sl.nq) {
                uint4* dst = reinterpret_cast<uint4*>(a.dq + ((int64_t)sl.qrow + r) * 64 + hc * 16);
#pragma unroll
                for (int c8 = 0; c8 < 2; ++c8) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(acc[8 * c8 + 0]) * a.scale, __uint_as_float(acc[8 * c8 + 1]) * a.scale);
                    w.y = pack_bf16x2(__uint_as_float(acc[8 * c8 + 2]) * a.scale, __uint_as_float(acc[8 * c8 + 3]) * a.scale);
                    w.z = pack_bf16x2(__uint_as_float(acc[8 * c8 + 4]) * a.scale, __uint_as_float(acc[8 * c8 + 5]) * a.scale);
                    w.w = pack_bf16x2(__uint_as_float(acc[8 * c8 + 6]) * a.scale, __uint_as_float(acc[8 * c8 + 7]) * a.scale);
                    dst[c8] = w;
                }
            }
        } else if (ok && sl.active && n_items == 0 && r < sl.nq) {
            uint4* dst = reinterpret_cast<uint4*>(a.dq + ((int64_t)sl.qrow + r) * 64 + hc * 16);
            dst[0] = make_uint4(0, 0, 0, 0);
            dst[1] = make_uint4(0, 0, 0, 0);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------ dK, dV

namespace bw {

struct Unit {
    int h, kind, item, first, end;
};

__device__ __forceinline__ Unit load_unit(const int4* units, int u) {
    const int4 v = __ldg(units + u);
    Unit x;
    x.h = v.x;
    x.kind = (int)((uint32_t)v.y >> 24);
    x.item = v.y & 0xFFFFFF;
    x.first = v.z;
    x.end = v.w;
    return x;
}

// Key item of a unit: first row in its row maps, valid rows [lo, hi).
__device__ __forceinline__ void key_item(const TcArgs& g, const Unit& x, int32_t* krow, int* lo, int* hi) {
    if (x.kind == 0) {
        const int j = x.item;
        const int f = g.tpf == 1 ? j : (int)__umulhi((uint32_t)j, g.tpf_magic);
        const int n0 = (j - f * g.tpf) * 128;
        const int nk = min(128, g.tokens - n0);
        *krow = x.h * g.L + f * g.tokens + n0;
        *lo = min(nk, max(0, g.n_sink - n0));
        *hi = nk;
    } else if (x.kind == 1) {
        *krow = x.h * g.n_sink_rows + x.item * 128;
        *lo = 0;
        *hi = min(128, g.n_sink_rows - x.item * 128);
    } else {
        *krow = x.h * g.ntp + x.item * 128;
        *lo = 0;
        *hi = min(128, g.nt - x.item * 128);
    }
}

__device__ __forceinline__ int unit_query_tile(const BwdArgs& a, const Unit& x, int n) {
    return x.kind == 0 ? __ldg(a.rev + x.first + n) : x.first + n;
}

}  // namespace bw

__global__ void __launch_bounds__(640, 1) attn_bwd_dkv_kernel(const __grid_constant__ BwdArgs a) {
    using Lay = bw::KVLay;
    constexpr int RS = Lay::RS, TS = Lay::TS;
    constexpr int kT = bw::kT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = bw::align1024(smem_raw);
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* sK = smem + Lay::kK;
    uint8_t* sV = smem + Lay::kV;
    uint8_t* sRows = smem + Lay::kRows;
    uint8_t* sTr = smem + Lay::kTr;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBars);
    uint64_t* rows_full = bars;               // [RS] Q, dO rows and row terms of a pair loaded
    uint64_t* rows_empty = rows_full + RS;    // [RS] ... consumed by S^T, dP^T and the elementwise warps
    uint64_t* t_full = rows_empty + RS;       // [TS] Q^T, dO^T of a pair loaded
    uint64_t* t_empty = t_full + TS;          // [TS] ... consumed by dV, dK
    uint64_t* kvu_full = t_empty + TS;        // unit's K, V rows loaded
    uint64_t* kvu_empty = kvu_full + 1;       // unit's K, V rows consumed
    uint64_t* s_full = kvu_empty + 1;         // S^T, dP^T in TMEM
    uint64_t* s_free = s_full + 1;            // S^T, dP^T read
    uint64_t* pd_full = s_free + 1;           // P^T, dS^T in TMEM
    uint64_t* pd_done = pd_full + 1;          // dV, dK products of the pair done
    uint64_t* unit_done = pd_done + 1;        // unit's accumulators final
    uint64_t* acc_free = unit_done + 1;       // unit's accumulators read
    uint64_t* drain_bar = acc_free + 1;
    const TcArgs& g = a.geo;

    if (threadIdx.x == 0) {
        for (int s = 0; s < RS; ++s) {
            mbar_init(&rows_full[s], 1);
            mbar_init(&rows_empty[s], 1 + bw::kCompute);  // the products' commit + every reader of the row terms
        }
        for (int s = 0; s < TS; ++s) {
            mbar_init(&t_full[s], 1);
            mbar_init(&t_empty[s], 1);
        }
        mbar_init(kvu_full, 1);
        mbar_init(kvu_empty, 1);
        mbar_init(s_full, 1);
        mbar_init(s_free, bw::kCompute);
        mbar_init(pd_full, bw::kCompute);
        mbar_init(pd_done, 1);
        mbar_init(unit_done, 1);
        mbar_init(acc_free, bw::kCompute);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    const int n_units = *a.n_units;

    if (warp == 0 || warp == 2) {
        // ------------------------------------------------------------------ TMA producers
        // warp 0: each unit's K, V rows, then the Q and dO rows and row terms of its pairs;
        // warp 2: the transposed Q, dO tiles of its pairs
        const bool rows = warp == 0;
        const int depth = rows ? RS : TS;
        uint64_t* full = rows ? rows_full : t_full;
        uint64_t* empty = rows ? rows_empty : t_empty;
        const bool leader = tc::elect_one();
        uint32_t pc = 0;  // pairs issued by this warp
        uint32_t issued_mask = 0, phase_mask = 0;
        int kvu_loads = 0;
        bool ok = true;
        int ui = 0;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ui) {
            const bw::Unit x = bw::load_unit(a.units, u);
            if (rows) {
                if (ui > 0 && !mbar_wait_warp(kvu_empty, (ui - 1) & 1, abort_flag)) { ok = false; break; }
                if (leader) {
                    int32_t krow;
                    int lo, hi;
                    bw::key_item(g, x, &krow, &lo, &hi);
                    const CUtensorMap* mk = x.kind == 1 ? &g.tm_sk : (x.kind == 2 ? &g.tm_lk : &g.tm_k);
                    const CUtensorMap* mv = x.kind == 1 ? &a.tm_sv : (x.kind == 2 ? &a.tm_lv : &a.tm_v);
                    mbar_arrive_expect_tx(kvu_full, 2 * kT);
                    tma_load_2d(sK, mk, kvu_full, 0, krow);
                    tma_load_2d(sV, mv, kvu_full, 0, krow);
                }
                ++kvu_loads;
            }
            const int npairs = x.end - x.first;
            for (int n = 0; n < npairs; ++n, ++pc) {
                const uint32_t s = pc % depth, ph = (pc / depth) & 1u;
                if (!mbar_wait_warp(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
                if (leader) {
                    const int i = bw::unit_query_tile(a, x, n);
                    const int64_t ti = (int64_t)x.h * g.nt + i;
                    if (rows) {
                        int32_t qrow;
                        int nq;
                        bw::query_tile(g, x.h, i, &qrow, &nq);
                        uint8_t* d = sRows + s * Lay::kRowStage;
                        mbar_arrive_expect_tx(&full[s], 2 * kT + 1024);
                        tma_load_2d(d, &g.tm_q, &full[s], 0, qrow);
                        tma_load_2d(d + kT, &a.tm_do, &full[s], 0, qrow);
                        bulk_load(d + 2 * kT, a.lse2t + ti * 128, 512, &full[s]);
                        bulk_load(d + 2 * kT + 512, a.dt + ti * 128, 512, &full[s]);
                    } else {
                        uint8_t* d = sTr + s * Lay::kTrStage;
                        mbar_arrive_expect_tx(&full[s], 2 * kT);
                        tma_load_2d(d, &a.tm_qt, &full[s], 0, (int32_t)(ti * 64));
                        tma_load_2d(d + kT / 2, &a.tm_qt, &full[s], 64, (int32_t)(ti * 64));
                        tma_load_2d(d + kT, &a.tm_dot, &full[s], 0, (int32_t)(ti * 64));
                        tma_load_2d(d + kT + kT / 2, &a.tm_dot, &full[s], 64, (int32_t)(ti * 64));
                    }
                }
                issued_mask |= 1u << s;
                phase_mask = (phase_mask & ~(1u << s)) | (ph << s);
            }
        }
        if (!ok) {
            for (int s = 0; s < depth; ++s)
                if ((issued_mask >> s) & 1u) tc::drain_wait(&full[s], (phase_mask >> s) & 1u);
            if (kvu_loads > 0) tc::drain_wait(kvu_full, (kvu_loads - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        const bool leader = tc::elect_one();
        bool ok = true, any_mma = false;
        const uint64_t dkd = smem_desc_sw128(smem_u32(sK), 16, 1024);
        const uint64_t dvd = smem_desc_sw128(smem_u32(sV), 16, 1024);
        const uint64_t dr0 = smem_desc_sw128(smem_u32(sRows), 16, 1024);
        const uint64_t dt0 = smem_desc_sw128(smem_u32(sTr), 16, 1024);
        constexpr uint64_t kRowStep = (uint64_t)Lay::kRowStage >> 4;
        constexpr uint64_t kTrStep = (uint64_t)Lay::kTrStage >> 4;
        constexpr uint64_t kTile16 = (uint64_t)kT >> 4;
        uint32_t pc = 0;
        int ui = 0;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ui) {
            const bw::Unit x = bw::load_unit(a.units, u);
            const int npairs = x.end - x.first;
            if (!mbar_wait_warp(kvu_full, ui & 1, abort_flag)) { ok = false; break; }
            for (int n = 0; n <= npairs && ok; ++n) {
                if (n < npairs) {
                    const uint32_t gp = pc + n, s = gp % RS, ph = (gp / RS) & 1u;
                    if (!mbar_wait_warp(&rows_full[s], ph, abort_flag)) { ok = false; break; }
                    if (gp > 0 && !mbar_wait_warp(s_free, (gp - 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    if (leader) {
                        const uint64_t dst = dr0 + s * kRowStep;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)  // S^T = K Q^T
                            umma_ss(tmem + Lay::colS, dkd + 2 * kk, dst + 2 * kk, tc::kIdescS, kk > 0);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)  // dP^T = V dO^T
                            umma_ss(tmem + Lay::colDP, dvd + 2 * kk, dst + kTile16 + 2 * kk, tc::kIdescS, kk > 0);
                        umma_commit(s_full);
                        umma_commit(&rows_empty[s]);
                        if (n == npairs - 1) umma_commit(kvu_empty);
                    }
                    __syncwarp();
                    any_mma = true;
                }
                if (n >= 1) {
                    const int m = n - 1;
                    const uint32_t gp = pc + m, s = gp % TS, ph = (gp / TS) & 1u;
                    if (!mbar_wait_warp(pd_full, gp & 1, abort_flag)) { ok = false; break; }
                    if (m == 0 && ui > 0 && !mbar_wait_warp(acc_free, (ui - 1) & 1, abort_flag)) { ok = false; break; }
                    if (!mbar_wait_warp(&t_full[s], ph, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    if (leader) {
                        const uint64_t dqt = dt0 + s * kTrStep;
                        const uint64_t ddot = dqt + kTile16;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {  // dV += P^T dO
                            const uint64_t off = (uint64_t)((kk >> 2) * (8192 >> 4) + (kk & 3) * 2);
                            umma_ts(tmem + Lay::colDV, tmem + Lay::colP + 8 * kk, ddot + off, tc::kIdescPV,
                                    (m > 0 || kk > 0));
                        }
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {  // dK += dS^T Q (scaled in the epilogue)
                            const uint64_t off = (uint64_t)((kk >> 2) * (8192 >> 4) + (kk & 3) * 2);
                            umma_ts(tmem + Lay::colDK, tmem + Lay::colDS + 8 * kk, dqt + off, tc::kIdescPV,
                                    (m > 0 || kk > 0));
                        }
                        umma_commit(&t_empty[s]);
                        umma_commit(pd_done);
                        if (m == npairs - 1) umma_commit(unit_done);
                    }
                    __syncwarp();
                }
            }
            pc += npairs;
        }
        if (any_mma) {
            if (leader) umma_commit(drain_bar);
            __syncwarp();
            tc::drain_wait(drain_bar, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ P^T, dS^T (thread = key row)
        const int hc = (warp - 4) >> 2;  // query columns [32 hc, 32 hc + 32)
        const int quad = warp & 3;
        const int t = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + Lay::colS + lane_off + hc * 32;
        const uint32_t tDP = tmem + Lay::colDP + lane_off + hc * 32;
        const uint32_t tP = tmem + Lay::colP + lane_off + hc * 16;
        const uint32_t tDS = tmem + Lay::colDS + lane_off + hc * 16;
        const float2 scale2 = make_float2(g.scale_log2, g.scale_log2);
        const int words = g.ntp >> 5;
        uint32_t pc = 0;
        bool ok = true;
        int ui = 0;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ui) {
            const bw::Unit x = bw::load_unit(a.units, u);
            const int npairs = x.end - x.first;
            const int j_lm = x.item * 128 + t;  // landmark chunks: this row's tile
            const float bias = x.kind == 2 ? __ldg(g.lbias2 + j_lm) : 0.0f;
            const float2 bias2 = make_float2(bias, bias);
            for (int n = 0; n < npairs; ++n) {
                const uint32_t gp = pc + n, s = gp % RS;
                bool masked = false;
                if (x.kind == 2) {
                    const int i = bw::unit_query_tile(a, x, n);
                    const uint32_t w = __ldg(a.listed_bits + ((int64_t)x.h * g.nt + i) * words + (j_lm >> 5));
                    masked = (w >> (j_lm & 31)) & 1u;
                }
                if (!mbar_wait_warp(s_full, gp & 1, abort_flag)) { ok = false; break; }
                // the pair's row terms came with its row tiles (bulk copy): observe that barrier
                // directly (the stage is not re-armed before this thread's arrival on rows_empty)
                if (!mbar_wait_warp(&rows_full[s], (gp / RS) & 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                // S^T, dP^T in two 16-column halves (fewer live registers): the next pair's S^T
                // product queues behind this pair's predecessor's dV, dK products in the tensor
                // pipe anyway, so holding S^T a little longer costs nothing
                // row terms of this warpgroup's 32 query columns: -LSE (base 2) and -D
                const float2* nls = reinterpret_cast<const float2*>(sRows + s * Lay::kRowStage + 2 * kT) + hc * 16;
                const float2* nds = nls + 64;
                uint32_t pp[16], pd[16];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t sv[16], dp[16];
                    tmem_ld_32x32b_x16(tS + half * 16, sv);
                    tmem_ld_32x32b_x16(tDP + half * 16, dp);
                    tmem_ld_wait16(sv);
                    tmem_ld_wait16(dp);
                    if (half == 1) {
                        tc_fence_before();
                        mbar_arrive(s_free);  // the next pair's products may overwrite S^T and dP^T now
                    }
#pragma unroll
                    for (int c2 = 0; c2 < 8; ++c2) {
                        const int cc = half * 8 + c2;
                        const float2 nl = nls[cc];
                        const float2 nb = x.kind == 2 ? __fadd2_rn(bias2, nl) : nl;
                        const float2 xv = __ffma2_rn(
                            make_float2(__uint_as_float(sv[2 * c2]), __uint_as_float(sv[2 * c2 + 1])), scale2, nb);
                        float2 p;
                        p.x = ex2_approx(xv.x);
                        p.y = ex2_approx(xv.y);
                        if (masked) p = make_float2(0.0f, 0.0f);
                        const float2 ds = __fmul2_rn(
                            p, __fadd2_rn(make_float2(__uint_as_float(dp[2 * c2]), __uint_as_float(dp[2 * c2 + 1])),
                                          nds[cc]));
                        pp[cc] = pack_bf16x2(p.x, p.y);
                        pd[cc] = pack_bf16x2(ds.x, ds.y);
                    }
                }
                mbar_arrive(&rows_empty[s]);  // row terms read: the stage may be refilled once the products are done
                if (gp > 0) {
                    if (!mbar_wait_warp(pd_done, (gp - 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                }
                tmem_st_32x32b_x16(tP, pp);
                tmem_st_32x32b_x16(tDS, pd);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(pd_full);
            }
            if (!ok) break;
            // ---- epilogue: warpgroups 0, 1 add the unit's dV rows (dims 0-31, 32-63), 2, 3 its dK rows
            if (!mbar_wait_warp(unit_done, ui & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t acc[32];
            const uint32_t tA = tmem + (hc < 2 ? Lay::colDV : Lay::colDK) + lane_off + (hc & 1) * 32;
            tmem_ld_32x32b_x32(tA, acc);
            tmem_ld_wait(acc);
            tc_fence_before();
            mbar_arrive(acc_free);
            int32_t krow;
            int lo, hi;
            bw::key_item(g, x, &krow, &lo, &hi);
            float* dst = nullptr;
            if (t >= lo && t < hi) {
                if (x.kind == 0) {
                    dst = (hc < 2 ? a.dv32 : a.dk32) + ((int64_t)krow + t) * 64;
                } else if (x.kind == 1) {
                    const int sr = x.item * 128 + t;
                    const int tok = (sr / g.n_sink) * g.tokens + sr % g.n_sink;
                    dst = (hc < 2 ? a.dv32 : a.dk32) + ((int64_t)x.h * g.L + tok) * 64;
                } else {
                    dst = (hc < 2 ? a.dvbar : a.dkbar) + ((int64_t)x.h * g.ntp + j_lm) * 64;
                }
            }
            if (dst) {
                const float mul = hc < 2 ? 1.0f : a.scale;
                float4* d4 = reinterpret_cast<float4*>(dst) + (hc & 1) * 8;
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                    atomicAdd(d4 + q4, make_float4(__uint_as_float(acc[4 * q4 + 0]) * mul,
                                                   __uint_as_float(acc[4 * q4 + 1]) * mul,
                                                   __uint_as_float(acc[4 * q4 + 2]) * mul,
                                                   __uint_as_float(acc[4 * q4 + 3]) * mul));
            }
            pc += npairs;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------ preparation

// Per query tile row, negated for the kernels' fused multiply-adds: -LSE in base-2 units (-inf
// past the tile or where no key was attended) and -D = -rowsum(dO * O) (0 past the tile); eight
// threads per row, 16 bytes each.
__global__ void __launch_bounds__(256) bwd_rows_kernel(const __nv_bfloat16* o, const __nv_bfloat16* d_o,
                                                       const float* lse, float* lse2t, float* dt, int32_t bh,
                                                       int32_t nt, int32_t tpf, int32_t tokens, int32_t L) {
    const int64_t idx = (int64_t)blockIdx.x * 32 + (threadIdx.x >> 3);  // (h, tile, row)
    const int part = threadIdx.x & 7;
    const bool in_range = idx < (int64_t)bh * nt * 128;  // no early exit: the shuffles below take full warps
    const int r = (int)(idx & 127);
    const int64_t hi_ = idx >> 7;
    const int h = (int)(hi_ / nt), i = (int)(hi_ % nt);
    const int f = i / tpf, slot = i % tpf;
    const int nq = min(128, tokens - slot * 128);
    float d = 0.0f, l2 = -INFINITY;
    if (in_range && r < nq) {
        const int64_t row = (int64_t)h * L + (int64_t)f * tokens + slot * 128 + r;
        const uint4 ov = __ldg(reinterpret_cast<const uint4*>(o + row * 64) + part);
        const uint4 gv = __ldg(reinterpret_cast<const uint4*>(d_o + row * 64) + part);
        const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            d = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(gw[e] << 16), d);
            d = fmaf(__uint_as_float(ow[e] & 0xFFFF0000u), __uint_as_float(gw[e] & 0xFFFF0000u), d);
        }
        const float lv = __ldg(lse + row);
        if (isfinite(lv)) l2 = -lv * 1.4426950408889634f;
    }
    d += __shfl_xor_sync(0xffffffffu, d, 1);
    d += __shfl_xor_sync(0xffffffffu, d, 2);
    d += __shfl_xor_sync(0xffffffffu, d, 4);
    if (in_range && part == 0) {
        lse2t[idx] = l2;
        dt[idx] = r < nq ? -d : 0.0f;
    }
}

// Listed-tile bitmap of every query tile (landmark mode) and the reverse-list counts.
__global__ void bwd_scan_lists_kernel(const int32_t* kept_idx, const int32_t* kept_cnt, int32_t max_kept,
                                      int32_t bh, int32_t nt, int32_t words, uint32_t* listed_bits,
                                      int32_t* rev_cnt) {
    const int64_t total = (int64_t)bh * nt * max_kept;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t li = e / max_kept;  // h * nt + i
        const int n = (int)(e % max_kept);
        const int cnt = min(max(__ldg(kept_cnt + li), 0), max_kept);
        if (n >= cnt) continue;
        const int j = __ldg(kept_idx + e);
        if (j < 0 || j >= nt) continue;
        const int64_t h = li / nt;
        atomicAdd(rev_cnt + h * nt + j, 1);
        if (listed_bits) atomicOr(listed_bits + li * words + (j >> 5), 1u << (j & 31));
    }
}

// One block: CSR offsets of the reverse lists (per key tile, over all heads), the unit table
// and the number of units.  fill[] starts at each list's offset for bwd_fill_lists_kernel.
// Units are written longest first, so that the persistent dK/dV kernel's round-robin walk over
// the table gives every CTA about the same work: the fixed sink / landmark units, then every
// whole run of kBwdChunk query tiles, then the shorter remainders of the lists by length
// descending (equal lengths in any order: their contributions meet in f32 atomics anyway).
// Writes at most units_cap units: a plan that would need more (possible only for malformed lists)
// is cut at the capacity, reported as SA_ERR_BAD_LIST, and the unit count clamped to it.
__global__ void __launch_bounds__(1024) bwd_plan_kernel(const int32_t* rev_cnt, int32_t* fill, int4* units,
                                                        int32_t* n_units, int32_t bh, int32_t nt,
                                                        int32_t n_sink_tiles, int32_t n_lm_chunks,
                                                        int64_t units_cap) {
    __shared__ int64_t s_e[1024], s_f[1024];
    __shared__ int32_t s_rem[kBwdChunk];     // remainder units of each length (1 .. kBwdChunk - 1)
    __shared__ int64_t s_cursor[kBwdChunk];  // next slot of each remainder length
    const int64_t M = (int64_t)bh * nt;
    const int64_t per = (M + 1023) / 1024;
    const int64_t b0 = min(M, per * threadIdx.x), b1 = min(M, b0 + per);
    if (threadIdx.x < kBwdChunk) s_rem[threadIdx.x] = 0;
    __syncthreads();
    int64_t se = 0, sf = 0;
    for (int64_t x = b0; x < b1; ++x) {
        const int c = rev_cnt[x];
        se += c;
        sf += c / kBwdChunk;
        if (c % kBwdChunk) atomicAdd(&s_rem[c % kBwdChunk], 1);
    }
    s_e[threadIdx.x] = se;
    s_f[threadIdx.x] = sf;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {  // inclusive scans (Hillis-Steele)
        const int64_t ae = threadIdx.x >= off ? s_e[threadIdx.x - off] : 0;
        const int64_t af = threadIdx.x >= off ? s_f[threadIdx.x - off] : 0;
        __syncthreads();
        s_e[threadIdx.x] += ae;
        s_f[threadIdx.x] += af;
        __syncthreads();
    }
    const int64_t chunks_q = (nt + kBwdChunk - 1) / kBwdChunk;
    const int64_t n_fixed = (int64_t)bh * (n_sink_tiles + n_lm_chunks) * chunks_q;
    const int64_t n_full = s_f[1023];
    if (threadIdx.x == 0) {  // remainder lengths kBwdChunk-1 down to 1 follow the whole runs
        int64_t pos = n_fixed + n_full;
        for (int r = kBwdChunk - 1; r >= 1; --r) {
            s_cursor[r] = pos;
            pos += s_rem[r];
        }
        s_cursor[0] = pos;  // total
    }
    __syncthreads();
    int64_t e0 = s_e[threadIdx.x] - se, u0 = n_fixed + s_f[threadIdx.x] - sf;
    for (int64_t x = b0; x < b1; ++x) {
        const int c = rev_cnt[x];
        fill[x] = (int32_t)e0;
        const int h = (int)(x / nt), j = (int)(x % nt);
        for (int q = 0; (q + 1) * kBwdChunk <= c; ++q) {
            if (u0 >= units_cap) {
                sa_flag_error(SA_ERR_BAD_LIST);
                break;
            }
            units[u0++] = make_int4(h, j, (int32_t)(e0 + q * kBwdChunk), (int32_t)(e0 + (q + 1) * kBwdChunk));
        }
        const int r = c % kBwdChunk;
        if (r) {
            const int64_t slot = (int64_t)atomicAdd(reinterpret_cast<unsigned long long*>(&s_cursor[r]), 1ull);
            if (slot >= units_cap)
                sa_flag_error(SA_ERR_BAD_LIST);
            else
                units[slot] = make_int4(h, j, (int32_t)(e0 + c - r), (int32_t)(e0 + c));
        }
        e0 += c;
    }
    for (int64_t f = threadIdx.x; f < n_fixed && f < units_cap; f += 1024) {
        const int64_t per_head = (n_sink_tiles + n_lm_chunks) * chunks_q;
        const int h = (int)(f / per_head);
        const int64_t r = f % per_head;
        const int it = (int)(r / chunks_q), q = (int)(r % chunks_q);
        const int kind = it < n_sink_tiles ? 1 : 2;
        const int item = it < n_sink_tiles ? it : it - n_sink_tiles;
        units[f] = make_int4(h, (kind << 24) | item, q * kBwdChunk, min(nt, (q + 1) * kBwdChunk));
    }
    if (threadIdx.x == 1023) *n_units = (int32_t)min(units_cap, s_cursor[0]);
}

__global__ void bwd_fill_lists_kernel(const int32_t* kept_idx, const int32_t* kept_cnt, int32_t max_kept,
                                      int32_t bh, int32_t nt, int32_t* fill, int32_t* rev) {
    const int64_t total = (int64_t)bh * nt * max_kept;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t li = e / max_kept;
        const int n = (int)(e % max_kept);
        const int cnt = min(max(__ldg(kept_cnt + li), 0), max_kept);
        if (n >= cnt) continue;
        const int j = __ldg(kept_idx + e);
        if (j < 0 || j >= nt) continue;
        const int64_t h = li / nt;
        const int pos = atomicAdd(fill + h * nt + j, 1);
        rev[pos] = (int32_t)(li - h * nt);
    }
}

// dK, dV in bf16: the fp32 accumulators plus, in landmark mode, 1/c_j of the landmark
// gradient of the row's tile on every non-sink row.  Eight dims per thread.
__global__ void __launch_bounds__(256) bwd_finalize_kernel(const float* dk32, const float* dv32, const float* dkbar,
                                                           const float* dvbar, __nv_bfloat16* dk, __nv_bfloat16* dv,
                                                           int32_t bh, int32_t L, int32_t tokens, int32_t tpf,
                                                           int32_t n_sink, int32_t ntp) {
    const int64_t total = (int64_t)bh * L * 8;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = e >> 3;  // h * L + t
        const int part = (int)(e & 7);
        const float4* k4 = reinterpret_cast<const float4*>(dk32 + row * 64) + 2 * part;
        const float4* v4 = reinterpret_cast<const float4*>(dv32 + row * 64) + 2 * part;
        float4 ka = k4[0], kb = k4[1], va = v4[0], vb = v4[1];
        if (dkbar) {
            const int64_t h = row / L;
            const int tt = (int)(row - h * L);
            const int f = tt / tokens, n = tt - f * tokens;
            if (n >= n_sink) {
                const int slot = n >> 7;
                const int n0 = slot * 128;
                const int c = min(128, tokens - n0) - max(0, n_sink - n0);
                const float w = 1.0f / (float)c;
                const int64_t lr = (h * ntp + (int64_t)f * tpf + slot) * 64;
                const float4* lk4 = reinterpret_cast<const float4*>(dkbar + lr) + 2 * part;
                const float4* lv4 = reinterpret_cast<const float4*>(dvbar + lr) + 2 * part;
                const float4 la = lk4[0], lb = lk4[1], ma = lv4[0], mb = lv4[1];
                ka = make_float4(fmaf(la.x, w, ka.x), fmaf(la.y, w, ka.y), fmaf(la.z, w, ka.z), fmaf(la.w, w, ka.w));
                kb = make_float4(fmaf(lb.x, w, kb.x), fmaf(lb.y, w, kb.y), fmaf(lb.z, w, kb.z), fmaf(lb.w, w, kb.w));
                va = make_float4(fmaf(ma.x, w, va.x), fmaf(ma.y, w, va.y), fmaf(ma.z, w, va.z), fmaf(ma.w, w, va.w));
                vb = make_float4(fmaf(mb.x, w, vb.x), fmaf(mb.y, w, vb.y), fmaf(mb.z, w, vb.z), fmaf(mb.w, w, vb.w));
            }
        }
        uint4 ko, vo;
        ko.x = pack_bf16x2(ka.x, ka.y);
        ko.y = pack_bf16x2(ka.z, ka.w);
        ko.z = pack_bf16x2(kb.x, kb.y);
        ko.w = pack_bf16x2(kb.z, kb.w);
        vo.x = pack_bf16x2(va.x, va.y);
        vo.y = pack_bf16x2(va.z, va.w);
        vo.z = pack_bf16x2(vb.x, vb.y);
        vo.w = pack_bf16x2(vb.z, vb.w);
        reinterpret_cast<uint4*>(dk + row * 64)[part] = ko;
        reinterpret_cast<uint4*>(dv + row * 64)[part] = vo;
    }
}
