// Step 4 on the 5th-generation tensor cores: block-sparse / dense attention forward for
// bf16, d = 64, tile = 128 ("Zebra3D" abstract: tile-sparse attention with landmark
// summaries; "AVGGT" 2.B.2: special tokens kept, discarded columns as mean K/V pairs).
//
// One CTA owns NSLOT query tiles ("slots"); each slot walks its own item list:
//   sparse: the listed key tiles, then the sink segment in 128-row chunks, then (landmark
//           mode) every 128-tile chunk of the landmark table with listed tiles masked out;
//   dense:  every 128-row key tile of the head.
// Warp roles (NSLOT = 2 -> 320 threads, one CTA per SM):
//   warp 0      TMA producer: Q tiles, then the K/V tile of each item into a STAGES-deep
//               shared-memory ring (128-byte swizzle, gathered by tile index);
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer:
//                 S_x = Q_x K^T      (M=128, N=128, K=64; both operands K-major in smem)
//                 O_x += P_x V       (M=128, N=64,  K=128; P from TMEM, V MN-major in smem);
//   warps 2..   one 128-thread softmax group per slot; thread r owns row r of its slot:
//               tcgen05.ld of S, masking, base-2 online softmax with a lazy max (the
//               accumulator is rescaled only when the row max grows by more than 2^8),
//               P written back to TMEM as bf16, O rescale in TMEM, final normalisation.
// TMEM columns per slot: S 128 (f32), P 64 (bf16 pairs), O 64 (f32).
// Every wait is bounded (g_sa_wait_limit_ns): a wait that runs out records SA_ERR_TIMEOUT,
// raises the CTA abort flag, every role drains what it has in flight and the CTA exits.
// No TMA multicast and no clusters are used.
#pragma once
#include "sa_device.cuh"

struct __align__(64) TcArgs {
    CUtensorMap tm_q, tm_k, tm_v;    // [bh*L][64] bf16, box 64 x 128
    CUtensorMap tm_sk, tm_sv;        // [bh*S*n_sink][64] sink segment
    CUtensorMap tm_lk, tm_lv;        // [bh*ntp][64] landmark tables
    const int32_t* kept_idx;
    const int32_t* kept_cnt;
    const float* lbias2;             // [ntp] log2(c_j) or -inf
    __nv_bfloat16* o;
    float* lse;
    int32_t max_kept;
    int32_t frames, tokens, n_sink, tpf, nt, L, ntp;
    int32_t n_sink_rows, n_sink_tiles, n_lm_chunks;
    int32_t dense, landmark;
    int32_t q_per_head, total_items;
    float scale_log2;
};

namespace tc {

constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 64, 1);

struct Item {
    int kind;     // 0 = key tile, 1 = sink chunk, 2 = landmark chunk, -1 = skipped
    int32_t row;  // first row in the item's tensor map
    int lo, hi;   // valid key columns [lo, hi)
    int chunk;    // landmark chunk index
};

struct Slot {
    bool active;
    int h, i;
    int32_t qrow;  // first row of the query tile in tm_q
    int nq;        // valid query rows
    int cnt;       // listed tiles
    const int32_t* list;
    int n_items;
};

__device__ __forceinline__ Slot make_slot(const TcArgs& a, int item) {
    Slot s;
    s.active = item < a.total_items;
    s.h = s.active ? item / a.q_per_head : 0;
    s.i = s.active ? item % a.q_per_head : 0;
    s.list = nullptr;
    s.cnt = 0;
    if (a.dense) {
        s.qrow = s.h * a.L + s.i * 128;
        s.nq = min(128, a.L - s.i * 128);
        s.n_items = s.active ? (a.L + 127) / 128 : 0;
    } else {
        const int f = s.i / a.tpf, slot = s.i % a.tpf;
        s.qrow = s.h * a.L + f * a.tokens + slot * 128;
        s.nq = min(128, a.tokens - slot * 128);
        if (s.active) {
            const int64_t li = (int64_t)s.h * a.nt + s.i;
            s.cnt = max(0, min(a.kept_cnt[li], a.max_kept));
            s.list = a.kept_idx + li * a.max_kept;
        }
        s.n_items = s.active ? s.cnt + a.n_sink_tiles + (a.landmark ? a.n_lm_chunks : 0) : 0;
    }
    return s;
}

__device__ __forceinline__ Item get_item(const TcArgs& a, const Slot& s, int n) {
    Item it;
    it.chunk = 0;
    if (a.dense) {
        it.kind = 0;
        it.row = s.h * a.L + n * 128;
        it.lo = 0;
        it.hi = min(128, a.L - n * 128);
        return it;
    }
    if (n < s.cnt) {
        const int j = __ldg(s.list + n);
        if (j < 0 || j >= a.nt) {
            it.kind = -1;
            it.row = s.h * a.L;
            it.lo = it.hi = 0;
            return it;
        }
        const int f = j / a.tpf, slot = j % a.tpf;
        const int n0 = slot * 128;
        const int nk = min(128, a.tokens - n0);
        it.kind = 0;
        it.row = s.h * a.L + f * a.tokens + n0;
        it.lo = min(nk, max(0, a.n_sink - n0));
        it.hi = nk;
        return it;
    }
    n -= s.cnt;
    if (n < a.n_sink_tiles) {
        it.kind = 1;
        it.row = s.h * a.n_sink_rows + n * 128;
        it.lo = 0;
        it.hi = min(128, a.n_sink_rows - n * 128);
        return it;
    }
    n -= a.n_sink_tiles;
    it.kind = 2;
    it.row = s.h * a.ntp + n * 128;
    it.lo = 0;
    it.hi = 128;
    it.chunk = n;
    return it;
}

// Bounded wait that ignores the abort flag (used only to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = sa_globaltimer();
    const uint64_t limit = g_sa_wait_limit_ns;
    while (!mbar_test(bar, parity)) {
        if (sa_globaltimer() - t0 > limit) {
            sa_flag_error(SA_ERR_TIMEOUT);
            return;
        }
    }
}

}  // namespace tc

template <int NSLOT, int STAGES>
struct TcLayout {
    static constexpr int kThreads = 64 + 128 * NSLOT;
    static constexpr uint32_t kTmemCols = NSLOT == 1 ? 256 : 512;
    static constexpr int kQ = 0;
    static constexpr int kKV = NSLOT * tc::kTileBytes;
    static constexpr int kBars = kKV + STAGES * 2 * tc::kTileBytes;
    // q_full[N], kv_full[S], kv_empty[S], s_full[N], s_free[N], p_full[N], pv_done[N], drain[1]
    static constexpr int kNumBars = 5 * NSLOT + 2 * STAGES + 1;
    static constexpr int kMisc = kBars + 8 * kNumBars;  // tmem base (4 B), abort flag (4 B)
    static constexpr int kMask = (kMisc + 8 + 15) & ~15;
    static constexpr uint32_t colS(int x) { return x * 128; }
    static constexpr uint32_t colP(int x) { return NSLOT * 128 + x * 64; }
    static constexpr uint32_t colO(int x) { return NSLOT * 128 + NSLOT * 64 + x * 64; }
    static size_t smem_bytes(int mask_words) { return 1024 + kMask + (size_t)NSLOT * mask_words * 4; }
};

template <int NSLOT, int STAGES>
__global__ void __launch_bounds__(64 + 128 * NSLOT, 1) attn_tc_kernel(const __grid_constant__ TcArgs a) {
    using Lay = TcLayout<NSLOT, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + Lay::kQ;
    uint8_t* sKV = smem + Lay::kKV;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBars);
    uint64_t* q_full = bars;
    uint64_t* kv_full = q_full + NSLOT;
    uint64_t* kv_empty = kv_full + STAGES;
    uint64_t* s_full = kv_empty + STAGES;
    uint64_t* s_free = s_full + NSLOT;
    uint64_t* p_full = s_free + NSLOT;
    uint64_t* pv_done = p_full + NSLOT;
    uint64_t* drain_bar = pv_done + NSLOT;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);
    uint32_t* lmask = reinterpret_cast<uint32_t*>(smem + Lay::kMask);
    const int mask_words = a.landmark ? (a.nt + 31) / 32 : 0;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    tc::Slot slots[NSLOT];
#pragma unroll
    for (int x = 0; x < NSLOT; ++x) slots[x] = tc::make_slot(a, blockIdx.x * NSLOT + x);
    int max_items = 0;
#pragma unroll
    for (int x = 0; x < NSLOT; ++x) max_items = max(max_items, slots[x].n_items);

    if (threadIdx.x == 0) {
        for (int x = 0; x < NSLOT; ++x) {
            mbar_init(&q_full[x], 1);
            mbar_init(&s_full[x], 1);
            mbar_init(&s_free[x], 128);
            mbar_init(&p_full[x], 128);
            mbar_init(&pv_done[x], 1);
        }
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&a.tm_q);
        tma_prefetch_desc(&a.tm_k);
        tma_prefetch_desc(&a.tm_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, Lay::kTmemCols);
        tmem_relinquish();
    }
    // kept-tile bit masks for the landmark chunks
    const int sx = warp >= 2 ? (warp - 2) >> 2 : 0;
    const int st = threadIdx.x - 64 - 128 * sx;  // 0..127 inside a softmax group
    if (warp >= 2 && mask_words)
        for (int w = st; w < mask_words; w += 128) lmask[sx * mask_words + w] = 0u;
    __syncthreads();
    if (warp >= 2 && mask_words)
        for (int n = st; n < slots[sx].cnt; n += 128) {
            const int j = __ldg(slots[sx].list + n);
            if (j >= 0 && j < a.nt) atomicOr(&lmask[sx * mask_words + (j >> 5)], 1u << (j & 31));
        }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t issued_phase[STAGES];
            bool issued[STAGES];
#pragma unroll
            for (int s = 0; s < STAGES; ++s) issued[s] = false;
            bool ok = true;
            for (int x = 0; x < NSLOT; ++x)
                if (slots[x].active) {
                    mbar_arrive_expect_tx(&q_full[x], tc::kTileBytes);
                    tma_load_2d(sQ + x * tc::kTileBytes, &a.tm_q, &q_full[x], 0, slots[x].qrow);
                }
            uint32_t seq = 0;
            for (int n = 0; n < max_items && ok; ++n) {
                for (int x = 0; x < NSLOT; ++x) {
                    if (n >= slots[x].n_items) continue;
                    const uint32_t s = seq % STAGES, ph = (seq / STAGES) & 1u;
                    ++seq;
                    if (!mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const tc::Item it = tc::get_item(a, slots[x], n);
                    const CUtensorMap* mk = it.kind == 1 ? &a.tm_sk : (it.kind == 2 ? &a.tm_lk : &a.tm_k);
                    const CUtensorMap* mv = it.kind == 1 ? &a.tm_sv : (it.kind == 2 ? &a.tm_lv : &a.tm_v);
                    uint8_t* dk = sKV + s * 2 * tc::kTileBytes;
                    mbar_arrive_expect_tx(&kv_full[s], 2 * tc::kTileBytes);
                    tma_load_2d(dk, mk, &kv_full[s], 0, it.row);
                    tma_load_2d(dk + tc::kTileBytes, mv, &kv_full[s], 0, it.row);
                    issued[s] = true;
                    issued_phase[s] = ph;
                }
            }
            if (!ok) {  // let every copy this thread started land before the CTA exits
                for (int s = 0; s < STAGES; ++s)
                    if (issued[s]) tc::drain_wait(&kv_full[s], issued_phase[s]);
                for (int x = 0; x < NSLOT; ++x)
                    if (slots[x].active) tc::drain_wait(&q_full[x], 0);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            bool any_mma = false;
            for (int x = 0; x < NSLOT && ok; ++x)
                if (slots[x].active) ok = mbar_wait(&q_full[x], 0, abort_flag);
            tc_fence_after();
            uint32_t seq = 0;
            int stage_of[NSLOT][2];
            for (int n = 0; n <= max_items && ok; ++n) {
                for (int x = 0; x < NSLOT && ok; ++x) {
                    if (n < slots[x].n_items) {
                        const uint32_t s = seq % STAGES, ph = (seq / STAGES) & 1u;
                        ++seq;
                        if (!mbar_wait(&kv_full[s], ph, abort_flag)) { ok = false; break; }
                        if (n > 0 && !mbar_wait(&s_free[x], (n - 1) & 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t qa = smem_u32(sQ + x * tc::kTileBytes);
                        const uint32_t ka = smem_u32(sKV + s * 2 * tc::kTileBytes);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_ss(tmem + Lay::colS(x), smem_desc_sw128(qa + 32 * kk, 16, 1024),
                                    smem_desc_sw128(ka + 32 * kk, 16, 1024), tc::kIdescS, kk > 0);
                        umma_commit(&s_full[x]);
                        any_mma = true;
                        stage_of[x][n & 1] = s;
                    }
                    if (n >= 1 && n <= slots[x].n_items) {
                        const int m = n - 1;
                        if (!mbar_wait(&p_full[x], m & 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const int s = stage_of[x][m & 1];
                        const uint32_t va = smem_u32(sKV + s * 2 * tc::kTileBytes + tc::kTileBytes);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_ts(tmem + Lay::colO(x), tmem + Lay::colP(x) + 8 * kk,
                                    smem_desc_sw128(va + 2048 * kk, 1024, 1024), tc::kIdescPV,
                                    (m > 0 || kk > 0));
                        umma_commit(&kv_empty[s]);
                        umma_commit(&pv_done[x]);
                    }
                }
            }
            // every MMA (and its commits) must be finished before TMEM is released
            if (any_mma) {
                umma_commit(drain_bar);
                tc::drain_wait(drain_bar, 0);
            }
        }
    } else {
        // ------------------------------------------------------------------ softmax group
        const int x = sx;
        const tc::Slot& sl = slots[x];
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + Lay::colS(x) + lane_off;
        const uint32_t tP = tmem + Lay::colP(x) + lane_off;
        const uint32_t tO = tmem + Lay::colO(x) + lane_off;
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int n = 0; n < sl.n_items; ++n) {
            const tc::Item it = tc::get_item(a, sl, n);
            if (!mbar_wait_warp(&s_full[x], n & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t s0[32], s1[32], s2[32], s3[32];
            tmem_ld_32x32b_x32(tS + 0, s0);
            tmem_ld_32x32b_x32(tS + 32, s1);
            tmem_ld_32x32b_x32(tS + 64, s2);
            tmem_ld_32x32b_x32(tS + 96, s3);
            tmem_ld_wait(s0);
            reg_fence(s1);
            reg_fence(s2);
            reg_fence(s3);
            tc_fence_before();
            mbar_arrive(&s_free[x]);

            // logits in base-2 units, masked columns at -inf
            float xs[128];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                xs[c] = __uint_as_float(s0[c]) * a.scale_log2;
                xs[32 + c] = __uint_as_float(s1[c]) * a.scale_log2;
                xs[64 + c] = __uint_as_float(s2[c]) * a.scale_log2;
                xs[96 + c] = __uint_as_float(s3[c]) * a.scale_log2;
            }
            if (it.kind == 2) {
                const float4* bp = reinterpret_cast<const float4*>(a.lbias2 + it.chunk * 128);
                const uint32_t* mw = lmask + x * mask_words + it.chunk * 4;
#pragma unroll
                for (int c4 = 0; c4 < 32; ++c4) {
                    const float4 b = __ldg(bp + c4);
                    const int j = it.chunk * 128 + 4 * c4;
                    const uint32_t word = (j >> 5) < mask_words ? mw[c4 >> 3] : 0u;
                    const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const bool listed = (word >> ((4 * c4 + u) & 31)) & 1u;
                        xs[4 * c4 + u] = listed ? -INFINITY : xs[4 * c4 + u] + bb[u];
                    }
                }
            } else {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c < it.lo || c >= it.hi) xs[c] = -INFINITY;
            }
            float mx = xs[0];
#pragma unroll
            for (int c = 1; c < 128; ++c) mx = fmaxf(mx, xs[c]);
            float m_new = m_run;
            if (mx > m_run + 8.0f) m_new = mx;  // lazy max: rescale only on growth beyond 2^8
            const float m_use = m_new == -INFINITY ? 0.0f : m_new;
            const float alpha = ex2_approx(m_run - m_use);  // 0 on the first item
            float sum = 0.0f;
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float p0 = ex2_approx(xs[2 * c] - m_use);
                const float p1 = ex2_approx(xs[2 * c + 1] - m_use);
                sum += p0 + p1;
                pk[c] = pack_bf16x2(p0, p1);
            }
            if (n > 0) {
                // the previous P.V product must be done before O is rescaled or P overwritten
                if (!mbar_wait_warp(&pv_done[x], (n - 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.0f)) {
                    uint32_t o0[32], o1[32];
                    tmem_ld_32x32b_x32(tO + 0, o0);
                    tmem_ld_32x32b_x32(tO + 32, o1);
                    tmem_ld_wait(o0);
                    reg_fence(o1);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        o0[c] = __float_as_uint(__uint_as_float(o0[c]) * alpha);
                        o1[c] = __float_as_uint(__uint_as_float(o1[c]) * alpha);
                    }
                    tmem_st_32x32b_x32(tO + 0, o0);
                    tmem_st_32x32b_x32(tO + 32, o1);
                }
            }
            l_run = l_run * alpha + sum;
            m_run = m_new;
            uint32_t pa[32], pb[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                pa[c] = pk[c];
                pb[c] = pk[32 + c];
            }
            tmem_st_32x32b_x32(tP + 0, pa);
            tmem_st_32x32b_x32(tP + 32, pb);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[x]);
        }
        // ---- epilogue: O / l, LSE, store valid rows
        if (ok && sl.n_items > 0 && mbar_wait_warp(&pv_done[x], (sl.n_items - 1) & 1, abort_flag)) {
            tc_fence_after();
            uint32_t o0[32], o1[32];
            tmem_ld_32x32b_x32(tO + 0, o0);
            tmem_ld_32x32b_x32(tO + 32, o1);
            tmem_ld_wait(o0);
            reg_fence(o1);
            if (r < sl.nq) {
                const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
                uint4* dst = reinterpret_cast<uint4*>(a.o + ((int64_t)sl.qrow + r) * 64);
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(o0[8 * c8 + 0]) * inv, __uint_as_float(o0[8 * c8 + 1]) * inv);
                    w.y = pack_bf16x2(__uint_as_float(o0[8 * c8 + 2]) * inv, __uint_as_float(o0[8 * c8 + 3]) * inv);
                    w.z = pack_bf16x2(__uint_as_float(o0[8 * c8 + 4]) * inv, __uint_as_float(o0[8 * c8 + 5]) * inv);
                    w.w = pack_bf16x2(__uint_as_float(o0[8 * c8 + 6]) * inv, __uint_as_float(o0[8 * c8 + 7]) * inv);
                    dst[c8] = w;
                }
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(o1[8 * c8 + 0]) * inv, __uint_as_float(o1[8 * c8 + 1]) * inv);
                    w.y = pack_bf16x2(__uint_as_float(o1[8 * c8 + 2]) * inv, __uint_as_float(o1[8 * c8 + 3]) * inv);
                    w.z = pack_bf16x2(__uint_as_float(o1[8 * c8 + 4]) * inv, __uint_as_float(o1[8 * c8 + 5]) * inv);
                    w.w = pack_bf16x2(__uint_as_float(o1[8 * c8 + 6]) * inv, __uint_as_float(o1[8 * c8 + 7]) * inv);
                    dst[4 + c8] = w;
                }
                if (a.lse) {
                    const float m_fin = m_run == -INFINITY ? 0.0f : m_run;
                    a.lse[(int64_t)sl.qrow + r] =
                        l_run > 0.0f ? (m_fin + log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
                }
            }
        }
        // report skipped list entries once per slot
        if (ok && st == 0 && !a.dense)
            for (int n = 0; n < sl.cnt; ++n) {
                const int j = __ldg(sl.list + n);
                if (j < 0 || j >= a.nt) {
                    sa_flag_error(SA_ERR_BAD_LIST);
                    break;
                }
            }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::kTmemCols);
    }
}
