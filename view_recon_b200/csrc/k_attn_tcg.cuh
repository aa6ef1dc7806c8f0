// Step 4 on the 5th-generation tensor cores for the shapes the bf16 / tile-128 kernel
// (k_attn_tc.cuh) does not take: f32 inputs (kind::tf32 products: f32 operands rounded to tf32,
// f32 accumulation) with tile 64 or 128, and bf16 inputs with tile 64 ("Zebra3D" abstract:
// tile-sparse attention with landmark summaries; "AVGGT" 2.B.2: special tokens kept, discarded
// columns as mean key/value pairs).  Same attended set, same online softmax, same bounded waits.
//
// Every item is 64 keys: a listed tile of 64 rows is one item, a listed tile of 128 rows two
// (its keys 0..63 and 64..127); then the sink segment in 64-row chunks, then (landmark mode)
// the landmark table in 64-tile chunks; dense mode walks 64-row key chunks.  A query tile is
// read as 128 rows whatever the tile (M = 128 products); with tile 64 the rows past the tile
// are computed and dropped.
// Warp roles (384 threads, one CTA per SM, no register split: 64-key items fit the launch's
// registers), as in the tile-128 kernel: warps 0/2 load (TMA,
// 128-byte swizzle, no multicast), warps 1/3 issue tcgen05.mma, warpgroup 1+x runs the softmax
// of slot x, thread r owning row r:
//   S_x = Q_x K^T   (M=128, N=64, K=64 in steps of 32 bytes: 16 bf16 or 8 tf32 elements)
//   O_x += P_x V    (M=128, N=64, K=64 keys; P read from TMEM, V^T tiles K-major)
// A row of 64 elements is one 128-byte swizzle atom in bf16 and two in f32, so an f32 tile is
// two boxes side by side ([rows][32] each) and the K steps switch atoms half way.
// TMEM per slot: S 64 columns, P 64 (f32) or 32 (bf16 pairs), O 64: at most 384 of 512.
#pragma once
#include "k_attn_tc.cuh"

struct __align__(64) TcgArgs {
    CUtensorMap tm_q;            // [bh*L][64] E, box inner x 128 rows
    CUtensorMap tm_k, tm_sk, tm_lk;    // keys, sink keys, landmark keys: box inner x 64 rows
    CUtensorMap tm_vt, tm_svt, tm_lvt; // transposed V items [items*64][64] E, box inner x 64 rows
    const int32_t* kept_idx;
    const int32_t* kept_cnt;
    const float* lbias2;  // [ntp] log2(c_j) or -inf
    void* o;
    float* lse;
    int32_t max_kept;
    int32_t frames, tokens, tile, n_sink, tpf, nt, L, ntp;
    int32_t sub;          // items per listed tile (tile / 64)
    int32_t n_vt;         // transposed V items per head
    int32_t n_sink_rows, n_sink_items, n_lm_items;
    int32_t dense, landmark;
    int32_t q_per_head, total_items;
    float scale_log2;
};

namespace tcg {

// f32 -> the nearest tf32 value (ties away from zero), kept in an f32 container.  The tensor
// cores read only the top 19 bits of an f32 operand, i.e. they truncate; operands rounded first
// carry half the error and no bias.
__device__ __forceinline__ float tf32_rn(float x) {
    uint32_t y;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
    return __uint_as_float(y);
}

template <bool F32>
struct Cfg {
    static constexpr int kElem = F32 ? 4 : 2;
    static constexpr int kAtoms = F32 ? 2 : 1;              // 128-byte atoms per 64-element row
    static constexpr int kQBytes = 128 * 64 * kElem;        // 128 rows
    static constexpr int kKBytes = 64 * 64 * kElem;         // 64 keys
    static constexpr int kVBytes = 64 * 64 * kElem;         // 64 dims x 64 keys
    static constexpr int kStageBytes = kKBytes + kVBytes;
    static constexpr int kStages = F32 ? 2 : 4;
    static constexpr int kKSteps = F32 ? 8 : 4;             // 32-byte K steps over 64 elements
    static constexpr int kPCols = F32 ? 64 : 32;            // P columns in TMEM
    // instruction descriptor: D f32; A/B bf16 (1) or tf32 (2); K-major A and B; N/8; M/16
    static constexpr uint32_t kFmt = F32 ? 2u : 1u;
    static constexpr uint32_t kIdesc = (1u << 4) | (kFmt << 7) | (kFmt << 10) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
    static constexpr int kThreads = 384;
    static constexpr int kQ = 0;
    static constexpr int kKV = 2 * kQBytes;
    static constexpr int kBars = kKV + 2 * kStages * kStageBytes;
    static constexpr int kBarsPerSlot = 6 + 2 * kStages;
    static constexpr int kMisc = kBars + 8 * kBarsPerSlot * 2;
    static constexpr int kEnd = kMisc + 16;
    static constexpr uint32_t colS(int x) { return x * 64; }
    static constexpr uint32_t colP(int x) { return 128 + x * 64; }
    static constexpr uint32_t colO(int x) { return 256 + x * 64; }
    static size_t smem_bytes() { return 1024 + kEnd; }
};

struct Item {
    int kind;      // 0 = key rows of a listed tile, 1 = sink chunk, 2 = landmark chunk, -1 = skipped
    int32_t krow;  // first row in the key tensor map
    int32_t vrow;  // first row in the transposed-V tensor map
    int lo, hi;    // valid key columns [lo, hi) of the 64
    int chunk;     // landmark chunk index
};

struct Slot {
    bool active;
    int h, i;
    int32_t qrow;
    int nq;
    int cnt;       // listed tiles
    int n_listed;  // items of listed tiles (cnt * sub)
    const int32_t* list;
    int n_items;
};

__device__ __forceinline__ Slot make_slot(const TcgArgs& a, int item) {
    Slot s;
    s.active = item < a.total_items;
    s.h = s.active ? item / a.q_per_head : 0;
    s.i = s.active ? item % a.q_per_head : 0;
    s.list = nullptr;
    s.cnt = 0;
    s.n_listed = 0;
    if (a.dense) {
        s.qrow = s.h * a.L + s.i * a.tile;
        s.nq = min(a.tile, a.L - s.i * a.tile);
        s.n_items = s.active ? (a.L + 63) / 64 : 0;
    } else {
        const int f = s.i / a.tpf, slot = s.i % a.tpf;
        s.qrow = s.h * a.L + f * a.tokens + slot * a.tile;
        s.nq = min(a.tile, a.tokens - slot * a.tile);
        if (s.active) {
            const int64_t li = (int64_t)s.h * a.nt + s.i;
            s.cnt = max(0, min(a.kept_cnt[li], a.max_kept));
            s.list = a.kept_idx + li * a.max_kept;
        }
        s.n_listed = s.cnt * a.sub;
        s.n_items = s.active ? s.n_listed + a.n_sink_items + (a.landmark ? a.n_lm_items : 0) : 0;
    }
    return s;
}

// Item n of slot s; j is the tile listed at position n / sub when n < s.n_listed.
__device__ __forceinline__ Item get_item(const TcgArgs& a, const Slot& s, int n, int j) {
    Item it;
    it.chunk = 0;
    if (a.dense) {
        it.kind = 0;
        it.krow = s.h * a.L + n * 64;
        it.vrow = (s.h * a.n_vt + n) * 64;
        it.lo = 0;
        it.hi = min(64, a.L - n * 64);
        return it;
    }
    if (n < s.n_listed) {
        const int half = n % a.sub;
        if (j < 0 || j >= a.nt) {
            it.kind = -1;
            it.krow = s.h * a.L;
            it.vrow = s.h * a.n_vt * 64;
            it.lo = it.hi = 0;
            return it;
        }
        const int f = j / a.tpf, slot = j - f * a.tpf;
        const int n0 = slot * a.tile + half * 64;
        const int nk = max(0, min(64, a.tokens - n0));
        it.kind = 0;
        it.krow = s.h * a.L + f * a.tokens + n0;
        it.vrow = (s.h * a.n_vt + j * a.sub + half) * 64;
        it.lo = min(nk, max(0, a.n_sink - n0));
        it.hi = nk;
        return it;
    }
    n -= s.n_listed;
    if (n < a.n_sink_items) {
        it.kind = 1;
        it.krow = s.h * a.n_sink_rows + n * 64;
        it.vrow = (s.h * a.n_sink_items + n) * 64;
        it.lo = 0;
        it.hi = min(64, a.n_sink_rows - n * 64);
        return it;
    }
    n -= a.n_sink_items;
    it.kind = 2;
    it.krow = s.h * a.ntp + n * 64;
    it.vrow = (s.h * a.n_lm_items + n) * 64;
    it.lo = 0;
    it.hi = 64;
    it.chunk = n;
    return it;
}

__device__ __forceinline__ int list_entry(const TcgArgs& a, const Slot& s, int n) {
    return (!a.dense && n < s.n_listed) ? __ldg(s.list + n / a.sub) : 0;
}

}  // namespace tcg

template <bool F32>
__global__ void __launch_bounds__(384, 1) attn_tcg_kernel(const __grid_constant__ TcgArgs a) {
    using C = tcg::Cfg<F32>;
    constexpr int STAGES = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(smem + C::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool is_softmax = warp >= 4;
    const int x = is_softmax ? (warp - 4) >> 2 : (warp >> 1);
    uint8_t* sQ = smem + C::kQ + x * C::kQBytes;
    uint8_t* sKV = smem + C::kKV + x * STAGES * C::kStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBars) + x * C::kBarsPerSlot;
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;
    uint64_t* kv_empty = kv_full + STAGES;
    uint64_t* s_full = kv_empty + STAGES;
    uint64_t* s_free = s_full + 1;
    uint64_t* p_full = s_free + 1;
    uint64_t* pv_done = p_full + 1;
    uint64_t* drain_bar = pv_done + 1;

    if (threadIdx.x == 0) {
        uint64_t* all = reinterpret_cast<uint64_t*>(smem + C::kBars);
        for (int y = 0; y < 2; ++y) {
            uint64_t* b = all + y * C::kBarsPerSlot;
            mbar_init(&b[0], 1);
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&b[1 + s], 1);
                mbar_init(&b[1 + STAGES + s], 1);
            }
            mbar_init(&b[1 + 2 * STAGES], 1);    // s_full
            mbar_init(&b[2 + 2 * STAGES], 128);  // s_free
            mbar_init(&b[3 + 2 * STAGES], 128);  // p_full
            mbar_init(&b[4 + 2 * STAGES], 1);    // pv_done
            mbar_init(&b[5 + 2 * STAGES], 1);    // drain
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if ((warp == 0 || warp == 2) && lane == 0) {
        tma_prefetch_desc(&a.tm_q);
        tma_prefetch_desc(&a.tm_k);
        tma_prefetch_desc(&a.tm_vt);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    const tcg::Slot sl = tcg::make_slot(a, blockIdx.x * 2 + x);

    if (!is_softmax) {
        const int n_items = sl.n_items;
        if ((warp & 1) == 0) {
            // ------------------------------------------------------------------ TMA producer
            const bool leader = tc::elect_one();
            uint32_t issued_mask = 0, phase_mask = 0;
            bool ok = true;
            if (n_items > 0 && leader) {
                mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
                for (int at = 0; at < C::kAtoms; ++at)
                    tma_load_2d(sQ + at * (C::kQBytes / C::kAtoms), &a.tm_q, q_full, at * (128 / C::kElem), sl.qrow);
            }
            for (int n = 0; n < n_items; ++n) {
                const uint32_t s = n % STAGES, ph = (n / STAGES) & 1u;
                if (!mbar_wait_warp(&kv_empty[s], ph ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                if (leader) {
                    const tcg::Item it = tcg::get_item(a, sl, n, tcg::list_entry(a, sl, n));
                    const CUtensorMap* mk = it.kind == 1 ? &a.tm_sk : (it.kind == 2 ? &a.tm_lk : &a.tm_k);
                    const CUtensorMap* mv = it.kind == 1 ? &a.tm_svt : (it.kind == 2 ? &a.tm_lvt : &a.tm_vt);
                    uint8_t* dk = sKV + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&kv_full[s], C::kStageBytes);
#pragma unroll
                    for (int at = 0; at < C::kAtoms; ++at) {
                        tma_load_2d(dk + at * (C::kKBytes / C::kAtoms), mk, &kv_full[s], at * (128 / C::kElem), it.krow);
                        tma_load_2d(dk + C::kKBytes + at * (C::kVBytes / C::kAtoms), mv, &kv_full[s],
                                    at * (128 / C::kElem), it.vrow);
                    }
                }
                issued_mask |= 1u << s;
                phase_mask = (phase_mask & ~(1u << s)) | (ph << s);
            }
            if (!ok) {
                for (int s = 0; s < STAGES; ++s)
                    if ((issued_mask >> s) & 1u) tc::drain_wait(&kv_full[s], (phase_mask >> s) & 1u);
                if (n_items > 0) tc::drain_wait(q_full, 0);
            }
        } else {
            // ------------------------------------------------------------------ MMA issuer
            const bool leader = tc::elect_one();
            bool ok = n_items == 0 || mbar_wait_warp(q_full, 0, abort_flag);
            bool any_mma = false;
            tc_fence_after();
            // a K step is 32 bytes (2 in descriptor units); an atom of 128 rows (Q) or 64 rows
            // (K, V^T) of 128 bytes follows the previous one
            const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(smem_u32(sKV), 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(smem_u32(sKV + C::kKBytes), 16, 1024);
            constexpr uint64_t kStageStep = C::kStageBytes >> 4;
            constexpr uint64_t kQAtom = (C::kQBytes / C::kAtoms) >> 4;
            constexpr uint64_t kKAtom = (C::kKBytes / C::kAtoms) >> 4;
            constexpr uint64_t kVAtom = (C::kVBytes / C::kAtoms) >> 4;
            constexpr int kPer = C::kKSteps / C::kAtoms;  // K steps per atom (4)
            for (int n = 0; n <= n_items && ok; ++n) {
                if (n < n_items) {
                    const uint32_t s = n % STAGES, ph = (n / STAGES) & 1u;
                    if (!mbar_wait_warp(&kv_full[s], ph, abort_flag)) { ok = false; break; }
                    if (n > 0 && !mbar_wait_warp(s_free, (n - 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    if (leader) {
                        const uint64_t dk = dk0 + s * kStageStep;
#pragma unroll
                        for (int kk = 0; kk < C::kKSteps; ++kk) {
                            const int at = kk / kPer, w = kk % kPer;
                            const uint64_t aq = dq + at * kQAtom + 2 * w;
                            const uint64_t bk = dk + at * kKAtom + 2 * w;
                            if constexpr (F32) {
                                asm volatile(
                                    "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                    "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(
                                        tmem + C::colS(x)),
                                    "l"(aq), "l"(bk), "r"(C::kIdesc), "r"((uint32_t)(kk > 0))
                                    : "memory");
                            } else {
                                umma_ss(tmem + C::colS(x), aq, bk, C::kIdesc, kk > 0);
                            }
                        }
                        umma_commit(s_full);
                    }
                    __syncwarp();
                    any_mma = true;
                }
                if (n >= 1) {
                    const int m = n - 1;
                    const uint32_t s = m % STAGES;
                    if (!mbar_wait_warp(p_full, m & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    if (leader) {
                        const uint64_t dv = dv0 + s * kStageStep;
#pragma unroll
                        for (int kk = 0; kk < C::kKSteps; ++kk) {
                            const int at = kk / kPer, w = kk % kPer;
                            const uint32_t pa = tmem + C::colP(x) + 8 * kk;
                            const uint64_t bv = dv + at * kVAtom + 2 * w;
                            const uint32_t acc = (m > 0 || kk > 0) ? 1u : 0u;
                            if constexpr (F32) {
                                asm volatile(
                                    "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                    "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(
                                        tmem + C::colO(x)),
                                    "r"(pa), "l"(bv), "r"(C::kIdesc), "r"(acc)
                                    : "memory");
                            } else {
                                umma_ts(tmem + C::colO(x), pa, bv, C::kIdesc, acc);
                            }
                        }
                        umma_commit(&kv_empty[s]);
                        umma_commit(pv_done);
                    }
                    __syncwarp();
                }
            }
            if (any_mma) {
                if (leader) umma_commit(drain_bar);
                __syncwarp();
                tc::drain_wait(drain_bar, 0);
            }
        }
    } else {
        // ---------------------------------------------------------------------- softmax group
        const int st = threadIdx.x - 128 - 128 * x;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + C::colS(x) + lane_off;
        const uint32_t tP = tmem + C::colP(x) + lane_off;
        const uint32_t tO = tmem + C::colO(x) + lane_off;
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        int lm_ptr = 0;
        for (int n = 0; n < sl.n_items; ++n) {
            const tcg::Item it = tcg::get_item(a, sl, n, tcg::list_entry(a, sl, n));
            if (it.kind < 0 && st == 0 && n % a.sub == 0) sa_flag_error(SA_ERR_BAD_LIST);
            if (!mbar_wait_warp(s_full, n & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[64];
            uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(sv + 0);
            uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(sv + 32);
            tmem_ld_32x32b_x32(tS + 0, s0);
            tmem_ld_32x32b_x32(tS + 32, s1);
            tmem_ld_wait(s0);
            reg_fence(s1);
            tc_fence_before();
            mbar_arrive(s_free);

            float mul = a.scale_log2;
            if (it.kind == 2) {
                uint32_t mw[2] = {0u, 0u};
                const int c_lo = it.chunk * 64;
                while (lm_ptr < sl.cnt) {
                    const int j = __ldg(sl.list + lm_ptr);
                    if (j >= c_lo + 64) break;
                    if (j >= c_lo) mw[(j - c_lo) >> 5] |= 1u << (j & 31);
                    ++lm_ptr;
                }
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const bool listed = (mw[c >> 5] >> (c & 31)) & 1u;
                    const float xv = fmaf(__uint_as_float(sv[c]), a.scale_log2, __ldg(a.lbias2 + c_lo + c));
                    sv[c] = __float_as_uint(listed ? -INFINITY : xv);
                }
                mul = 1.0f;
            } else if (it.lo > 0 || it.hi < 64) {
#pragma unroll
                for (int w2 = 0; w2 < 2; ++w2) {
                    const int b0 = min(max(it.lo - 32 * w2, 0), 32), b1 = min(max(it.hi - 32 * w2, 0), 32);
                    const uint32_t below_hi = b1 == 32 ? 0xFFFFFFFFu : ((1u << b1) - 1u);
                    const uint32_t below_lo = b0 == 32 ? 0xFFFFFFFFu : ((1u << b0) - 1u);
                    const uint32_t valid = below_hi & ~below_lo;
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        if (!((valid >> u) & 1u)) sv[32 * w2 + u] = __float_as_uint(-INFINITY);
                }
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; c += 2) mx = fmax3(mx, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
            mx *= mul;
            float m_new = m_run;
            if (mx > m_run + 8.0f) m_new = mx;
            const float m_use = m_new == -INFINITY ? 0.0f : m_new;
            const float alpha = ex2_approx(m_run - m_use);
            float acc0 = 0.0f, acc1 = 0.0f;
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(sv[c]), mul, -m_use));
                const float p1 = ex2_approx(fmaf(__uint_as_float(sv[c + 1]), mul, -m_use));
                acc0 += p0;
                acc1 += p1;
                if constexpr (F32) {
                    pk[c] = __float_as_uint(tcg::tf32_rn(p0));
                    pk[c + 1] = __float_as_uint(tcg::tf32_rn(p1));
                } else {
                    pk[c >> 1] = pack_bf16x2(p0, p1);
                }
            }
            l_run = l_run * alpha + (acc0 + acc1);
            m_run = m_new;
            if (n > 0) {
                if (!mbar_wait_warp(pv_done, (n - 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
                    for (int c = 0; c < 64; c += 16) {
                        uint32_t ov[16];
                        tmem_ld_32x32b_x16(tO + c, ov);
                        tmem_ld_wait16(ov);
#pragma unroll
                        for (int u = 0; u < 16; ++u) ov[u] = __float_as_uint(__uint_as_float(ov[u]) * alpha);
                        tmem_st_32x32b_x16(tO + c, ov);
                    }
                }
            }
            uint32_t(&pa)[32] = *reinterpret_cast<uint32_t(*)[32]>(pk + 0);
            tmem_st_32x32b_x32(tP + 0, pa);
            if constexpr (F32) {
                uint32_t(&pb)[32] = *reinterpret_cast<uint32_t(*)[32]>(pk + 32);
                tmem_st_32x32b_x32(tP + 32, pb);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        // ---- epilogue
        if (ok && sl.n_items > 0 && mbar_wait_warp(pv_done, (sl.n_items - 1) & 1, abort_flag)) {
            tc_fence_after();
            uint32_t o0[32], o1[32];
            tmem_ld_32x32b_x32(tO + 0, o0);
            tmem_ld_32x32b_x32(tO + 32, o1);
            tmem_ld_wait(o0);
            reg_fence(o1);
            if (r < sl.nq) {
                const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
                const int64_t row = (int64_t)sl.qrow + r;
                if constexpr (F32) {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.o) + row * 64);
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        dst[c4] = make_float4(__uint_as_float(o0[4 * c4]) * inv, __uint_as_float(o0[4 * c4 + 1]) * inv,
                                              __uint_as_float(o0[4 * c4 + 2]) * inv,
                                              __uint_as_float(o0[4 * c4 + 3]) * inv);
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4)
                        dst[8 + c4] = make_float4(__uint_as_float(o1[4 * c4]) * inv,
                                                  __uint_as_float(o1[4 * c4 + 1]) * inv,
                                                  __uint_as_float(o1[4 * c4 + 2]) * inv,
                                                  __uint_as_float(o1[4 * c4 + 3]) * inv);
                } else {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + row * 64);
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        dst[c8] = make_uint4(pack_bf16x2(__uint_as_float(o0[8 * c8]) * inv, __uint_as_float(o0[8 * c8 + 1]) * inv),
                                             pack_bf16x2(__uint_as_float(o0[8 * c8 + 2]) * inv, __uint_as_float(o0[8 * c8 + 3]) * inv),
                                             pack_bf16x2(__uint_as_float(o0[8 * c8 + 4]) * inv, __uint_as_float(o0[8 * c8 + 5]) * inv),
                                             pack_bf16x2(__uint_as_float(o0[8 * c8 + 6]) * inv, __uint_as_float(o0[8 * c8 + 7]) * inv));
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8)
                        dst[4 + c8] = make_uint4(pack_bf16x2(__uint_as_float(o1[8 * c8]) * inv, __uint_as_float(o1[8 * c8 + 1]) * inv),
                                                 pack_bf16x2(__uint_as_float(o1[8 * c8 + 2]) * inv, __uint_as_float(o1[8 * c8 + 3]) * inv),
                                                 pack_bf16x2(__uint_as_float(o1[8 * c8 + 4]) * inv, __uint_as_float(o1[8 * c8 + 5]) * inv),
                                                 pack_bf16x2(__uint_as_float(o1[8 * c8 + 6]) * inv, __uint_as_float(o1[8 * c8 + 7]) * inv));
                }
                if (a.lse) {
                    const float m_fin = m_run == -INFINITY ? 0.0f : m_run;
                    a.lse[row] = l_run > 0.0f ? (m_fin + log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
                }
            }
        } else if (ok && sl.active && sl.n_items == 0 && r < sl.nq) {
            const int64_t row = (int64_t)sl.qrow + r;
            if constexpr (F32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.o) + row * 64);
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) dst[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + row * 64);
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) dst[c8] = make_uint4(0, 0, 0, 0);
            }
            if (a.lse) a.lse[row] = -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------- operand preparation

// Element loads and stores in f32 arithmetic for the two input types.
template <typename T>
__device__ __forceinline__ float load_elem(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p, int64_t i) {
    return __ldg(p + i);
}
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void store_elem(T* p, int64_t i, float x);
template <>
__device__ __forceinline__ void store_elem<float>(float* p, int64_t i, float x) {
    p[i] = x;
}
template <>
__device__ __forceinline__ void store_elem<__nv_bfloat16>(__nv_bfloat16* p, int64_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}


// Transposed V items: item t of head h is the [64][64] block (dims x keys) of source rows
// [start, start + valid), zero past valid.  Frame mode: t = tile * sub + half of the frame-aligned
// tiling (start = h*L + f*N + slot*tile + half*64); flat mode: start = h*rows_per_head + t*64.
struct Vt64Args {
    const void* src;
    void* dst;  // [bh][items_per_head][64][64] E
    int32_t items_per_head;
    int32_t frame_mode;
    int32_t tokens, tpf, tile, sub, L;
    int32_t rows_per_head;
};

// An operand value in element type E: f32 operands go to the tf32 products rounded to nearest.
template <typename E>
__device__ __forceinline__ float tf32_or_same(float x);
template <>
__device__ __forceinline__ float tf32_or_same<float>(float x) { return tcg::tf32_rn(x); }
template <>
__device__ __forceinline__ float tf32_or_same<__nv_bfloat16>(float x) { return x; }

template <typename E>
__global__ void __launch_bounds__(256) vtile64_transpose_kernel(Vt64Args a) {
    __shared__ float s[64][65];
    const int t = blockIdx.x, h = blockIdx.y;
    int64_t start;
    int valid;
    if (a.frame_mode) {
        const int j = t / a.sub, half = t % a.sub;
        const int f = j / a.tpf, slot = j % a.tpf;
        const int n0 = slot * a.tile + half * 64;
        start = (int64_t)h * a.L + (int64_t)f * a.tokens + n0;
        valid = max(0, min(64, a.tokens - n0));
    } else {
        start = (int64_t)h * a.rows_per_head + (int64_t)t * 64;
        valid = min(64, a.rows_per_head - t * 64);
    }
    const E* src = static_cast<const E*>(a.src) + start * 64;
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
        const int key = i >> 6, d = i & 63;
        s[key][d] = key < valid ? load_elem<E>(src, (int64_t)key * 64 + d) : 0.0f;
    }
    __syncthreads();
    E* dst = static_cast<E*>(a.dst) + ((int64_t)h * a.items_per_head + t) * 64 * 64;
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
        const int d = i >> 6, key = i & 63;
        store_elem<E>(dst, (int64_t)d * 64 + key, tf32_or_same<E>(s[key][d]));
    }
}

// Q, K or sink-K rows rounded to tf32 (the f32 path's product operands); n elements.
__global__ void round_tf32_kernel(const float* src, float* dst, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = tcg::tf32_rn(__ldg(src + i));
}

// Landmark tables in element type E for 64-tile chunks: key means row-major [bh][ntp][64]
// (zero past nt), value means transposed per chunk [bh][ntp/64][64][64], and log2(c_j) per tile
// (-inf where c_j = 0 or j >= nt).
template <typename E>
__global__ void landmark64_prep_kernel(const float* k_pool, const float* v_pool, const int32_t* k_cnt, E* lk, E* lvt,
                                       float* lbias2, int32_t bh, int32_t nt, int32_t ntp) {
    const int64_t n1 = (int64_t)bh * ntp * 64;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n1;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t rowp = idx >> 6;  // h * ntp + j
        const int d = (int)(idx & 63);
        const int64_t h = rowp / ntp, j = rowp % ntp;
        store_elem<E>(lk, idx, tf32_or_same<E>(j < nt ? __ldg(k_pool + (h * nt + j) * 64 + d) : 0.0f));
        // transposed value chunk: element (chunk, d, key) of head h
        const int64_t ch = j / 64, key = j % 64;
        store_elem<E>(lvt, ((h * (ntp / 64) + ch) * 64 + d) * 64 + key,
                      tf32_or_same<E>(j < nt ? __ldg(v_pool + (h * nt + j) * 64 + d) : 0.0f));
        if (h == 0 && d == 0) {
            const int c = j < nt ? k_cnt[j] : 0;
            lbias2[j] = c > 0 ? log2f((float)c) : -INFINITY;
        }
    }
}
