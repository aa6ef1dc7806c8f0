// Step 4 on the 5th-generation tensor cores: block-sparse / dense attention forward for
// bf16, d = 64, tile = 128 ("Zebra3D" abstract: tile-sparse attention with landmark
// summaries; "AVGGT" 2.B.2: special tokens kept, discarded columns as mean K/V pairs).
//
// One CTA owns NSLOT = 2 query tiles ("slots"); each slot walks its own item list:
//   sparse: the listed key tiles, then the sink segment in 128-row chunks, then (landmark
//           mode) every 128-tile chunk of the landmark table with listed tiles masked out;
//   dense:  every 128-row key tile of the head.
// An item is a K tile ([128 keys][64] bf16, gathered by TMA straight from K) and the
// matching transposed V tile ([64][128 keys], prepared in the workspace, see
// k_attn_prep.cuh) so that both products read K-major shared-memory operands.
// The two slots are fully decoupled, so that one slot's exponentials fill the other's
// waits (TMEM round trips, barrier hand-offs) instead of running in lockstep with them:
// each has its own producer warp, its own MMA-issuing warp and its own STAGES-deep ring.
// Warp roles (384 threads, one CTA per SM):
//   warps 0, 2      TMA producers of slots 0, 1: the Q tile, then K + V^T of every item
//                   (128-byte swizzle);
//   warps 1, 3      tcgen05.mma issuers of slots 0, 1 (one elected lane; warp 1 also owns
//                   the TMEM allocation):
//                     S_x = Q_x K^T   (M=128, N=128, K=64; A and B K-major in shared memory),
//                     plus, for an item with key columns outside its valid range [lo, hi),
//                     S_x += 1 . bias^T (one K=16 step; bias -2^100 on those columns, 0
//                     elsewhere, written by the producer) so that the softmax needs no mask;
//                     O_x += P_x V    (M=128, N=64, K=128; P read from TMEM, V^T K-major);
//   warpgroup 1+x   the softmax group of slot x; thread r owns row r: tcgen05.ld of its 128
//                   scores, base-2 online softmax with a lazy max (O is rescaled
//                   only when the row max grows by more than 2^8), P written back to TMEM
//                   as bf16, O rescale in TMEM, final normalisation.
// TMEM columns per slot: S 128 (f32), P 64 (bf16 pairs), O 64 (f32): 512 in total.
// Every wait is bounded (g_sa_wait_limit_ns): a wait that runs out records SA_ERR_TIMEOUT,
// raises the CTA abort flag, every role drains what it has in flight and the CTA exits.
// No TMA multicast and no clusters are used.
#pragma once
#include "sa_device.cuh"

struct __align__(64) TcArgs {
    CUtensorMap tm_q, tm_k;     // [bh*L][64] bf16, box 64 x 128
    CUtensorMap tm_vt;          // [bh*n_vtiles*64][128] bf16 transposed V tiles, box 64 x 64
    CUtensorMap tm_sk, tm_svt;  // sink keys [bh*S*n_sink][64]; transposed sink V tiles
    CUtensorMap tm_lk, tm_lvt;  // landmark keys [bh*ntp][64]; transposed landmark V tiles
    const int32_t* kept_idx;
    const int32_t* kept_cnt;
    const float* lbias2;  // [ntp] log2(c_j) or -inf
    __nv_bfloat16* o;
    float* lse;
    int32_t max_kept;
    int32_t frames, tokens, n_sink, tpf, nt, L, ntp;
    int32_t Lk;        // dense: key rows per head (L, or the length of a compacted key sequence)
    int32_t n_vtiles;  // transposed V tiles per head (nt, or ceil(L/128) dense)
    int32_t n_sink_rows, n_sink_tiles, n_lm_chunks;
    int32_t dense, landmark;
    int32_t q_per_head, total_items;
    uint32_t tpf_magic;  // j / tpf == __umulhi(j, tpf_magic) for every tile index j < nt (tpf > 1)
    float scale_log2;
};

// Of every 8 column pairs of a score row, this many take their exponentials on the FMA pipe
// (exp2_poly2) and the rest on the MUFU (ex2.approx): sparse launches (no mask code in the
// softmax) and dense launches (masks in the softmax) were each timed with 0 to 3.
#ifndef SA_EXP2_FMA_PAIRS_PER8
#define SA_EXP2_FMA_PAIRS_PER8 1
#endif
#ifndef SA_EXP2_FMA_PAIRS_PER8_DENSE
#define SA_EXP2_FMA_PAIRS_PER8_DENSE 2
#endif

namespace tc {

constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 64, 0);  // V^T: K-major B

struct Item {
    int kind;      // 0 = key tile, 1 = sink chunk, 2 = landmark chunk, -1 = skipped
    int32_t krow;  // first row of the K tile in its tensor map
    int32_t vrow;  // first row of the V^T tile in its tensor map
    int lo, hi;    // valid key columns [lo, hi)
    int chunk;     // landmark chunk index
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
        s.n_items = s.active ? (a.Lk + 127) / 128 : 0;
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

__device__ __forceinline__ Item get_item_j(const TcArgs& a, const Slot& s, int n, int j);

// Item n of slot s, reading its list entry from global memory.
__device__ __forceinline__ Item get_item(const TcArgs& a, const Slot& s, int n) {
    const int j = (!a.dense && n < s.cnt) ? __ldg(s.list + n) : 0;
    return get_item_j(a, s, n, j);
}

// Item n of slot s; j is the list entry s.list[n] when n < s.cnt (see ListWindow).
__device__ __forceinline__ Item get_item_j(const TcArgs& a, const Slot& s, int n, int j) {
    Item it;
    it.chunk = 0;
    if (a.dense) {
        it.kind = 0;
        it.krow = s.h * a.Lk + n * 128;
        it.vrow = (s.h * a.n_vtiles + n) * 64;
        it.lo = 0;
        it.hi = min(128, a.Lk - n * 128);
        return it;
    }
    if (n < s.cnt) {
        if (j < 0 || j >= a.nt) {
            it.kind = -1;
            it.krow = s.h * a.L;
            it.vrow = s.h * a.n_vtiles * 64;
            it.lo = it.hi = 0;
            return it;
        }
        const int f = a.tpf == 1 ? j : (int)__umulhi((uint32_t)j, a.tpf_magic), slot = j - f * a.tpf;
        const int n0 = slot * 128;
        const int nk = min(128, a.tokens - n0);
        it.kind = 0;
        it.krow = s.h * a.L + f * a.tokens + n0;
        it.vrow = (s.h * a.n_vtiles + j) * 64;
        it.lo = min(nk, max(0, a.n_sink - n0));
        it.hi = nk;
        return it;
    }
    n -= s.cnt;
    if (n < a.n_sink_tiles) {
        it.kind = 1;
        it.krow = s.h * a.n_sink_rows + n * 128;
        it.vrow = (s.h * a.n_sink_tiles + n) * 64;
        it.lo = 0;
        it.hi = min(128, a.n_sink_rows - n * 128);
        return it;
    }
    n -= a.n_sink_tiles;
    it.kind = 2;
    it.krow = s.h * a.ntp + n * 128;
    it.vrow = (s.h * a.n_lm_chunks + n) * 64;
    it.lo = 0;
    it.hi = 128;
    it.chunk = n;
    return it;
}

// The slot's kept list, read 32 entries at a time: lane l holds entry 32w + l of the current
// window w and of the next one (loaded a whole window ahead, so no item waits for a global
// load); entry n is one warp shuffle.  All 32 lanes must call entry() for every n in order.
struct ListWindow {
    int32_t cur, next;
    __device__ __forceinline__ ListWindow(const TcArgs& a, const Slot& s, int lane) {
        const bool listed = !a.dense && s.cnt > 0;
        cur = (listed && lane < s.cnt) ? __ldg(s.list + lane) : 0;
        next = (listed && 32 + lane < s.cnt) ? __ldg(s.list + 32 + lane) : 0;
    }
    __device__ __forceinline__ int entry(const TcArgs& a, const Slot& s, int n, int lane) {
        if (a.dense || n >= s.cnt) return 0;  // uniform over the warp
        const int j = __shfl_sync(0xffffffffu, cur, n & 31);
        if ((n & 31) == 31) {
            cur = next;
            const int e = n + 33 + lane;
            next = e < s.cnt ? __ldg(s.list + e) : 0;
        }
        return j;
    }
};

// Bounded wait that ignores the abort flag (used only to drain in-flight work).  Copies and
// MMAs already issued complete in microseconds; the limit is at least 1 s whatever the
// caller's wait limit, so that a CTA never exits with work of its own still in flight.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = sa_globaltimer();
    const uint64_t limit = max(g_sa_wait_limit_ns, 1000000000ull);
    while (!mbar_test(bar, parity)) {
        if (sa_globaltimer() - t0 > limit) {
            sa_flag_error(SA_ERR_TIMEOUT);
            return;
        }
    }
}

__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

}  // namespace tc

template <int NSLOT, int STAGES, bool BIAS>
struct TcLayout {
    static constexpr int kThreads = 128 + 128 * NSLOT;
    static constexpr uint32_t kTmemCols = 512;
    // registers per thread after the split: warpgroup 0 gives, the softmax groups take (the
    // producer's bias writes want a few more control registers in sparse launches)
    static constexpr uint32_t kRegsControl = BIAS ? 48 : 40;
    static constexpr uint32_t kRegsSoftmax = BIAS ? 224 : 232;
    static constexpr uint32_t kRegsNeeded = 128 * kRegsControl + 128 * NSLOT * kRegsSoftmax;
    static constexpr int kQ = 0;
    static constexpr int kKV = NSLOT * tc::kTileBytes;                 // [slot][stage] K + V^T
    // BIAS: the mask operands, a tile of ones (A) and, at the four 16-column K steps of one
    // more tile, the column-bias operand (B) of each [slot][stage]
    static constexpr int kOnes = kKV + NSLOT * STAGES * 2 * tc::kTileBytes;
    static constexpr int kBias = kOnes + (BIAS ? tc::kTileBytes : 0);
    static constexpr int kBars = kBias + (BIAS ? tc::kTileBytes : 0);
    // per slot: q_full, kv_full[S], kv_empty[S], s_full, s_free, p_full, pv_done, drain
    static constexpr int kBarsPerSlot = 6 + 2 * STAGES;
    static constexpr int kMisc = kBars + 8 * kBarsPerSlot * NSLOT;  // tmem base, abort flag
    static constexpr int kMeta = kMisc + 16;  // [slot][stage] the item's {kind, lo, hi, chunk}
    static constexpr int kEnd = kMeta + NSLOT * STAGES * 16;
    static constexpr uint32_t colS(int x) { return x * 128; }
    static constexpr uint32_t colP(int x) { return NSLOT * 128 + x * 64; }
    static constexpr uint32_t colO(int x) { return NSLOT * 128 + NSLOT * 64 + x * 64; }
    static size_t smem_bytes() { return 1024 + kEnd; }
};

// LANDMARK: the call has landmark chunks (a.landmark): the producer also writes their bias
// (multiplicity terms, listed tiles masked); without them it carries no landmark code.
// BIAS: key columns outside an item's valid range are masked by the bias product on the tensor
// cores (the ring then has room for at most four stages); otherwise the softmax masks them.
template <int NSLOT, int STAGES, bool LANDMARK, bool BIAS>
__global__ void __launch_bounds__(128 + 128 * NSLOT, 1) attn_tc_kernel(const __grid_constant__ TcArgs a) {
    using Lay = TcLayout<NSLOT, STAGES, BIAS>;
    static_assert(BIAS || !LANDMARK, "landmark chunks take their bias through the bias product");
    static_assert(NSLOT == 2, "warp roles are laid out for two slots");
    static_assert(NSLOT * (128 + 64 + 64) <= 512, "TMEM columns");
    static_assert(!BIAS || NSLOT * STAGES <= 4, "one 16-column K step of the bias tile per ring stage");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool is_softmax = warp >= 4;
    // the slot this warp works for: control warps 0,1 -> slot 0, 2,3 -> slot 1
    const int x = is_softmax ? (warp - 4) >> 2 : (warp >> 1);
    uint8_t* sQ = smem + Lay::kQ + x * tc::kTileBytes;
    uint8_t* sKV = smem + Lay::kKV + x * STAGES * 2 * tc::kTileBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBars) + x * Lay::kBarsPerSlot;
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;
    uint64_t* kv_empty = kv_full + STAGES;
    uint64_t* s_full = kv_empty + STAGES;
    uint64_t* s_free = s_full + 1;
    uint64_t* p_full = s_free + 1;
    uint64_t* pv_done = p_full + 1;
    uint64_t* drain_bar = pv_done + 1;
    // each item's {kind, lo, hi, chunk}, written by the producer before it arms the stage's
    // kv_full barrier, whose completion the MMA issuer (and, masking in the softmax, the softmax)
    // observes before reading it
    int4* meta = reinterpret_cast<int4*>(smem + Lay::kMeta) + x * STAGES;

    if (threadIdx.x == 0) {
        uint64_t* all = reinterpret_cast<uint64_t*>(smem + Lay::kBars);
        for (int y = 0; y < NSLOT; ++y) {
            uint64_t* b = all + y * Lay::kBarsPerSlot;
            mbar_init(&b[0], 1);  // q_full
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&b[1 + s], 1);           // kv_full
                mbar_init(&b[1 + STAGES + s], 1);  // kv_empty
            }
            mbar_init(&b[1 + 2 * STAGES], 1);      // s_full
            mbar_init(&b[2 + 2 * STAGES], 128);    // s_free
            mbar_init(&b[3 + 2 * STAGES], 128);    // p_full
            mbar_init(&b[4 + 2 * STAGES], 1);      // pv_done
            mbar_init(&b[5 + 2 * STAGES], 1);      // drain
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (BIAS) {
        // every bf16 element of the ones tile is 1.0, so each of its 16-column K steps is the
        // all-ones A operand of the mask product, whatever the swizzle
        uint4* ones = reinterpret_cast<uint4*>(smem + Lay::kOnes);
        const uint4 v = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        for (int i = threadIdx.x; i < tc::kTileBytes / 16; i += Lay::kThreads) ones[i] = v;
        fence_proxy_async_smem();
    }
    if ((warp == 0 || warp == 2) && lane == 0) {
        tma_prefetch_desc(&a.tm_q);
        tma_prefetch_desc(&a.tm_k);
        tma_prefetch_desc(&a.tm_vt);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, Lay::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    const tc::Slot sl = tc::make_slot(a, blockIdx.x * NSLOT + x);

    if (!is_softmax) {
        setmaxnreg_dec<Lay::kRegsControl>();
        const int n_items = sl.n_items;
        if ((warp & 1) == 0) {
            // -------------------------------------------------------------- TMA producer (slot x)
            // The whole warp walks the loop (waits are per lane); one elected lane issues.
            const bool leader = tc::elect_one();
            uint32_t issued_mask = 0, phase_mask = 0;  // per ring stage: a load was issued / its parity
            bool ok = true;
            const bool withhold = g_sa_test_withhold != 0 && blockIdx.x == 0 && x == 0;
            if (n_items > 0 && leader && !withhold) {
                mbar_arrive_expect_tx(q_full, tc::kTileBytes);
                tma_load_2d(sQ, &a.tm_q, q_full, 0, sl.qrow);
            }
            tc::ListWindow win(a, sl, lane);
            int lm_ptr = 0;  // landmark chunks: list cursor (warp-uniform)
            for (int n = 0; n < n_items; ++n) {
                const uint32_t s = n % STAGES, ph = (n / STAGES) & 1u;
                if (!mbar_wait_warp(&kv_empty[s], ph ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                const int j_cur = win.entry(a, sl, n, lane);
                const tc::Item it = tc::get_item_j(a, sl, n, j_cur);
                const bool lm_item = LANDMARK && it.kind == 2;
                if (BIAS && (lm_item || it.lo > 0 || it.hi < 128)) {
                    // The item's column bias, B operand of one more product S += ones . bias^T
                    // (every element of the A tile is 1, so row r of the bias, key column r, adds
                    // the sum of its sixteen bf16 elements to column r of S).  The stage's K step q
                    // sits in the 16-byte chunks 2q, 2q + 1 of each 128-byte row, stored at
                    // chunk ^ (r & 7) (128-byte swizzle).
                    const int q = x * STAGES + (int)s;
                    uint8_t* bias = smem + Lay::kBias;
                    if (!lm_item) {
                        // key columns outside [lo, hi): sixteen elements of -2^96, so that S there
                        // becomes -2^100; zeros elsewhere leave S unchanged
                        for (int r = lane; r < 128; r += 32) {
                            const uint32_t w = (r < it.lo || r >= it.hi) ? 0xEF80EF80u : 0u;
                            const uint4 v = make_uint4(w, w, w, w);
                            *reinterpret_cast<uint4*>(bias + r * 128 + (((2 * q) ^ (r & 7)) << 4)) = v;
                            *reinterpret_cast<uint4*>(bias + r * 128 + (((2 * q + 1) ^ (r & 7)) << 4)) = v;
                        }
                    } else {
                        // landmark chunk: the listed tiles of the chunk (the next run of the
                        // ascending list, 32 entries per step) get -2^100, the others their
                        // multiplicity term log2(c_j) in units of S (divided by the base-2 scale),
                        // split into three bf16 parts so that their sum keeps f32 accuracy
                        const int c_lo = it.chunk * 128;
                        uint32_t mw[4] = {0u, 0u, 0u, 0u};
                        for (;;) {
                            const int e = lm_ptr + lane;
                            const int j = e < sl.cnt ? __ldg(sl.list + e) : 0x7FFFFFFF;
                            const bool here = j >= c_lo && j < c_lo + 128;
#pragma unroll
                            for (int w4 = 0; w4 < 4; ++w4)
                                mw[w4] |= __reduce_or_sync(0xffffffffu,
                                                           (here && ((j - c_lo) >> 5) == w4) ? 1u << (j & 31) : 0u);
                            const int used = __popc(__ballot_sync(0xffffffffu, j < c_lo + 128));
                            lm_ptr += used;
                            if (used < 32) break;
                        }
#pragma unroll
                        for (int w4 = 0; w4 < 4; ++w4) {
                            const int r = 32 * w4 + lane;
                            const float b2 = __ldg(a.lbias2 + c_lo + r);  // log2 c_j, or -inf
                            uint4 v = make_uint4(0u, 0u, 0u, 0u);
                            if (((mw[w4] >> lane) & 1u) || !(b2 > -INFINITY)) {
                                v.x = 0xF180u;  // -2^100
                            } else {
                                const float b = __fdiv_rn(b2, a.scale_log2);
                                const __nv_bfloat16 p0 = __float2bfloat16_rn(b);
                                const float r1 = b - __bfloat162float(p0);
                                const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
                                const __nv_bfloat16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
                                v.x = (uint32_t)__bfloat16_as_ushort(p0) | ((uint32_t)__bfloat16_as_ushort(p1) << 16);
                                v.y = (uint32_t)__bfloat16_as_ushort(p2);
                            }
                            *reinterpret_cast<uint4*>(bias + r * 128 + (((2 * q) ^ (r & 7)) << 4)) = v;
                            *reinterpret_cast<uint4*>(bias + r * 128 + (((2 * q + 1) ^ (r & 7)) << 4)) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    fence_proxy_async_smem();  // the MMA reads it through the async proxy
                }
                __syncwarp();
                if (leader) {
                    if (it.kind < 0) sa_flag_error(SA_ERR_BAD_LIST);  // skipped list entry
                    const CUtensorMap* mk = it.kind == 1 ? &a.tm_sk : (it.kind == 2 ? &a.tm_lk : &a.tm_k);
                    const CUtensorMap* mv = it.kind == 1 ? &a.tm_svt : (it.kind == 2 ? &a.tm_lvt : &a.tm_vt);
                    uint8_t* dk = sKV + s * 2 * tc::kTileBytes;
                    meta[s] = make_int4(it.kind, it.lo, it.hi, it.chunk);
                    // releases meta[s] and the warp's bias rows
                    mbar_arrive_expect_tx(&kv_full[s], 2 * tc::kTileBytes);
                    tma_load_2d(dk, mk, &kv_full[s], 0, it.krow);
                    tma_load_2d(dk + tc::kTileBytes, mv, &kv_full[s], 0, it.vrow);
                    tma_load_2d(dk + tc::kTileBytes + tc::kTileBytes / 2, mv, &kv_full[s], 64, it.vrow);
                }
                issued_mask |= 1u << s;
                phase_mask = (phase_mask & ~(1u << s)) | (ph << s);
            }
            if (!ok) {  // let every copy this warp started land before the CTA exits
                for (int s = 0; s < STAGES; ++s)
                    if ((issued_mask >> s) & 1u) tc::drain_wait(&kv_full[s], (phase_mask >> s) & 1u);
                if (n_items > 0 && !withhold) tc::drain_wait(q_full, 0);
            }
        } else {
            // -------------------------------------------------------------- MMA issuer (slot x)
            const bool leader = tc::elect_one();
            bool ok = n_items == 0 || mbar_wait_warp(q_full, 0, abort_flag);
            bool any_mma = false;
            tc_fence_after();
            const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(smem_u32(sKV), 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(smem_u32(sKV + tc::kTileBytes), 16, 1024);
            const uint64_t d_ones = smem_desc_sw128(smem_u32(smem + Lay::kOnes), 16, 1024);
            const uint64_t d_bias = smem_desc_sw128(smem_u32(smem + Lay::kBias), 16, 1024) + 2 * (x * STAGES);
            constexpr uint64_t kStageStep = (2 * tc::kTileBytes) >> 4;
            // S(n) is issued as soon as its tile has landed and the softmax has read S(n-1),
            // P.V(n-1) right after it, as soon as P(n-1) is in TMEM
            for (int n = 0; n <= n_items && ok; ++n) {
                if (n < n_items) {
                    const uint32_t s = n % STAGES, ph = (n / STAGES) & 1u;
                    if (!mbar_wait_warp(&kv_full[s], ph, abort_flag)) { ok = false; break; }
                    if (n > 0 && !mbar_wait_warp(s_free, (n - 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    if (leader) {
                        const uint64_t dk = dk0 + s * kStageStep;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_ss(tmem + Lay::colS(x), dq + 2 * kk, dk + 2 * kk, tc::kIdescS, kk > 0);
                        // columns outside [lo, hi), landmark chunks: add the bias the producer wrote
                        const int4 md = meta[s];
                        if (BIAS && ((LANDMARK && md.x == 2) || md.y > 0 || md.z < 128))
                            umma_ss(tmem + Lay::colS(x), d_ones, d_bias + 2 * s, tc::kIdescS, 1);
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
                        // V^T is two 64-key swizzle atoms of 8 KB; a K=16 step is 32 bytes
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_ts(tmem + Lay::colO(x), tmem + Lay::colP(x) + 8 * kk,
                                    dv + (uint64_t)((kk >> 2) * (8192 >> 4) + (kk & 3) * 2), tc::kIdescPV,
                                    (m > 0 || kk > 0));
                        umma_commit(&kv_empty[s]);
                        umma_commit(pv_done);
                    }
                    __syncwarp();
                }
            }
            // every MMA (and its commits) must be finished before TMEM is released
            if (any_mma) {
                if (leader) umma_commit(drain_bar);
                __syncwarp();
                tc::drain_wait(drain_bar, 0);
            }
        }
    } else {
        // ------------------------------------------------------------------ softmax group
        setmaxnreg_inc<Lay::kRegsSoftmax>();
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + Lay::colS(x) + lane_off;
        const uint32_t tP = tmem + Lay::colP(x) + lane_off;
        const uint32_t tO = tmem + Lay::colO(x) + lane_off;
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int n = 0; n < sl.n_items; ++n) {
            // softmax masking only: the item's valid columns, as the producer decoded them; its
            // stage has landed (S(n) was computed from it), so this wait returns at once and
            // orders the read
            int lo = 0, hi = 128;
            if (!BIAS) {
                if (!mbar_wait_warp(&kv_full[n % STAGES], (n / STAGES) & 1u, abort_flag)) { ok = false; break; }
                const int4 md = meta[n % STAGES];
                lo = md.y;
                hi = md.z;
            }
            if (!mbar_wait_warp(s_full, n & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[128];
            uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(sv + 0);
            uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(sv + 32);
            uint32_t(&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(sv + 64);
            uint32_t(&s3)[32] = *reinterpret_cast<uint32_t(*)[32]>(sv + 96);
            tmem_ld_32x32b_x128(tS, sv);
            tmem_ld_wait(s0);
            reg_fence(s1);
            reg_fence(s2);
            reg_fence(s3);
            tc_fence_before();
            mbar_arrive(s_free);

            // Key columns outside an item's valid range and listed tiles of a landmark chunk arrive
            // as -2^100, landmark chunks with their multiplicity term added (BIAS: the bias
            // product); without BIAS the invalid columns are set to -inf here.
            const float mul = a.scale_log2;
            if (!BIAS && (lo > 0 || hi < 128)) {
                // valid columns [lo, hi) as four 32-bit words; one bit test and select per column
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4) {
                    const int b0 = min(max(lo - 32 * w4, 0), 32), b1 = min(max(hi - 32 * w4, 0), 32);
                    const uint32_t below_hi = b1 == 32 ? 0xFFFFFFFFu : ((1u << b1) - 1u);
                    const uint32_t below_lo = b0 == 32 ? 0xFFFFFFFFu : ((1u << b0) - 1u);
                    const uint32_t valid = below_hi & ~below_lo;
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        if (!((valid >> u) & 1u)) sv[32 * w4 + u] = __float_as_uint(-INFINITY);
                }
            }
            float mx8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mx8[u] = __uint_as_float(sv[u]);
#pragma unroll
            for (int c = 8; c < 128; c += 16)
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    mx8[u] = fmax3(mx8[u], __uint_as_float(sv[c + u]), __uint_as_float(sv[c + 8 + u]));
            const float mx_raw = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                       fmaxf(mx8[6], mx8[7]));
            const float mx = mx_raw * mul;  // base-2 units (-inf stays -inf)
            float m_new = m_run;
            if (mx > m_run + 8.0f) m_new = mx;  // lazy max: rescale only on growth beyond 2^8
            const float m_use = m_new == -INFINITY ? 0.0f : m_new;
            const float alpha = ex2_approx(m_run - m_use);  // 0 on the first item
            const float2 mul2 = make_float2(mul, mul);
            const float2 neg2 = make_float2(-m_use, -m_use);
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float2 xv =
                    __ffma2_rn(make_float2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), mul2, neg2);
                float2 p;
                if ((c & 7) >= 8 - (BIAS ? SA_EXP2_FMA_PAIRS_PER8 : SA_EXP2_FMA_PAIRS_PER8_DENSE)) {
                    p = exp2_poly2(xv);  // FMA pipe: takes load off the MUFU
                } else {
                    p.x = ex2_approx(xv.x);
                    p.y = ex2_approx(xv.y);
                }
                acc[c & 3] = __fadd2_rn(acc[c & 3], p);
                pk[c] = pack_bf16x2(p.x, p.y);
            }
            const float2 acc_all = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
            l_run = l_run * alpha + (acc_all.x + acc_all.y);
            m_run = m_new;
            if (n > 0) {
                // the previous P.V product must be done before O is rescaled or P overwritten;
                // the exponentials above overlap with it
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
            uint32_t(&pb)[32] = *reinterpret_cast<uint32_t(*)[32]>(pk + 32);
            tmem_st_32x32b_x32(tP + 0, pa);
            tmem_st_32x32b_x32(tP + 32, pb);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        // ---- epilogue: O / l, LSE, store valid rows
        if (ok && sl.n_items > 0 && mbar_wait_warp(pv_done, (sl.n_items - 1) & 1, abort_flag)) {
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
        } else if (ok && sl.active && sl.n_items == 0 && r < sl.nq) {
            // nothing to attend: zero output, LSE = -inf
            uint4* dst = reinterpret_cast<uint4*>(a.o + ((int64_t)sl.qrow + r) * 64);
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) dst[c8] = make_uint4(0, 0, 0, 0);
            if (a.lse) a.lse[(int64_t)sl.qrow + r] = -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Lay::kTmemCols);
    }
}
