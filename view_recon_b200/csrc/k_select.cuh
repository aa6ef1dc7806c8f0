// Step 3: per-query-tile top-k selection ("SAF3R" abstract: dynamic, input-dependent choice
// of the most promising interactions; "AVGGT" 2.B.1/2.B.2: own frame and diagonal kept).
//
// Two kernels with the same result, chosen by row length: short rows (up to
// SEL_WARP_MAX_NT tiles) take one warp per row, several rows per CTA and no block-wide
// barrier; long rows take one 256-thread CTA per row (select_topk_block_kernel, below),
// which keeps enough warps resident when a row fills tens of KB of shared memory.
// Selection is exact for the order (score descending, tile index ascending).  Scores become order-preserving
// 32-bit keys (larger float -> larger unsigned key; non-candidates get key 0, candidates at
// least 1), and the k-th largest key T is found most significant digit first:
//   1. the row lands in the warp's shared memory by one bulk copy; one pass turns it into
//      keys in place and builds a 1024-bin histogram of key bits 31..22 (sign, exponent and
//      one mantissa bit: half-octave bins whatever the scores' scale);
//   2. a two-step warp search finds the bin holding the k-th largest; the keys inside that
//      bin are gathered into a short list (or, when the bin is huge, left in the row);
//   3. the gathered keys alone are refined on bits 21..14, 13..6 and 5..0 until the
//      remaining need is a whole bin or T itself is known;
//   4. one ballot pass over the row emits the kept tiles in ascending order: the own frame,
//      every key above T, and the first `need` keys equal to T in index order.
// The row is read from memory once; everything after the copy stays in shared memory.
// The block kernel follows the same plan with a 4096-bin first level over the whole CTA.
#pragma once
#include "sa_device.cuh"

#define SEL_MAX_NT 32768       // row in shared memory: 128 KB
#define SEL_WARP_MAX_NT 2048   // longest row taken by the warp-per-row kernel
#define SEL_MAX_WARPS 8
#define SEL_H1 1024        // first level: key bits 31..22
#define SEL_H2 256         // refinement digits: bits 21..14, 13..6, 5..0
#define SEL_LCAP 256       // boundary-bin keys gathered for refinement (more: refined from the row)
#define SEL_WORD_MIN_WORDS 16  // rows of at least this many 32-tile words: word-per-lane gather and emission
#define SEL_SMEM_BUDGET (44 * 1024)  // per CTA: small CTAs of few rows keep ~20 warps per SM resident

struct SelectArgs {
    const float* scores;  // row (local y, local x) at scores + (y * rows + x) * lds
    int64_t lds;
    int32_t* kept_idx;    // [bh][nt][max_kept]
    int32_t* kept_cnt;    // [bh][nt]
    int32_t nt, tpf, tile, tokens, n_sink;
    int32_t k, max_kept;
    int32_t h0, i0, rows;
    const int32_t* k_head;  // per-head budgets [bh] (device), or null: every head uses k
    int32_t k_max;          // bound on every k_head entry (max_kept was checked against it)
};

// Budget of head h: k, or k_head[h] clamped to [0, k_max] (an entry outside is reported).
__device__ __forceinline__ uint32_t sel_budget(const SelectArgs& a, int h, bool reporter) {
    if (!a.k_head) return (uint32_t)max(a.k, 0);
    const int kh = __ldg(a.k_head + h);
    if ((kh < 0 || kh > a.k_max) && reporter) sa_flag_error(SA_ERR_INVALID_ARG);
    return (uint32_t)min(max(kh, 0), a.k_max);
}

// Shared memory of one warp, in words: the row (4 words of slack so that its 16-byte-aligned
// middle lands 16-byte aligned), the histogram, the gathered keys.
__host__ __device__ inline size_t select_stage_words(int nt) { return ((size_t)nt + 4 + 3) & ~(size_t)3; }
__host__ __device__ inline size_t select_warp_words(int nt) { return select_stage_words(nt) + SEL_H1 + SEL_LCAP; }
// Rows (warps) per CTA for a row length: as many as fit the budget, 1 to SEL_MAX_WARPS.
__host__ __device__ inline int select_warps(int nt) {
    const size_t w = (size_t)SEL_SMEM_BUDGET / (4 * select_warp_words(nt));
    return w < 1 ? 1 : (w > SEL_MAX_WARPS ? SEL_MAX_WARPS : (int)w);
}
__host__ __device__ inline size_t select_smem_bytes(int nt) {
    return (size_t)select_warps(nt) * 4 * select_warp_words(nt);
}

__device__ __forceinline__ uint32_t f32_order_key(float f) {
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct SelBin {
    uint32_t bin, above, count, total;  // boundary bin, entries above it, in it, in all bins
};

// Warp-wide: over NB bins find b with above(b) < want <= above(b) + hist[b], above(b) counting
// the entries of the bins higher than b, for want = min(want_in, total).  Lane l first sums
// bins [l*C, l*C+C) (C = NB/32), a suffix scan picks the lane, then that lane's C bins are
// spread over the warp and scanned the same way.  Meaningful when want >= 1.
template <int NB>
__device__ __forceinline__ SelBin sel_find_bin_warp(const uint32_t* hist, uint32_t want_in) {
    constexpr int C = NB / 32;
    const int lane = threadIdx.x & 31;
    uint32_t lsum = 0;
#pragma unroll
    for (int u = 0; u < C; u += 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(hist + lane * C + u);
        lsum += v.x + v.y + v.z + v.w;
    }
    uint32_t suf = lsum;  // entries in lanes >= lane
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += y;
    }
    SelBin r;
    r.total = __shfl_sync(0xffffffffu, suf, 0);
    const uint32_t want = min(want_in, r.total);
    const uint32_t above_l = suf - lsum;
    const uint32_t hit = __ballot_sync(0xffffffffu, above_l < want && want <= suf);
    const int L = hit ? __ffs(hit) - 1 : 0;
    const uint32_t above_L = __shfl_sync(0xffffffffu, above_l, L);
    // second step: bin L*C + lane (lanes >= C hold nothing)
    const uint32_t mine = lane < C ? hist[L * C + lane] : 0u;
    uint32_t suf2 = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, suf2, off);
        if (lane + off < 32) suf2 += y;
    }
    const uint32_t above2 = above_L + suf2 - mine;
    const uint32_t hit2 = __ballot_sync(0xffffffffu, lane < C && above2 < want && want <= above2 + mine);
    const int b = hit2 ? __ffs(hit2) - 1 : 0;
    r.bin = (uint32_t)(L * C + b);
    r.above = __shfl_sync(0xffffffffu, above2, b);
    r.count = __shfl_sync(0xffffffffu, mine, b);
    return r;
}

__device__ __forceinline__ uint32_t sel_warp_inclusive_scan(uint32_t v, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += y;
    }
    return v;
}

// Masks of the 32-tile word w of a staged row of keys (bit j: tile 32 w + j; tiles past nt and
// of the own frame [f0, f1) excluded from .y, the own frame always set in .x):
//   .x  selected: key >= sel_from (candidates only, key >= 1), unless sel_none
//   .y  in range: key - lo < span (candidates only)
// The reads start at element `rot` mod 32 (16-byte chunk rot mod 8 when vec), so that lanes
// reading different words hit different banks; past nt they land in the slack or the next
// region of the warp's shared memory and are masked.
__device__ __forceinline__ uint2 sel_word_mask(const uint32_t* keys, int w, int nt, int f0, int f1, uint32_t sel_from,
                                               bool sel_none, uint32_t lo, uint32_t span, bool vec, int rot) {
    uint32_t sm = 0u, im = 0u;
    if (vec) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int qq = (q + rot) & 7;
            const uint4 k4 = reinterpret_cast<const uint4*>(keys + w * 32)[qq];
            const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t key = kv[u];
                sm |= ((!sel_none && key >= sel_from && key != 0u) ? 1u : 0u) << (4 * qq + u);
                im |= ((key != 0u && key - lo < span) ? 1u : 0u) << (4 * qq + u);
            }
        }
    } else {
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
            const int jj = (j + rot) & 31;
            const uint32_t key = keys[w * 32 + jj];
            sm |= ((!sel_none && key >= sel_from && key != 0u) ? 1u : 0u) << jj;
            im |= ((key != 0u && key - lo < span) ? 1u : 0u) << jj;
        }
    }
    const int rem = nt - w * 32;
    const uint32_t valid = rem >= 32 ? 0xFFFFFFFFu : ((1u << rem) - 1u);
    const int lo_b = min(max(f0 - 32 * w, 0), 32), hi_b = min(max(f1 - 32 * w, 0), 32);
    const uint32_t own = (hi_b == 32 ? 0xFFFFFFFFu : ((1u << hi_b) - 1u)) & ~(lo_b == 32 ? 0xFFFFFFFFu : ((1u << lo_b) - 1u));
    return make_uint2((sm & valid) | own, im & valid & ~own);
}

__global__ void __launch_bounds__(32 * SEL_MAX_WARPS) select_topk_warp_kernel(SelectArgs a) {
    extern __shared__ __align__(16) uint32_t sel_smem[];
    __shared__ __align__(8) uint64_t bars[SEL_MAX_WARPS];
    __shared__ int aborts[SEL_MAX_WARPS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int x = blockIdx.x * nw + warp;  // local row
    if (x >= a.rows) return;               // no CTA-wide synchronisation follows
    const int nt = a.nt;
    const int nwords = (nt + 31) >> 5;
    uint32_t* stage = sel_smem + (size_t)warp * select_warp_words(nt);
    uint32_t* hist = stage + select_stage_words(nt);  // [SEL_H1]
    uint32_t* lkeys = hist + SEL_H1;                  // [SEL_LCAP]
    uint64_t* bar = &bars[warp];
    volatile int* abort_flag = &aborts[warp];

    const int h = a.h0 + blockIdx.y, i = a.i0 + x;
    const float* row = a.scores + ((int64_t)blockIdx.y * a.rows + x) * a.lds;
    const int f0 = (i / a.tpf) * a.tpf, f1 = f0 + a.tpf;  // own-frame tiles [f0, f1)
    const int s0 = a.n_sink / a.tile;                      // slots below s0 hold no key row

    // ---- stage the row: one bulk copy for its 16-byte-aligned middle [ha, hb), plain loads
    // for the (at most 3 + 3) scores at either end; keys[c] = stage[mis + c]
    const uint32_t mis = (uint32_t)(reinterpret_cast<uintptr_t>(row) >> 2) & 3u;
    const int ha = min(nt, (int)((4u - mis) & 3u));
    const int n4 = (nt - ha) >> 2;
    const int hb = ha + 4 * n4;
    uint32_t* keys = stage + mis;
    if (lane == 0) {
        *abort_flag = 0;
        if (n4 > 0) {
            mbar_init(bar, 1);
            fence_barrier_init();
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar, (uint32_t)n4 * 16u);
            bulk_load(keys + ha, row + ha, (uint32_t)n4 * 16u, bar);
        }
    }
    if (lane < ha) keys[lane] = __float_as_uint(__ldg(row + lane));
    if (lane >= 16 && lane - 16 < nt - hb) keys[hb + lane - 16] = __float_as_uint(__ldg(row + hb + lane - 16));
#pragma unroll
    for (int u = 0; u < SEL_H1 / 128; ++u)
        reinterpret_cast<uint4*>(hist)[u * 32 + lane] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    if (n4 > 0 && !__all_sync(0xffffffffu, mbar_wait(bar, 0, abort_flag))) return;  // timed out

    // ---- 1. keys in place + first-level histogram (every tile outside the own frame counts
    // here; tiles of whole sink slots are taken out afterwards, without a division per tile)
    auto to_key = [&](int c, uint32_t bits) -> uint32_t {
        if (c >= f0 && c < f1) return 0u;
        const uint32_t key = max(f32_order_key(__uint_as_float(bits)), 1u);
        atomicAdd(&hist[key >> 22], 1u);
        return key;
    };
    if (lane < ha) keys[lane] = to_key(lane, keys[lane]);
    for (int g = lane; g < n4; g += 32) {
        uint4* p = reinterpret_cast<uint4*>(keys + ha) + g;
        uint4 v = *p;
        const int c = ha + 4 * g;
        v.x = to_key(c, v.x);
        v.y = to_key(c + 1, v.y);
        v.z = to_key(c + 2, v.z);
        v.w = to_key(c + 3, v.w);
        *p = v;
    }
    if (lane < nt - hb) keys[hb + lane] = to_key(hb + lane, keys[hb + lane]);
    __syncwarp();
    if (s0 > 0) {  // slots below s0 hold sink rows only: not candidates
        for (int e = lane; e < (nt / a.tpf) * s0; e += 32) {
            const int fr = e / s0, c = fr * a.tpf + (e - fr * s0);
            const uint32_t key = keys[c];
            if (key != 0u) {
                atomicSub(&hist[key >> 22], 1u);
                keys[c] = 0u;
            }
        }
        __syncwarp();
    }

    const uint32_t k_req = sel_budget(a, h, lane == 0);
    const SelBin b1 = sel_find_bin_warp<SEL_H1>(hist, k_req);
    const uint32_t ncand = b1.total;
    const uint32_t kk = min(k_req, ncand);
    // kept: own frame, key != 0 and ((key >> shift) > prefix, or == prefix and (whole, or
    // among the first `need` such keys in index order))
    uint32_t prefix, need = 0;
    int shift = 0;
    bool whole;
    if (kk == 0) {          // none of the candidates
        prefix = 0xFFFFFFFFu;
        whole = false;
    } else if (kk == ncand) {  // all of them
        prefix = 1u;
        whole = true;
    } else {
        prefix = b1.bin;
        shift = 22;
        need = kk - b1.above;
        whole = need == b1.count;
    }

    if (!whole && kk > 0) {
        // ---- 2. gather the keys of the boundary bin (all of them land in the list unless
        // there are more than SEL_LCAP; then the refinement reads them from the row).  Long
        // rows: lane l takes the 32-tile words l, l + 32, ...; a word's mask is built in
        // registers, a warp scan places its keys
        uint32_t m = 0;
        if (nwords >= SEL_WORD_MIN_WORDS) {
            const uint32_t bin_lo = prefix << 22;  // the bin is [bin_lo, bin_lo + 2^22)
            for (int r0 = 0; r0 < nwords; r0 += 32) {
                const int w = r0 + lane;
                const uint32_t im = w < nwords ? sel_word_mask(keys, w, nt, f0, f1, 0xFFFFFFFFu, true, bin_lo,
                                                               1u << 22, mis == 0u, lane).y
                                               : 0u;
                const uint32_t cnt = __popc(im);
                const uint32_t inc = sel_warp_inclusive_scan(cnt, lane);
                uint32_t pos2 = m + inc - cnt;
                for (uint32_t e = im; e; e &= e - 1u) {
                    if (pos2 < SEL_LCAP) lkeys[pos2] = keys[w * 32 + __ffs(e) - 1];
                    ++pos2;
                }
                m += __shfl_sync(0xffffffffu, inc, 31);
            }
        } else {  // short rows: one tile per lane and ballots
            for (int c0 = 0; c0 < nt; c0 += 32) {
                const int c = c0 + lane;
                const uint32_t key = c < nt ? keys[c] : 0u;
                const bool in = key != 0u && (key >> 22) == prefix;
                const uint32_t bi = __ballot_sync(0xffffffffu, in);
                const uint32_t pos = m + __popc(bi & ((1u << lane) - 1u));
                if (in && pos < SEL_LCAP) lkeys[pos] = key;
                m += __popc(bi);
            }
        }
        __syncwarp();
        const bool from_list = m <= SEL_LCAP;
        const uint32_t* src = from_list ? lkeys : keys;
        const int src_n = from_list ? (int)m : nt;
        // ---- 3. refine on 8, 8 and 6 more bits
        for (int lvl = 0; lvl < 3 && !whole; ++lvl) {
            const int width = lvl < 2 ? 8 : 6;
            const int lo = 14 - 8 * lvl < 0 ? 0 : 14 - 8 * lvl;  // 14, 6, 0
            const uint32_t digit_mask = (1u << width) - 1u;
            reinterpret_cast<uint4*>(hist)[lane] = make_uint4(0u, 0u, 0u, 0u);
            reinterpret_cast<uint4*>(hist)[32 + lane] = make_uint4(0u, 0u, 0u, 0u);
            __syncwarp();
            for (int e = lane; e < src_n; e += 32) {
                const uint32_t key = src[e];
                if (key != 0u && (key >> (lo + width)) == prefix) atomicAdd(&hist[(key >> lo) & digit_mask], 1u);
            }
            __syncwarp();
            const SelBin r = sel_find_bin_warp<SEL_H2>(hist, need);
            prefix = (prefix << width) | r.bin;
            need -= r.above;
            whole = need == r.count;
            shift = lo;
            __syncwarp();
        }
    }

    // ---- 4. emit the kept tiles in ascending order: own frame, keys above the threshold,
    // and the first `need` keys at it in index order; for long rows word by word, lane l
    // taking words l, l + 32, ... of each round, warp scans placing the ties and the output
    int32_t* out = a.kept_idx + ((int64_t)h * nt + i) * a.max_kept;
    uint32_t pos = 0, tie_before = 0;
    if (nwords >= SEL_WORD_MIN_WORDS) {
        const uint64_t lo64 = (uint64_t)prefix << shift, hi64 = ((uint64_t)prefix + 1ull) << shift;
        const uint64_t from64 = whole ? lo64 : hi64;
        const bool sel_none = from64 > 0xFFFFFFFFull;
        const uint32_t sel_from = sel_none ? 0xFFFFFFFFu : max((uint32_t)from64, 1u);
        const bool ties = !whole && need > 0 && lo64 <= 0xFFFFFFFFull;
        const uint32_t t_lo = ties ? (uint32_t)lo64 : 0u;
        const uint32_t t_span = ties ? (uint32_t)(hi64 - lo64) : 0u;  // shift <= 22: span <= 2^22
        for (int r0 = 0; r0 < nwords; r0 += 32) {
            const int w = r0 + lane;
            uint2 mk = make_uint2(0u, 0u);
            if (w < nwords) mk = sel_word_mask(keys, w, nt, f0, f1, sel_from, sel_none, t_lo, t_span, mis == 0u, lane);
            uint32_t sm = mk.x, tm = mk.y;
            const uint32_t tc = __popc(tm);
            const uint32_t tinc = sel_warp_inclusive_scan(tc, lane);
            const uint32_t tb = tie_before + tinc - tc;  // ties in earlier words
            if (tm && tb < need) {
                const uint32_t take = min(tc, need - tb);
                for (uint32_t t = 0; t < take; ++t) {
                    const uint32_t low = tm & (0u - tm);
                    sm |= low;
                    tm ^= low;
                }
            }
            tie_before += __shfl_sync(0xffffffffu, tinc, 31);
            const uint32_t sc = __popc(sm);
            const uint32_t sinc = sel_warp_inclusive_scan(sc, lane);
            uint32_t o = pos + sinc - sc;
            for (uint32_t e = sm; e; e &= e - 1u) {
                if (o < (uint32_t)a.max_kept) out[o] = w * 32 + __ffs(e) - 1;
                ++o;
            }
            pos += __shfl_sync(0xffffffffu, sinc, 31);
        }
    } else {  // short rows: one tile per lane and ballots
        for (int c0 = 0; c0 < nt; c0 += 32) {
            const int c = c0 + lane;
            const uint32_t key = c < nt ? keys[c] : 0u;
            const uint32_t p = key >> shift;
            const bool own = c >= f0 && c < f1;
            const bool above = key != 0u && (p > prefix || (whole && p == prefix));
            const bool tie = !whole && key != 0u && p == prefix;
            bool sel = own || above;
            const uint32_t bt = __ballot_sync(0xffffffffu, tie);
            if (bt) {
                sel = sel || (tie && tie_before + __popc(bt & ((1u << lane) - 1u)) < need);
                tie_before += __popc(bt);
            }
            const uint32_t bs = __ballot_sync(0xffffffffu, sel);
            const uint32_t o = pos + __popc(bs & ((1u << lane) - 1u));
            if (sel && o < (uint32_t)a.max_kept) out[o] = c;
            pos += __popc(bs);
        }
    }
    uint32_t tot = pos;
    if (tot > (uint32_t)a.max_kept) {
        if (lane == 0) sa_flag_error(SA_ERR_INVALID_ARG);
        tot = a.max_kept;
    }
    for (int p = tot + lane; p < a.max_kept; p += 32) out[p] = -1;
    if (lane == 0) a.kept_cnt[(int64_t)h * nt + i] = (int32_t)tot;
}

// ----------------------------------------------------------------------------------------------
// Block-per-row variant (long rows): 256 threads share one staged row.
#define SEL_BLOCK_THREADS 256
#define SEL_BLOCK_H1 4096  // first level: key bits 31..20
#define SEL_BLOCK_H2 1024  // refinement levels: key bits 19..10, then 9..0
__host__ __device__ inline size_t select_block_stage_words(int nt) { return ((size_t)nt + 4 + 3) & ~(size_t)3; }
__host__ __device__ inline size_t select_block_list_words(int nt) {
    const size_t w = ((size_t)nt + 1) / 2;
    return w > SEL_BLOCK_H1 ? ((w + 3) & ~(size_t)3) : (size_t)SEL_BLOCK_H1;
}
__host__ __device__ inline size_t select_block_smem_bytes(int nt) {
    return 4 * (select_block_stage_words(nt) + select_block_list_words(nt) + 2 * (((size_t)nt + 31) / 32));
}

// Exclusive scan of one value per thread over the whole block; returns the prefix and
// writes the block total to *total.  Uses `scratch` (>= 32 uint32) in shared memory.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* scratch, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        uint32_t w = lane < nw ? scratch[lane] : 0u;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < nw) scratch[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    const uint32_t before = (warp > 0 ? scratch[warp - 1] : 0u) + x - v;
    *total = scratch[(blockDim.x >> 5) - 1];
    __syncthreads();
    return before;
}

struct SelBlockBin {
    uint32_t bin, above, count;  // boundary bin, entries in higher bins, entries in it
};

// Over BPT * SEL_BLOCK_THREADS bins, find the bin b with above(b) < want <= above(b) + hist[b],
// above(b) counting the entries of the bins higher than b, for want = min(want_in, total).
// Returns the total; *out is written (and visible to all threads) when want >= 1.
template <int BPT>
__device__ __forceinline__ uint32_t sel_find_bin(const uint32_t* hist, uint32_t want_in, uint32_t* scratch,
                                                 SelBlockBin* out) {
    const int tid = threadIdx.x;
    uint32_t bins[BPT], lsum = 0;
    if constexpr (BPT % 4 == 0) {  // 16-byte reads: a thread's bins are contiguous
#pragma unroll
        for (int u = 0; u < BPT / 4; ++u) {
            const uint4 b4 = reinterpret_cast<const uint4*>(hist + BPT * tid)[u];
            bins[4 * u] = b4.x;
            bins[4 * u + 1] = b4.y;
            bins[4 * u + 2] = b4.z;
            bins[4 * u + 3] = b4.w;
        }
    } else {
#pragma unroll
        for (int u = 0; u < BPT; ++u) bins[u] = hist[BPT * tid + u];
    }
#pragma unroll
    for (int u = 0; u < BPT; ++u) lsum += bins[u];
    uint32_t total;
    const uint32_t before = block_exclusive_scan(lsum, scratch, &total);
    const uint32_t want = min(want_in, total);
    const uint32_t above_t = total - before - lsum;
    if (want > 0 && above_t < want && want <= above_t + lsum) {
        uint32_t acc = above_t;
#pragma unroll
        for (int u = BPT - 1; u >= 0; --u) {
            if (acc < want && acc + bins[u] >= want) {
                out->bin = BPT * tid + u;
                out->above = acc;
                out->count = bins[u];
            }
            acc += bins[u];
        }
    }
    __syncthreads();
    return total;
}

// Selection of one row (head h, query tile i) by the whole 256-thread CTA; sel_smem holds
// select_block_smem_bytes(nt) bytes.  The row is staged by one bulk copy (cg_rows == false) or,
// for rows that other CTAs of the same launch have just written, by L2-coherent loads.
// Returns false when a wait ran out (reported in the error word); the CTA is converged on
// return either way.
__device__ __forceinline__ bool select_row_block(const SelectArgs& a, int h, int i, const float* row,
                                                 bool cg_rows, uint32_t* sel_smem) {
    const int nt = a.nt;
    const int nwords = (nt + 31) >> 5;
    uint32_t* stage = sel_smem;
    uint32_t* hist1 = stage + select_block_stage_words(nt);   // [SEL_BLOCK_H1], then the list
    uint16_t* lst = reinterpret_cast<uint16_t*>(hist1);
    uint32_t* selmask = hist1 + select_block_list_words(nt);  // [nwords]
    uint32_t* eqmask = selmask + nwords;                // [nwords]
    __shared__ __align__(16) uint32_t hist2[SEL_BLOCK_H2];
    __shared__ uint32_t scratch[32];
    __shared__ __align__(8) uint64_t bar;
    __shared__ SelBlockBin sb;
    __shared__ uint32_t list_n;
    __shared__ int abort_flag;

    const int tid = threadIdx.x;
    const int f0 = (i / a.tpf) * a.tpf, f1 = f0 + a.tpf;  // own-frame tiles [f0, f1)
    const int s0 = a.n_sink / a.tile;                      // slots below s0 hold no key row

    // ---- stage the row: one bulk copy for its 16-byte-aligned middle, plain loads for the
    // (at most 3 + 3) scores at either end.  keys[c] = stage[mis + c], so that the copy's
    // destination keys + ha is 16-byte aligned like its source row + ha.
    const uint32_t mis = cg_rows ? 0u : (uint32_t)(reinterpret_cast<uintptr_t>(row) >> 2) & 3u;
    const int ha = cg_rows ? 0 : min(nt, (int)((4u - mis) & 3u));
    const int n4 = cg_rows ? 0 : (nt - ha) >> 2;
    const int hb = ha + 4 * n4;
    uint32_t* keys = stage + mis;
    if (tid == 0) {
        list_n = 0;
        abort_flag = 0;
        if (n4 > 0) {
            mbar_init(&bar, 1);
            fence_barrier_init();
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bar, (uint32_t)n4 * 16u);
            bulk_load(keys + ha, row + ha, (uint32_t)n4 * 16u, &bar);
        }
    }
    if (cg_rows) {
        for (int c = tid; c < nt; c += SEL_BLOCK_THREADS) keys[c] = __float_as_uint(__ldcg(row + c));
    } else {
        if (tid < ha) keys[tid] = __float_as_uint(__ldg(row + tid));
        if (tid >= 32 && tid - 32 < nt - hb) keys[hb + tid - 32] = __float_as_uint(__ldg(row + hb + tid - 32));
    }
#pragma unroll
    for (int u = 0; u < SEL_BLOCK_H1 / SEL_BLOCK_THREADS; ++u) hist1[u * SEL_BLOCK_THREADS + tid] = 0u;
    for (int w = tid; w < nwords; w += SEL_BLOCK_THREADS) eqmask[w] = 0u;
    __syncthreads();
    if (n4 > 0) {
        const bool ok = mbar_wait(&bar, 0, &abort_flag);
        if (__syncthreads_or(!ok)) return false;  // timed out: the error word says so
    }

    // ---- 1. keys in place + first-level histogram (sink slots taken out afterwards), four keys
    // per 16-byte access over the aligned middle of the row
    {
        auto to_key = [&](int c, uint32_t bits) -> uint32_t {
            if (c >= f0 && c < f1) return 0u;
            const uint32_t key = max(f32_order_key(__uint_as_float(bits)), 1u);
            atomicAdd(&hist1[key >> 20], 1u);
            return key;
        };
        const int va = min(nt, (int)((4u - mis) & 3u));  // keys + va is 16-byte aligned
        const int vn = (nt - va) >> 2;
        const int vb = va + 4 * vn;
        if (tid < va) keys[tid] = to_key(tid, keys[tid]);
        for (int g = tid; g < vn; g += SEL_BLOCK_THREADS) {
            uint4* p = reinterpret_cast<uint4*>(keys + va) + g;
            uint4 v = *p;
            const int c = va + 4 * g;
            v.x = to_key(c, v.x);
            v.y = to_key(c + 1, v.y);
            v.z = to_key(c + 2, v.z);
            v.w = to_key(c + 3, v.w);
            *p = v;
        }
        if (tid < nt - vb) keys[vb + tid] = to_key(vb + tid, keys[vb + tid]);
    }
    __syncthreads();
    if (s0 > 0) {  // slots below s0 hold sink rows only: not candidates
        for (int e = tid; e < (nt / a.tpf) * s0; e += SEL_BLOCK_THREADS) {
            const int fr = e / s0, c = fr * a.tpf + (e - fr * s0);
            const uint32_t key = keys[c];
            if (key != 0u) {
                atomicSub(&hist1[key >> 20], 1u);
                keys[c] = 0u;
            }
        }
        __syncthreads();
    }
    const uint32_t k_req = sel_budget(a, h, tid == 0);
    const uint32_t ncand = sel_find_bin<SEL_BLOCK_H1 / SEL_BLOCK_THREADS>(hist1, k_req, scratch, &sb);
    const uint32_t kk = min(k_req, ncand);
    // selected: own frame, or (key >> shift) > prefix, or == prefix and admitted; with
    // `whole` set every tile at == prefix is admitted
    const int mode = kk == 0 ? 0 : (kk == ncand ? 1 : 2);  // 0 none, 1 all candidates, 2 threshold
    uint32_t prefix = 0, need = 0;
    int shift = 20;
    bool whole = false;
    if (mode == 2) {
        prefix = sb.bin;
        need = kk - sb.above;
        whole = need == sb.count;
    }

    // ---- 2. bitmask of tiles above the boundary bin; list of the tiles inside it (the list
    // overwrites hist1, whose last reads precede the syncs inside sel_find_bin)
    // One thread per 32-tile word builds both masks in registers: selected = key at or above
    // sel_from (candidates only: key >= 1), boundary = key in [in_lo, in_lo + in_span).  Thread
    // t reads the word's keys starting at element t mod 32, so that a warp's shared-memory
    // reads hit 32 different banks.
    {
        uint32_t sel_from = 0xFFFFFFFFu, in_lo = 0u, in_span = 0u;
        bool sel_none = mode == 0;
        if (mode == 1) {
            sel_from = 1u;
        } else if (mode == 2) {
            const uint32_t lo = prefix << 20;
            if (whole) {
                sel_from = max(lo, 1u);
            } else {
                sel_from = prefix == 0xFFFu ? 0xFFFFFFFFu : (prefix + 1u) << 20;
                sel_none = prefix == 0xFFFu;  // nothing lies above the top bin
                in_lo = lo;
                in_span = 1u << 20;
            }
        }
        const bool vec = mis == 0u;  // keys 16-byte aligned: a word is eight 16-byte reads
        for (int wd = tid; wd < nwords; wd += SEL_BLOCK_THREADS) {
            uint32_t sm = 0u, im = 0u;
            // past nt the reads land in the slack or the next region: masked below
            if (vec) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int qq = (q + wd) & 7;  // rotated by the word: a quarter-warp reads 8 bank groups
                    const uint4 k4 = reinterpret_cast<const uint4*>(keys + wd * 32)[qq];
                    const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t key = kv[u];
                        const uint32_t sbit = (!sel_none && key >= sel_from && key != 0u) ? 1u : 0u;
                        const uint32_t ibit = (key != 0u && key - in_lo < in_span) ? 1u : 0u;
                        sm |= sbit << (4 * qq + u);
                        im |= ibit << (4 * qq + u);
                    }
                }
            } else {
#pragma unroll 8
                for (int j = 0; j < 32; ++j) {
                    const int jj = (j + wd) & 31;
                    const uint32_t key = keys[wd * 32 + jj];
                    const uint32_t sbit = (!sel_none && key >= sel_from && key != 0u) ? 1u : 0u;
                    const uint32_t ibit = (key != 0u && key - in_lo < in_span) ? 1u : 0u;
                    sm |= sbit << jj;
                    im |= ibit << jj;
                }
            }
            const int rem = nt - wd * 32;  // valid tiles in this word
            const uint32_t valid = rem >= 32 ? 0xFFFFFFFFu : ((1u << rem) - 1u);
            const int lo = min(max(f0 - 32 * wd, 0), 32), hi = min(max(f1 - 32 * wd, 0), 32);
            const uint32_t own = (hi == 32 ? 0xFFFFFFFFu : ((1u << hi) - 1u)) & ~(lo == 32 ? 0xFFFFFFFFu : ((1u << lo) - 1u));
            sm = (sm & valid) | own;
            im &= valid & ~own;
            selmask[wd] = sm;
            if (im) {
                uint32_t base = atomicAdd(&list_n, (uint32_t)__popc(im));
                while (im) {
                    const int b = __ffs(im) - 1;
                    im &= im - 1u;
                    lst[base++] = (uint16_t)(wd * 32 + b);
                }
            }
        }
    }
    __syncthreads();

    // ---- 3. refine the listed tiles on the lower key bits
    if (mode == 2 && !whole) {
        const uint32_t m = list_n;
        for (int lvl = 0; lvl < 2 && !whole; ++lvl) {
            const int sh = 10 - 10 * lvl;
            for (int b = tid; b < SEL_BLOCK_H2; b += SEL_BLOCK_THREADS) hist2[b] = 0u;
            __syncthreads();
            for (uint32_t e = tid; e < m; e += SEL_BLOCK_THREADS) {
                const uint32_t key = keys[lst[e]];
                if ((key >> (sh + 10)) == prefix) atomicAdd(&hist2[(key >> sh) & (SEL_BLOCK_H2 - 1)], 1u);
            }
            __syncthreads();
            sel_find_bin<SEL_BLOCK_H2 / SEL_BLOCK_THREADS>(hist2, need, scratch, &sb);
            prefix = (prefix << 10) | sb.bin;
            need -= sb.above;
            whole = need == sb.count;
            shift = sh;
            __syncthreads();
        }
        // admit the listed tiles above the threshold (and at it, when all of them are taken);
        // mark ties otherwise
        for (uint32_t e = tid; e < m; e += SEL_BLOCK_THREADS) {
            const int c = lst[e];
            const uint32_t p = keys[c] >> shift;
            if (p > prefix || (whole && p == prefix))
                atomicOr(&selmask[c >> 5], 1u << (c & 31));
            else if (p == prefix)
                atomicOr(&eqmask[c >> 5], 1u << (c & 31));
        }
        __syncthreads();
    }

    // ---- 4. ties in index order, then compaction; thread t owns words [w0, w1)
    const int wpt = (nwords + SEL_BLOCK_THREADS - 1) / SEL_BLOCK_THREADS;  // <= 4
    const int w0 = min(nwords, tid * wpt), w1 = min(nwords, w0 + wpt);
    uint32_t tot;
    if (mode == 2 && !whole) {  // shift == 0 here: the tied tiles share the exact threshold key
        uint32_t n_eq = 0;
        for (int w = w0; w < w1; ++w) n_eq += __popc(eqmask[w]);
        uint32_t before = block_exclusive_scan(n_eq, scratch, &tot);
        for (int w = w0; w < w1; ++w) {
            uint32_t e = eqmask[w], take = 0;
            const uint32_t pc = __popc(e);
            if (need > before) take = min(pc, need - before);
            uint32_t admit = 0;
            for (uint32_t t = 0; t < take; ++t) {
                const uint32_t low = e & (0u - e);
                admit |= low;
                e ^= low;
            }
            selmask[w] |= admit;
            before += pc;
        }
    }
    uint32_t n_sel = 0;
    for (int w = w0; w < w1; ++w) n_sel += __popc(selmask[w]);
    uint32_t pos = block_exclusive_scan(n_sel, scratch, &tot);
    int32_t* out = a.kept_idx + ((int64_t)h * nt + i) * a.max_kept;
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = selmask[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1u;
            if (pos < (uint32_t)a.max_kept) out[pos] = w * 32 + b;
            ++pos;
        }
    }
    if (tot > (uint32_t)a.max_kept) {
        if (tid == 0) sa_flag_error(SA_ERR_INVALID_ARG);
        tot = a.max_kept;
    }
    for (int p = tot + tid; p < a.max_kept; p += SEL_BLOCK_THREADS) out[p] = -1;
    if (tid == 0) a.kept_cnt[(int64_t)h * nt + i] = (int32_t)tot;
    __syncthreads();  // the CTA's shared memory may be reused right after
    return true;
}

__global__ void __launch_bounds__(SEL_BLOCK_THREADS) select_topk_block_kernel(SelectArgs a) {
    extern __shared__ __align__(16) uint32_t sel_smem[];
    const int h = a.h0 + blockIdx.y, i = a.i0 + blockIdx.x;
    const float* row = a.scores + ((int64_t)blockIdx.y * a.rows + blockIdx.x) * a.lds;
    select_row_block(a, h, i, row, false, sel_smem);
}
