// Step 3: per-query-tile top-k selection ("SAF3R" abstract: dynamic, input-dependent choice
// of the most promising interactions; "AVGGT" 2.B.1/2.B.2: own frame and diagonal kept).
//
// One 512-thread CTA per score row.  The row is staged in shared memory as order-preserving
// 32-bit keys (larger float -> larger unsigned key; non-candidates get key 0).  An exact
// MSB-first radix select finds the k-th largest candidate key: keys are first offset by the
// row minimum so that the first 8-bit digit already spreads over the populated range
// (raw float keys share their top exponent bits).  Ties at the threshold are broken by
// lower tile index through a block-wide prefix count, and the own-frame tiles, the keys
// above the threshold and the admitted ties are compacted in ascending index order with a
// second block scan.  Every row is read once from memory; everything else stays on chip.
#pragma once
#include "sa_device.cuh"

#define SEL_THREADS 512
#define SEL_MAX_NT 32768  // keys in shared memory: 128 KB

struct SelectArgs {
    const float* scores;  // row (local y, local x) at scores + (y * rows + x) * lds
    int64_t lds;
    int32_t* kept_idx;    // [bh][nt][max_kept]
    int32_t* kept_cnt;    // [bh][nt]
    int32_t nt, tpf, tile, tokens, n_sink;
    int32_t k, max_kept;
    int32_t h0, i0, rows;
};

__device__ __forceinline__ uint32_t f32_order_key(float f) {
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
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

__device__ __forceinline__ bool tile_has_keys(int slot, int tile, int tokens, int n_sink) {
    const int n0 = slot * tile;
    const int nq = min(tile, tokens - n0);
    return nq > max(0, n_sink - n0);
}

__global__ void __launch_bounds__(SEL_THREADS) select_topk_kernel(SelectArgs a) {
    extern __shared__ uint32_t keys[];  // [nt]
    __shared__ uint32_t hist[256];
    __shared__ uint32_t scratch[32];
    __shared__ uint32_t red_min[SEL_THREADS / 32], red_max[SEL_THREADS / 32], red_cnt[SEL_THREADS / 32];
    __shared__ uint32_t bc_digit, bc_above;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = a.h0 + blockIdx.y, i = a.i0 + blockIdx.x;
    const float* row = a.scores + ((int64_t)blockIdx.y * a.rows + blockIdx.x) * a.lds;
    const int nt = a.nt;
    const int frame = i / a.tpf;

    // ---- stage keys, count candidates and their key range
    uint32_t ncand = 0, kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int c = tid; c < nt; c += SEL_THREADS) {
        const bool cand = (c / a.tpf != frame) && tile_has_keys(c % a.tpf, a.tile, a.tokens, a.n_sink);
        uint32_t key = 0u;
        if (cand) {
            key = max(f32_order_key(__ldg(row + c)), 1u);
            ++ncand;
            kmin = min(kmin, key);
            kmax = max(kmax, key);
        }
        keys[c] = key;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        ncand += __shfl_xor_sync(0xffffffffu, ncand, off);
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
    }
    if (lane == 0) {
        red_cnt[warp] = ncand;
        red_min[warp] = kmin;
        red_max[warp] = kmax;
    }
    __syncthreads();
    ncand = 0;
    kmin = 0xFFFFFFFFu;
    kmax = 0u;
    for (int w = 0; w < SEL_THREADS / 32; ++w) {
        ncand += red_cnt[w];
        kmin = min(kmin, red_min[w]);
        kmax = max(kmax, red_max[w]);
    }
    const uint32_t kk = (uint32_t)min((int64_t)a.k, (int64_t)ncand);

    // ---- radix select of the kk-th largest (rel = key - kmin) among candidates
    // mode 0: none selected, 1: all candidates, 2: rel > tau plus the first `remaining` rel == tau
    int mode = kk == 0 ? 0 : (kk == ncand ? 1 : 2);
    uint32_t tau = 0, remaining = kk;
    if (mode == 2) {
        const uint32_t range = kmax - kmin;
        int s_hi = range ? 32 - __clz(range) : 0;
        uint32_t prefix = 0;
        while (s_hi > 0) {
            const int s_lo = max(s_hi - 8, 0);
            const uint32_t nbm = (1u << (s_hi - s_lo)) - 1u;
            for (int b = tid; b < 256; b += SEL_THREADS) hist[b] = 0u;
            __syncthreads();
            const uint64_t want_hi = (uint64_t)prefix >> s_hi;
            for (int c = tid; c < nt; c += SEL_THREADS) {
                const uint32_t key = keys[c];
                if (!key) continue;
                const uint32_t rel = key - kmin;
                if (((uint64_t)rel >> s_hi) == want_hi) atomicAdd(&hist[(rel >> s_lo) & nbm], 1u);
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t bins[8], lsum = 0;
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    bins[b] = hist[8 * lane + b];
                    lsum += bins[b];
                }
                uint32_t suf = lsum;  // sum over lanes >= lane
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t y = __shfl_down_sync(0xffffffffu, suf, off);
                    if (lane + off < 32) suf += y;
                }
                const uint32_t above_lane = suf - lsum;
                if (above_lane < remaining && remaining <= suf) {
                    uint32_t acc = above_lane;
                    for (int b = 7; b >= 0; --b) {
                        if (acc + bins[b] >= remaining) {
                            bc_digit = 8 * lane + b;
                            bc_above = acc;
                            break;
                        }
                        acc += bins[b];
                    }
                }
            }
            __syncthreads();
            remaining -= bc_above;
            prefix |= bc_digit << s_lo;
            s_hi = s_lo;
            __syncthreads();
        }
        tau = prefix;
    }

    // ---- flags over a contiguous chunk per thread, then two block scans
    const int per = (nt + SEL_THREADS - 1) / SEL_THREADS;  // <= 64
    const int c0 = min(nt, tid * per), c1 = min(nt, c0 + per);
    uint32_t n_eq = 0;
    if (mode == 2)
        for (int c = c0; c < c1; ++c) {
            const uint32_t key = keys[c];
            n_eq += (key != 0u && key - kmin == tau);
        }
    uint32_t tot;
    uint32_t eq_rank = block_exclusive_scan(n_eq, scratch, &tot);
    uint64_t sel_bits = 0;
    uint32_t n_sel = 0;
    for (int c = c0; c < c1; ++c) {
        const uint32_t key = keys[c];
        bool sel = (c / a.tpf == frame);
        if (key != 0u) {
            if (mode == 1) {
                sel = true;
            } else if (mode == 2) {
                const uint32_t rel = key - kmin;
                if (rel > tau) {
                    sel = true;
                } else if (rel == tau) {
                    sel = eq_rank < remaining;
                    ++eq_rank;
                }
            }
        }
        if (sel) {
            sel_bits |= 1ull << (c - c0);
            ++n_sel;
        }
    }
    uint32_t pos = block_exclusive_scan(n_sel, scratch, &tot);
    int32_t* out = a.kept_idx + ((int64_t)h * nt + i) * a.max_kept;
    for (int c = c0; c < c1; ++c) {
        if ((sel_bits >> (c - c0)) & 1ull) {
            if (pos < (uint32_t)a.max_kept) out[pos] = c;
            ++pos;
        }
    }
    if (tot > (uint32_t)a.max_kept) {
        if (tid == 0) sa_flag_error(SA_ERR_INVALID_ARG);
        tot = a.max_kept;
    }
    for (int p = tot + tid; p < a.max_kept; p += SEL_THREADS) out[p] = -1;
    if (tid == 0) a.kept_cnt[(int64_t)h * nt + i] = (int32_t)tot;
}
