// Step 3: per-query-tile top-k selection ("SAF3R" abstract: dynamic, input-dependent choice
// of the most promising interactions; "AVGGT" 2.B.1/2.B.2: own frame and diagonal kept).
//
// One 256-thread CTA per score row.  Selection is exact for the order (score descending,
// tile index ascending).  Scores become order-preserving 32-bit keys (larger float -> larger
// unsigned key; non-candidates get key 0, candidates at least 1), and the k-th largest key is
// found MSB first:
//   1. the row lands in shared memory by one bulk copy; one pass turns it into keys in place
//      and builds a 4096-bin histogram of the top 12 key bits (sign, exponent, 3 mantissa
//      bits: a relative resolution of 1/8 octave whatever the scores' scale);
//   2. the bin holding the k-th largest is found by a block-wide suffix count; one ballot
//      pass over the row marks every tile above that bin (and the own frame) in a bitmask and
//      lists the tiles inside it;
//   3. only the listed tiles are refined, on key bits 19..10 and 9..0, until the remaining
//      need is a whole bin or the exact threshold key is known;
//   4. tiles tied at the threshold are admitted in ascending index order by a prefix count
//      over a tie bitmask, and the bitmask is compacted into ascending indices.
// Each row is read from memory once; everything after the copy stays on chip.
#pragma once
#include "sa_device.cuh"

#define SEL_THREADS 256
#define SEL_MAX_NT 32768   // row in shared memory: 128 KB; list indices fit 16 bits
#define SEL_H1 4096        // first level: key bits 31..20
#define SEL_H2 1024        // refinement levels: key bits 19..10, then 9..0

struct SelectArgs {
    const float* scores;  // row (local y, local x) at scores + (y * rows + x) * lds
    int64_t lds;
    int32_t* kept_idx;    // [bh][nt][max_kept]
    int32_t* kept_cnt;    // [bh][nt]
    int32_t nt, tpf, tile, tokens, n_sink;
    int32_t k, max_kept;
    int32_t h0, i0, rows;
};

// Dynamic shared memory: the row (4 words of slack for alignment), the first-level histogram
// (later reused as the 16-bit list of boundary tiles), the selection and tie bitmasks.
__host__ __device__ inline size_t select_stage_words(int nt) { return ((size_t)nt + 4 + 3) & ~(size_t)3; }
__host__ __device__ inline size_t select_list_words(int nt) {
    const size_t w = ((size_t)nt + 1) / 2;
    return w > SEL_H1 ? ((w + 3) & ~(size_t)3) : (size_t)SEL_H1;
}
__host__ __device__ inline size_t select_smem_bytes(int nt) {
    return 4 * (select_stage_words(nt) + select_list_words(nt) + 2 * (((size_t)nt + 31) / 32));
}

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

struct SelBin {
    uint32_t bin, above, count;  // boundary bin, entries in higher bins, entries in it
};

// Over BPT * SEL_THREADS bins, find the bin b with above(b) < want <= above(b) + hist[b],
// above(b) counting the entries of the bins higher than b, for want = min(want_in, total).
// Returns the total; *out is written (and visible to all threads) when want >= 1.
template <int BPT>
__device__ __forceinline__ uint32_t sel_find_bin(const uint32_t* hist, uint32_t want_in, uint32_t* scratch,
                                                 SelBin* out) {
    const int tid = threadIdx.x;
    uint32_t bins[BPT], lsum = 0;
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
        bins[u] = hist[BPT * tid + u];
        lsum += bins[u];
    }
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

__global__ void __launch_bounds__(SEL_THREADS) select_topk_kernel(SelectArgs a) {
    extern __shared__ __align__(16) uint32_t sel_smem[];
    const int nt = a.nt;
    const int nwords = (nt + 31) >> 5;
    uint32_t* stage = sel_smem;
    uint32_t* hist1 = stage + select_stage_words(nt);   // [SEL_H1], then the list
    uint16_t* lst = reinterpret_cast<uint16_t*>(hist1);
    uint32_t* selmask = hist1 + select_list_words(nt);  // [nwords]
    uint32_t* eqmask = selmask + nwords;                // [nwords]
    __shared__ uint32_t hist2[SEL_H2];
    __shared__ uint32_t scratch[32];
    __shared__ __align__(8) uint64_t bar;
    __shared__ SelBin sb;
    __shared__ uint32_t list_n;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = a.h0 + blockIdx.y, i = a.i0 + blockIdx.x;
    const float* row = a.scores + ((int64_t)blockIdx.y * a.rows + blockIdx.x) * a.lds;
    const int f0 = (i / a.tpf) * a.tpf, f1 = f0 + a.tpf;  // own-frame tiles [f0, f1)
    const int s0 = a.n_sink / a.tile;                      // slots below s0 hold no key row

    // ---- stage the row: one bulk copy for its 16-byte-aligned middle, plain loads for the
    // (at most 3 + 3) scores at either end.  keys[c] = stage[mis + c], so that the copy's
    // destination keys + ha is 16-byte aligned like its source row + ha.
    const uint32_t mis = (uint32_t)(reinterpret_cast<uintptr_t>(row) >> 2) & 3u;
    const int ha = min(nt, (int)((4u - mis) & 3u));
    const int n4 = (nt - ha) >> 2;
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
    if (tid < ha) keys[tid] = __float_as_uint(__ldg(row + tid));
    if (tid >= 32 && tid - 32 < nt - hb) keys[hb + tid - 32] = __float_as_uint(__ldg(row + hb + tid - 32));
#pragma unroll
    for (int u = 0; u < SEL_H1 / SEL_THREADS; ++u) hist1[u * SEL_THREADS + tid] = 0u;
    for (int w = tid; w < nwords; w += SEL_THREADS) eqmask[w] = 0u;
    __syncthreads();
    if (n4 > 0) {
        const bool ok = mbar_wait(&bar, 0, &abort_flag);
        if (__syncthreads_or(!ok)) return;  // timed out: the error word says so
    }

    // ---- 1. keys in place + first-level histogram
    for (int c = tid; c < nt; c += SEL_THREADS) {
        const bool cand = (c < f0 || c >= f1) && (s0 == 0 || c % a.tpf >= s0);
        uint32_t key = 0u;
        if (cand) {
            key = max(f32_order_key(__uint_as_float(keys[c])), 1u);
            atomicAdd(&hist1[key >> 20], 1u);
        }
        keys[c] = key;
    }
    __syncthreads();
    const uint32_t k_req = (uint32_t)max(a.k, 0);
    const uint32_t ncand = sel_find_bin<SEL_H1 / SEL_THREADS>(hist1, k_req, scratch, &sb);
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
    for (int wd = warp; wd < nwords; wd += SEL_THREADS / 32) {
        const int c = wd * 32 + lane;
        const uint32_t key = c < nt ? keys[c] : 0u;
        const bool own = c >= f0 && c < f1;
        bool sel, in = false;
        if (mode == 0) {
            sel = own;
        } else if (mode == 1) {
            sel = own || key != 0u;
        } else {
            const uint32_t top = key >> 20;
            sel = own || (key != 0u && (top > prefix || (whole && top == prefix)));
            in = !whole && key != 0u && top == prefix;
        }
        const uint32_t bs = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) selmask[wd] = bs;
        const uint32_t bi = __ballot_sync(0xffffffffu, in);
        if (bi) {
            uint32_t base = 0;
            if (lane == 0) base = atomicAdd(&list_n, (uint32_t)__popc(bi));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (in) lst[base + __popc(bi & ((1u << lane) - 1u))] = (uint16_t)c;
        }
    }
    __syncthreads();

    // ---- 3. refine the listed tiles on the lower key bits
    if (mode == 2 && !whole) {
        const uint32_t m = list_n;
        for (int lvl = 0; lvl < 2 && !whole; ++lvl) {
            const int sh = 10 - 10 * lvl;
            for (int b = tid; b < SEL_H2; b += SEL_THREADS) hist2[b] = 0u;
            __syncthreads();
            for (uint32_t e = tid; e < m; e += SEL_THREADS) {
                const uint32_t key = keys[lst[e]];
                if ((key >> (sh + 10)) == prefix) atomicAdd(&hist2[(key >> sh) & (SEL_H2 - 1)], 1u);
            }
            __syncthreads();
            sel_find_bin<SEL_H2 / SEL_THREADS>(hist2, need, scratch, &sb);
            prefix = (prefix << 10) | sb.bin;
            need -= sb.above;
            whole = need == sb.count;
            shift = sh;
            __syncthreads();
        }
        // admit the listed tiles above the threshold (and at it, when all of them are taken);
        // mark ties otherwise
        for (uint32_t e = tid; e < m; e += SEL_THREADS) {
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
    const int wpt = (nwords + SEL_THREADS - 1) / SEL_THREADS;  // <= 4
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
    for (int p = tot + tid; p < a.max_kept; p += SEL_THREADS) out[p] = -1;
    if (tid == 0) a.kept_cnt[(int64_t)h * nt + i] = (int32_t)tot;
}
