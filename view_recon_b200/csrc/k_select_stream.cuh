// Step 3 without a score matrix: streamed selection in one persistent launch ("SAF3R"
// abstract: dynamic, input-dependent selection per head; no [bh][nt][nt] matrix is kept).
//
// The rows of every head are cut into blocks of R query tiles.  Each block is a list of work
// items: its 128 x 128 score tiles (same f32 FMA chain as sa_tile_scores), then one
// selection item per row.  Blocks follow each other head after head, alternating between two
// L2-sized buffers of R score rows.  CTAs take items in order from one atomic counter, so an
// item only ever waits for items taken before it (by CTAs that are running):
//   a score tile of block g waits until every row of block g - 2 (the same buffer) has been
//     selected;
//   a row of block g waits until every score tile of block g is written.
// Completion counts are published with a device-scope fence before the atomic increment and
// read with an acquire load; selection reads the buffer through L2 (ld.global.cg), never
// through a possibly stale L1 line.  Every wait is bounded (g_sa_wait_limit_ns); a wait that
// runs out records SA_ERR_TIMEOUT and raises a launch-wide abort word that all CTAs poll.
#pragma once
#include "k_scores.cuh"
#include "k_select.cuh"

struct StreamSelArgs {
    SelectArgs sel;        // lists, geometry, budgets (scores/lds/h0/i0/rows unused)
    const float* q_pool;   // [bh][nt][64]
    const float* k_pool;   // [bh][nt][64]
    float* buf;            // [2][R][nt]
    int32_t* ctl;          // [0] next item, [1] abort, [2 .. 2+G) tiles done, [2+G .. 2+2G) rows done
    int32_t bh, R, nblk, col_tiles;
    int64_t items_per_head, items_total;
};

__device__ __forceinline__ int32_t ld_acquire_i32(const int32_t* p) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Thread 0 waits until *p >= target (bounded); the result is broadcast to the CTA.
__device__ __forceinline__ bool stream_wait(const StreamSelArgs& a, const int32_t* p, int32_t target, int* s_ok) {
    if (threadIdx.x == 0) {
        bool ok = true;
        if (ld_acquire_i32(p) < target) {
            const uint64_t t0 = sa_globaltimer();
            const uint64_t limit = g_sa_wait_limit_ns;
            while (ld_acquire_i32(p) < target) {
                if (ld_acquire_i32(a.ctl + 1) != 0) {
                    ok = false;
                    break;
                }
                if (sa_globaltimer() - t0 > limit) {
                    sa_flag_error(SA_ERR_TIMEOUT);
                    atomicExch(a.ctl + 1, 1);
                    ok = false;
                    break;
                }
                __nanosleep(128);
            }
        }
        *s_ok = ok ? 1 : 0;
    }
    __syncthreads();
    return *s_ok != 0;
}

__global__ void __launch_bounds__(256) select_stream_kernel(const __grid_constant__ StreamSelArgs a) {
    extern __shared__ __align__(16) uint32_t ss_smem[];
    __shared__ int64_t s_item;
    __shared__ int s_ok;
    const int nt = a.sel.nt;
    const int G = a.bh * a.nblk;
    int32_t* tiles_done = a.ctl + 2;
    int32_t* rows_done = a.ctl + 2 + G;
    const int64_t full_block_items = (int64_t)((a.R + 127) / 128) * a.col_tiles + a.R;
    for (;;) {
        if (threadIdx.x == 0) s_item = atomicAdd(a.ctl, 1);
        __syncthreads();
        const int64_t t = s_item;
        __syncthreads();
        if (t >= a.items_total) break;
        // decode: head, block, then score tile or selection row inside the block
        const int h = (int)(t / a.items_per_head);
        int64_t rem = t - (int64_t)h * a.items_per_head;
        const int64_t b_full = rem / full_block_items;
        const int b = b_full < a.nblk - 1 ? (int)b_full : a.nblk - 1;
        rem -= (int64_t)b * full_block_items;
        const int rows_b = min(a.R, nt - b * a.R);
        const int tiles_b = ((rows_b + 127) / 128) * a.col_tiles;
        const int g = h * a.nblk + b;
        float* blk = a.buf + (int64_t)(g & 1) * a.R * nt;
        if (rem < tiles_b) {
            const int tr = (int)(rem / a.col_tiles), tc = (int)(rem % a.col_tiles);
            if (g >= 2) {
                const int gp = g - 2;
                const int bp = gp % a.nblk;
                const int rows_p = min(a.R, nt - bp * a.R);
                if (!stream_wait(a, rows_done + gp, rows_p, &s_ok)) break;
            }
            const float* qb = a.q_pool + ((int64_t)h * nt + (int64_t)b * a.R + tr * 128) * 64;
            const float* kb = a.k_pool + ((int64_t)h * nt + tc * 128) * 64;
            score_block_128(qb, rows_b - tr * 128, kb, nt - tc * 128, blk + (int64_t)tr * 128 * nt + tc * 128, nt,
                            reinterpret_cast<float*>(ss_smem));
            __syncthreads();
            if (threadIdx.x == 0) {
                __threadfence();
                atomicAdd(tiles_done + g, 1);
            }
        } else {
            const int r = (int)(rem - tiles_b);
            if (!stream_wait(a, tiles_done + g, tiles_b, &s_ok)) break;
            if (!select_row_block(a.sel, h, b * a.R + r, blk + (int64_t)r * nt, true, ss_smem)) {
                if (threadIdx.x == 0) atomicExch(a.ctl + 1, 1);
                break;
            }
            if (threadIdx.x == 0) {
                __threadfence();
                atomicAdd(rows_done + g, 1);
            }
        }
    }
}
