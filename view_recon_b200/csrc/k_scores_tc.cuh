// Step 2 on the 5th-generation tensor cores: tile scores s[h][i][j] = q_pool[h][i] . k_pool[h][j]
// ("SAF3R" abstract: rank the candidate interactions per head) to about f32 accuracy.
//
// A single tf32 product keeps 11 significant bits per operand, far from the ~1e-6 relative
// accuracy the ranking needs.  Every f32 operand is therefore split into two tf32 parts,
// x = hi + lo with hi = rn_tf32(x) and lo = rn_tf32(x - hi) (x - hi - lo is below 2^-22 |x|),
// and a . b is taken as hi.hi + hi.lo + lo.hi (the dropped lo.lo is below 2^-22 |a||b| per term),
// all accumulated in f32 by kind::tf32 MMAs ("split-precision" or 3xTF32 products).
//
// One CTA takes a 128-row tile of query tiles and a run of 128-column chunks of key tiles:
//   S (128 x 128 per chunk, f32 in TMEM) = sum over 8 K-steps of 8 of A_hi B_hi + A_hi B_lo + A_lo B_hi
// Warp roles (384 threads, one CTA per SM: 192 KB of operands):
//   warp 0           TMA producer: the A tile once, then the chunks' K rows into a 2-stage ring
//                    (f32 rows as two 128-byte swizzle atoms of 32 columns; no multicast);
//   warp 1           tcgen05.mma issuer (24 per chunk) and owner of the TMEM allocation;
//   warpgroup 1      splits the landed f32 operands in place into hi (same buffer) and lo (the
//                    buffer 32 KB above it); the split is elementwise, so the swizzled layout
//                    carries over to the lo buffer unchanged;
//   warpgroup 2      epilogue: thread r loads row r of the chunk (128 columns) from TMEM; each
//                    warp then passes its 32 rows through shared memory 32 columns at a time, so
//                    that every store instruction writes whole 128-byte runs of a row.
// TMEM: two 128-column accumulators, so the epilogue of one chunk overlaps the next chunk's MMAs.
// Every wait is bounded (g_sa_wait_limit_ns) and drains what the role has in flight.
#pragma once
#include "k_attn_tc.cuh"

struct __align__(64) ScoreTcArgs {
    CUtensorMap tm_q;   // q_pool as [bh*nt][64] f32, box 32 x 128
    CUtensorMap tm_k;   // k_pool as [bh*nt][64] f32, box 32 x 128
    float* out;         // row (local head z, local row r) at out + (z * rows + r) * ldo
    int64_t ldo;
    int32_t nt;
    int32_t h0, i0, rows;  // heads h0 + blockIdx.z; query tiles [i0, i0 + rows)
    int32_t n_chunks;      // ceil(nt / 128)
    int32_t chunks_per_cta;
    int32_t vec_out;       // 1: ldo and out allow 16-byte stores
};

namespace stc {

constexpr int kAtomBytes = 128 * 128;          // 128 rows x 32 f32
constexpr int kTileBytes = 2 * kAtomBytes;     // 128 rows x 64 f32
constexpr int kA = 0;                          // A hi, then A lo
constexpr int kB = 2 * kTileBytes;             // [2 stages] B hi, then B lo
constexpr int kStage = kB + 2 * 2 * kTileBytes;  // epilogue staging: [4 warps][32 rows][36] f32
constexpr int kStageRow = 36;                      // floats per staged row (16-byte aligned, conflict-free)
constexpr int kBars = kStage + 4 * 32 * kStageRow * 4;
// a_full, a_ready, b_full[2], b_ready[2], b_empty[2], d_full[2], d_empty[2], drain
constexpr int kNumBars = 13;
constexpr int kMisc = kBars + 8 * kNumBars;    // tmem base, abort flag
constexpr int kEnd = kMisc + 16;
constexpr size_t kSmemBytes = 1024 + kEnd;
constexpr uint32_t kTmemCols = 256;
// D f32 (bit 4), A and B tf32 (format 2 at bits 7 and 10), both K-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ float tf32_rn(float x) {
    uint32_t y;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
    return __uint_as_float(y);
}

// In place: x -> hi at p, lo at p + kTileBytes (the next 32 KB), for one 128 x 64 f32 tile.
__device__ __forceinline__ void split_tile(uint8_t* p, int t) {
    float4* hi = reinterpret_cast<float4*>(p);
    float4* lo = reinterpret_cast<float4*>(p + kTileBytes);
#pragma unroll 4
    for (int v = t; v < kTileBytes / 16; v += 128) {
        const float4 x = hi[v];
        float4 h, l;
        h.x = tf32_rn(x.x); l.x = tf32_rn(x.x - h.x);
        h.y = tf32_rn(x.y); l.y = tf32_rn(x.y - h.y);
        h.z = tf32_rn(x.z); l.z = tf32_rn(x.z - h.z);
        h.w = tf32_rn(x.w); l.w = tf32_rn(x.w - h.w);
        hi[v] = h;
        lo[v] = l;
    }
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %4, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(acc), "r"(kIdesc)
        : "memory");
}

// One 32 x 32 piece of a warp's rows (row = lane's TMEM lane, 32 columns from column c0 of
// the launch's output rows): staged in the warp's shared buffer, then stored row by row.
// vec: 16-byte stores (8 lanes per row, 4 rows per instruction); else one float per lane.
__device__ __forceinline__ void store_piece(float* st, const uint32_t (&v)[32], float* out, int64_t ldo,
                                            int row0, int rows_valid, int c0, int cols_valid, bool vec, int lane) {
    float4* mine = reinterpret_cast<float4*>(st + lane * kStageRow);
#pragma unroll
    for (int u = 0; u < 8; ++u)
        mine[u] = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]), __uint_as_float(v[4 * u + 2]),
                              __uint_as_float(v[4 * u + 3]));
    __syncwarp();
    if (vec) {
        const int rr = lane >> 3, cc = 4 * (lane & 7);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = 4 * j + rr;
            if (row0 + r < rows_valid)
                *reinterpret_cast<float4*>(out + (int64_t)(row0 + r) * ldo + c0 + cc) =
                    *reinterpret_cast<const float4*>(st + r * kStageRow + cc);
        }
    } else {
        for (int r = 0; r < 32; ++r)
            if (row0 + r < rows_valid && lane < cols_valid) out[(int64_t)(row0 + r) * ldo + c0 + lane] = st[r * kStageRow + lane];
    }
    __syncwarp();
}

}  // namespace stc

__global__ void __launch_bounds__(384, 1) score_tc_kernel(const __grid_constant__ ScoreTcArgs a) {
    using namespace stc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBars);
    uint64_t* a_full = bars + 0;
    uint64_t* a_ready = bars + 1;
    uint64_t* b_full = bars + 2;   // [2]
    uint64_t* b_ready = bars + 4;  // [2]
    uint64_t* b_empty = bars + 6;  // [2]
    uint64_t* d_full = bars + 8;   // [2]
    uint64_t* d_empty = bars + 10; // [2]
    uint64_t* drain_bar = bars + 12;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(smem + kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = a.h0 + blockIdx.z;
    const int r0 = blockIdx.y * 128;                     // first local row of the tile
    const int c_begin = blockIdx.x * a.chunks_per_cta;   // first chunk of this CTA
    const int n_chunks = max(0, min(a.chunks_per_cta, a.n_chunks - c_begin));

    if (threadIdx.x == 0) {
        mbar_init(a_full, 1);
        mbar_init(a_ready, 128);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_ready[s], 128);
            mbar_init(&b_empty[s], 1);
            mbar_init(&d_full[s], 1);
            mbar_init(&d_empty[s], 128);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&a.tm_q);
        tma_prefetch_desc(&a.tm_k);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        const bool leader = tc::elect_one();
        const int32_t arow = h * a.nt + a.i0 + r0;
        uint32_t issued = 0;  // bit s: a load into stage s is in flight or landed
        uint32_t phases = 0;  // bit s: parity of that load
        bool ok = true;
        if (n_chunks > 0 && leader) {
            mbar_arrive_expect_tx(a_full, kTileBytes);
            tma_load_2d(smem + kA, &a.tm_q, a_full, 0, arow);
            tma_load_2d(smem + kA + kAtomBytes, &a.tm_q, a_full, 32, arow);
        }
        for (int n = 0; n < n_chunks; ++n) {
            const int s = n & 1;
            const uint32_t ph = (n >> 1) & 1;
            if (!mbar_wait_warp(&b_empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
            if (leader) {
                const int32_t brow = h * a.nt + (c_begin + n) * 128;
                uint8_t* dst = smem + kB + s * 2 * kTileBytes;
                mbar_arrive_expect_tx(&b_full[s], kTileBytes);
                tma_load_2d(dst, &a.tm_k, &b_full[s], 0, brow);
                tma_load_2d(dst + kAtomBytes, &a.tm_k, &b_full[s], 32, brow);
            }
            issued |= 1u << s;
            phases = (phases & ~(1u << s)) | (ph << s);
        }
        if (!ok) {  // every copy this warp started lands before the CTA exits
            for (int s = 0; s < 2; ++s)
                if ((issued >> s) & 1u) tc::drain_wait(&b_full[s], (phases >> s) & 1u);
            if (n_chunks > 0) tc::drain_wait(a_full, 0);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        const bool leader = tc::elect_one();
        bool ok = n_chunks == 0 || mbar_wait_warp(a_ready, 0, abort_flag);
        bool any_mma = false;
        tc_fence_after();
        const uint64_t da_hi = smem_desc_sw128(smem_u32(smem + kA), 16, 1024);
        const uint64_t da_lo = smem_desc_sw128(smem_u32(smem + kA + kTileBytes), 16, 1024);
        constexpr uint64_t kAtom = kAtomBytes >> 4;
        for (int n = 0; n < n_chunks && ok; ++n) {
            const int s = n & 1;
            const uint32_t ph = (n >> 1) & 1;
            if (!mbar_wait_warp(&b_ready[s], ph, abort_flag)) { ok = false; break; }
            if (!mbar_wait_warp(&d_empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (leader) {
                uint8_t* b = smem + kB + s * 2 * kTileBytes;
                const uint64_t db_hi = smem_desc_sw128(smem_u32(b), 16, 1024);
                const uint64_t db_lo = smem_desc_sw128(smem_u32(b + kTileBytes), 16, 1024);
                const uint32_t d = tmem + (uint32_t)(s * 128);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {  // K step: 8 tf32 = 32 bytes; 4 per atom
                    const uint64_t off = (uint64_t)(ks >> 2) * kAtom + 2 * (ks & 3);
                    stc::mma_tf32(d, da_lo + off, db_hi + off, ks > 0 ? 1u : 0u);  // small terms first
                    stc::mma_tf32(d, da_hi + off, db_lo + off, 1u);
                    stc::mma_tf32(d, da_hi + off, db_hi + off, 1u);
                }
                umma_commit(&b_empty[s]);
                umma_commit(&d_full[s]);
            }
            __syncwarp();
            any_mma = true;
        }
        if (any_mma) {  // every MMA (and its commits) finished before TMEM is released
            if (leader) umma_commit(drain_bar);
            __syncwarp();
            tc::drain_wait(drain_bar, 0);
        }
    }
    else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------------ operand split
        const int t = threadIdx.x - 128;
        bool ok = n_chunks == 0 || mbar_wait(a_full, 0, abort_flag);
        if (ok && n_chunks > 0) {
            split_tile(smem + kA, t);
            fence_proxy_async_smem();  // the tensor cores read what these threads wrote
            mbar_arrive(a_ready);
        }
        for (int n = 0; n < n_chunks && ok; ++n) {
            const int s = n & 1;
            const uint32_t ph = (n >> 1) & 1;
            if (!mbar_wait(&b_full[s], ph, abort_flag)) { ok = false; break; }
            split_tile(smem + kB + s * 2 * kTileBytes, t);
            fence_proxy_async_smem();
            mbar_arrive(&b_ready[s]);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------------ epilogue
        const int quad = warp & 3;               // rows quad*32 .. +31 of the tile = its TMEM lanes
        float* out_z = a.out + (int64_t)blockIdx.z * a.rows * a.ldo;  // row 0 of this head's rows
        float* st = reinterpret_cast<float*>(smem + kStage) + quad * 32 * kStageRow;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        bool ok = true;
        for (int n = 0; n < n_chunks && ok; ++n) {
            const int s = n & 1;
            const uint32_t ph = (n >> 1) & 1;
            if (!mbar_wait_warp(&d_full[s], ph, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t v0[32], v1[32], v2[32], v3[32];
            const uint32_t src = tmem + lane_off + (uint32_t)(s * 128);
            tmem_ld_32x32b_x32(src + 0, v0);
            tmem_ld_32x32b_x32(src + 32, v1);
            tmem_ld_32x32b_x32(src + 64, v2);
            tmem_ld_32x32b_x32(src + 96, v3);
            tmem_ld_wait(v0);
            reg_fence(v1);
            reg_fence(v2);
            reg_fence(v3);
            tc_fence_before();
            mbar_arrive(&d_empty[s]);  // the accumulator may be overwritten from here on
            const int c0 = (c_begin + n) * 128;
            const int valid = min(128, a.nt - c0);
            const bool vec = a.vec_out && valid == 128;
            const int row0 = r0 + quad * 32;  // first local row of this warp
            stc::store_piece(st, v0, out_z, a.ldo, row0, a.rows, c0, valid, vec, lane);
            stc::store_piece(st, v1, out_z, a.ldo, row0, a.rows, c0 + 32, valid - 32, vec, lane);
            stc::store_piece(st, v2, out_z, a.ldo, row0, a.rows, c0 + 64, valid - 64, vec, lane);
            stc::store_piece(st, v3, out_z, a.ldo, row0, a.rows, c0 + 96, valid - 96, vec, lane);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}
