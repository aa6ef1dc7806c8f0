// Step 2: tile scores s[h][i][j] = q_pool[h][i] . k_pool[h][j] ("SAF3R" abstract: rank the
// candidate interactions per head).
//
// SIMT f32: the ranking must be exact to about 1e-6 relative, which rules out a single-pass
// tf32/bf16 tensor-core product.  Every output accumulates its 64 products in ascending e with
// FMA.  Rows [i0, i0 + rows) of head h0 + blockIdx.z are written at
// out + (blockIdx.z * rows + local row) * ldo.
//   tile_scores_kernel      64 x 64 blocks, 4 x 4 per thread (small tile counts: more CTAs);
//   tile_scores_big_kernel  128 x 128 blocks, 8 x 8 per thread, operands transposed in shared
//                           memory so a thread reads its 8 + 8 operands as four 16-byte words,
//                           packed f32x2 FMAs (large tile counts).
#pragma once
#include "sa_device.cuh"

struct ScoreArgs {
    const float* q_pool;  // [bh][nt][64]
    const float* k_pool;  // [bh][nt][64]
    float* out;
    int64_t ldo;          // row stride of out (elements)
    int32_t nt;
    int32_t h0;           // first head of this launch
    int32_t i0;           // first query tile (row) of this launch
    int32_t rows;         // rows per head in this launch
};

__global__ void __launch_bounds__(256) tile_scores_kernel(ScoreArgs a) {
    __shared__ float qs[64][65];
    __shared__ float ks[64][65];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int h = a.h0 + blockIdx.z;
    const int r_blk = blockIdx.y * 64;  // local row block
    const int c_blk = blockIdx.x * 64;
    const float* qb = a.q_pool + ((int64_t)h * a.nt + a.i0) * 64;
    const float* kb = a.k_pool + (int64_t)h * a.nt * 64;
    for (int idx = threadIdx.x; idx < 64 * 16; idx += 256) {
        const int r = idx >> 4, c4 = idx & 15;
        float4 x = make_float4(0, 0, 0, 0), y = x;
        if (r_blk + r < a.rows) x = __ldg(reinterpret_cast<const float4*>(qb + (int64_t)(r_blk + r) * 64) + c4);
        if (c_blk + r < a.nt) y = __ldg(reinterpret_cast<const float4*>(kb + (int64_t)(c_blk + r) * 64) + c4);
        qs[r][4 * c4 + 0] = x.x; qs[r][4 * c4 + 1] = x.y; qs[r][4 * c4 + 2] = x.z; qs[r][4 * c4 + 3] = x.w;
        ks[r][4 * c4 + 0] = y.x; ks[r][4 * c4 + 1] = y.y; ks[r][4 * c4 + 2] = y.z; ks[r][4 * c4 + 3] = y.w;
    }
    __syncthreads();
    float acc[4][4] = {};
#pragma unroll 8
    for (int e = 0; e < 64; ++e) {
        float qv[4], kv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            qv[u] = qs[ty + 16 * u][e];
            kv[u] = ks[tx + 16 * u][e];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(qv[u], kv[w], acc[u][w]);
    }
    float* ob = a.out + (int64_t)blockIdx.z * a.rows * a.ldo;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int r = r_blk + ty + 16 * u;
        if (r >= a.rows) continue;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int c = c_blk + tx + 16 * w;
            if (c < a.nt) ob[(int64_t)r * a.ldo + c] = acc[u][w];
        }
    }
}

#define SCORES_BIG_SMEM (2 * 64 * 128 * 4)

// One 128 x 128 block of scores by the whole 256-thread CTA: rows qb[0 .. rows_valid) and
// columns kb[0 .. cols_valid) (each a [64] f32 mean), written to ob[r * ldo + c]; smem holds
// SCORES_BIG_SMEM bytes (qT, kT: [64][128]).  Starts and ends with the CTA converged; the
// caller synchronises before reusing smem.
__device__ __forceinline__ void score_block_128(const float* qb, int rows_valid, const float* kb, int cols_valid,
                                                float* ob, int64_t ldo, float* smem) {
    float* qT = smem;             // [64 e][128 rows]
    float* kT = smem + 64 * 128;  // [64 e][128 cols]
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    // consecutive lanes take consecutive rows, so the transposed shared-memory writes of a warp
    // fall into 32 different banks
    for (int idx = threadIdx.x; idx < 128 * 16; idx += 256) {
        const int r = idx & 127, c4 = idx >> 7;  // row r, elements 4 c4 .. 4 c4 + 3
        float4 x = make_float4(0, 0, 0, 0), y = x;
        if (r < rows_valid) x = __ldg(reinterpret_cast<const float4*>(qb + (int64_t)r * 64) + c4);
        if (r < cols_valid) y = __ldg(reinterpret_cast<const float4*>(kb + (int64_t)r * 64) + c4);
        qT[(4 * c4 + 0) * 128 + r] = x.x;
        qT[(4 * c4 + 1) * 128 + r] = x.y;
        qT[(4 * c4 + 2) * 128 + r] = x.z;
        qT[(4 * c4 + 3) * 128 + r] = x.w;
        kT[(4 * c4 + 0) * 128 + r] = y.x;
        kT[(4 * c4 + 1) * 128 + r] = y.y;
        kT[(4 * c4 + 2) * 128 + r] = y.z;
        kT[(4 * c4 + 3) * 128 + r] = y.w;
    }
    __syncthreads();
    float2 acc[8][4];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int p = 0; p < 4; ++p) acc[u][p] = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int e = 0; e < 64; ++e) {
        const float4 qa = *reinterpret_cast<const float4*>(qT + e * 128 + ty * 8);
        const float4 qc = *reinterpret_cast<const float4*>(qT + e * 128 + ty * 8 + 4);
        const float4 ka = *reinterpret_cast<const float4*>(kT + e * 128 + tx * 8);
        const float4 kc = *reinterpret_cast<const float4*>(kT + e * 128 + tx * 8 + 4);
        const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qc.x, qc.y, qc.z, qc.w};
        const float2 kv[4] = {make_float2(ka.x, ka.y), make_float2(ka.z, ka.w), make_float2(kc.x, kc.y),
                              make_float2(kc.z, kc.w)};
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int p = 0; p < 4; ++p) acc[u][p] = __ffma2_rn(make_float2(qv[u], qv[u]), kv[p], acc[u][p]);
    }
    const int c0 = tx * 8;
    const bool vec = ((ldo & 3) == 0) && (c0 + 8 <= cols_valid) && ((reinterpret_cast<uintptr_t>(ob) & 15u) == 0);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int r = ty * 8 + u;
        if (r >= rows_valid) continue;
        float* dst = ob + (int64_t)r * ldo + c0;
        if (vec) {
            reinterpret_cast<float4*>(dst)[0] = make_float4(acc[u][0].x, acc[u][0].y, acc[u][1].x, acc[u][1].y);
            reinterpret_cast<float4*>(dst)[1] = make_float4(acc[u][2].x, acc[u][2].y, acc[u][3].x, acc[u][3].y);
        } else {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                if (c0 + 2 * p < cols_valid) dst[2 * p] = acc[u][p].x;
                if (c0 + 2 * p + 1 < cols_valid) dst[2 * p + 1] = acc[u][p].y;
            }
        }
    }
}

// 128 x 128 block per 256-thread CTA; dynamic shared memory SCORES_BIG_SMEM (qT, kT: [64][128]).
__global__ void __launch_bounds__(256) tile_scores_big_kernel(ScoreArgs a) {
    extern __shared__ __align__(16) float big_smem[];
    const int h = a.h0 + blockIdx.z;
    const int r_blk = blockIdx.y * 128;
    const int c_blk = blockIdx.x * 128;
    const float* qb = a.q_pool + ((int64_t)h * a.nt + a.i0 + r_blk) * 64;
    const float* kb = a.k_pool + ((int64_t)h * a.nt + c_blk) * 64;
    float* ob = a.out + ((int64_t)blockIdx.z * a.rows + r_blk) * a.ldo + c_blk;
    score_block_128(qb, a.rows - r_blk, kb, a.nt - c_blk, ob, a.ldo, big_smem);
}
