// Step 2: tile scores s[h][i][j] = q_pool[h][i] . k_pool[h][j] ("SAF3R" abstract: rank the
// candidate interactions per head).
//
// SIMT f32: the ranking must be exact to about 1e-6 relative, which rules out a single-pass
// tf32/bf16 tensor-core product.  A 256-thread CTA computes a 64 x 64 block of one head with
// both 64 x 64 operand blocks staged in shared memory; every thread owns a 4 x 4 sub-block
// and accumulates the 64 products in ascending e with FMA.  Rows [i0, i0 + rows) of head
// h0 + blockIdx.z are written at out + (blockIdx.z * rows + local row) * ldo.
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
