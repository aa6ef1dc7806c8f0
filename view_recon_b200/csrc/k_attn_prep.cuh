// Operand preparation for the tensor-core attention kernel.
//
// The P.V product reads V as its B operand.  Staged as loaded ([keys][dims], dims
// contiguous) V is an MN-major operand, and tcgen05.mma then costs about 132 cycles per
// K=16 step at N = 64 -- a quarter of the tensor pipe's rate.  K-major (Vt = [dims][keys],
// keys contiguous) it costs 72.  These kernels therefore write, once per call, every
// 128-key tile the attention kernel may gather as a transposed [64][128] bf16 block in the
// workspace (rows of the tile past its valid range are zero), plus the landmark tables.
// They are HBM-bound copies: one read and one write of V (and of the small pooled tables).
#pragma once
#include "sa_device.cuh"

// Tile t of head h covers rows [start, start + valid) of the source [rows][64] matrix.
//   frame mode (frame-aligned key tiles): t = (frame, slot), start = h*L + f*N + slot*128
//   flat mode: start = h*rows_per_head + t*128
struct VtArgs {
    const __nv_bfloat16* src;
    __nv_bfloat16* dst;  // [bh][tiles_per_head][64][128]
    int32_t tiles_per_head;
    int32_t frame_mode;
    int32_t tokens, tpf, L;  // frame mode
    int32_t rows_per_head;   // flat mode
};

__global__ void __launch_bounds__(256) vtile_transpose_kernel(VtArgs a) {
    __shared__ uint32_t s[128][33];  // 128 keys x 64 dims as bf16 pairs, padded
    const int t = blockIdx.x, h = blockIdx.y;
    int64_t start;
    int valid;
    if (a.frame_mode) {
        const int f = t / a.tpf, slot = t % a.tpf;
        start = (int64_t)h * a.L + (int64_t)f * a.tokens + slot * 128;
        valid = min(128, a.tokens - slot * 128);
    } else {
        start = (int64_t)h * a.rows_per_head + (int64_t)t * 128;
        valid = min(128, a.rows_per_head - t * 128);
    }
    const uint4* src = reinterpret_cast<const uint4*>(a.src + start * 64);
    for (int i = threadIdx.x; i < 128 * 8; i += 256) {  // 8 x 16 B per key row
        const int key = i >> 3, c = i & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (key < valid) v = __ldg(src + (int64_t)key * 8 + c);
        s[key][4 * c + 0] = v.x;
        s[key][4 * c + 1] = v.y;
        s[key][4 * c + 2] = v.z;
        s[key][4 * c + 3] = v.w;
    }
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(a.dst + ((int64_t)h * a.tiles_per_head + t) * 64 * 128);
    for (int p = threadIdx.x; p < 64 * 8; p += 256) {  // (dim, 16-key group): one 32-byte sector
        const int d = p & 63, kg = p >> 6;
        uint32_t w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t lo = s[16 * kg + 2 * u][d >> 1], hi = s[16 * kg + 2 * u + 1][d >> 1];
            const uint32_t a0 = (d & 1) ? (lo >> 16) : (lo & 0xFFFFu);
            const uint32_t a1 = (d & 1) ? (hi >> 16) : (hi & 0xFFFFu);
            w[u] = a0 | (a1 << 16);
        }
        dst[(int64_t)d * 16 + 2 * kg] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[(int64_t)d * 16 + 2 * kg + 1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

// Landmark tables: row-major bf16 copies of the key tile means (zero past nt), the value
// tile means as transposed [64][128] blocks per 128-tile chunk, and the per-tile logit bias
// log2(c_j) in base-2 units (-inf where c_j = 0 or j >= nt).
__global__ void landmark_prep_kernel(const float* k_pool, const float* v_pool, const int32_t* k_cnt,
                                     __nv_bfloat16* lk, __nv_bfloat16* lvt, float* lbias2, int32_t bh, int32_t nt,
                                     int32_t ntp) {
    const int64_t n4 = (int64_t)bh * ntp * 16;  // float4 groups of the key table
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n4;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t rowp = idx >> 4;  // h * ntp + j
        const int c4 = (int)(idx & 15);
        const int64_t h = rowp / ntp, j = rowp % ntp;
        float4 x = make_float4(0, 0, 0, 0);
        if (j < nt) x = __ldg(reinterpret_cast<const float4*>(k_pool + (h * nt + j) * 64) + c4);
        uint2 px;
        px.x = pack_bf16x2(x.x, x.y);
        px.y = pack_bf16x2(x.z, x.w);
        reinterpret_cast<uint2*>(lk)[idx] = px;
        if (h == 0 && c4 == 0) {
            const int c = j < nt ? k_cnt[j] : 0;
            lbias2[j] = c > 0 ? log2f((float)c) : -INFINITY;
        }
    }
    const int64_t nchunks = ntp / 128;
    const int64_t nv = (int64_t)bh * nchunks * 64 * 16;  // (h, chunk, dim, 8-key group)
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < nv;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int kg = (int)(idx & 15);
        const int d = (int)((idx >> 4) & 63);
        const int64_t hc = idx >> 10;  // h * nchunks + chunk
        const int64_t h = hc / nchunks, ch = hc % nchunks;
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float e[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int64_t j = ch * 128 + 8 * kg + 2 * u + q;
                e[q] = j < nt ? __ldg(v_pool + (h * nt + j) * 64 + d) : 0.0f;
            }
            w[u] = pack_bf16x2(e[0], e[1]);
        }
        reinterpret_cast<uint4*>(lvt)[(hc * 64 + d) * 16 + kg] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}
