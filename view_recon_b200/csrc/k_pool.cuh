// Step 1: tile pooling ("Zebra3D" abstract: tile summaries; "AVGGT" 2.B.2: mean key/value).
//
// A tile's rows are contiguous in memory and are streamed with 128-bit read-only loads, 512
// contiguous bytes per warp instruction for bf16 (4 rows of 64 elements), accumulated in f32
// registers and reduced with shuffles (bf16: four warps per tile; f32: one warp per tile).
// HBM bound: every byte of Q and K (and V in landmark mode) is read exactly once.
#pragma once
#include "sa_device.cuh"

struct PoolArgs {
    const void* q;
    const void* k;
    const void* v;  // may be null; pooled only when v_pool is set, copied to sink_v when that is set
    float* q_pool;
    float* k_pool;
    float* v_pool;  // null unless v
    int32_t* k_cnt;
    void* sink_k;
    void* sink_v;
    int32_t bh, frames, tokens, tile, n_sink, tpf, nt;
};

__device__ __forceinline__ void bf16x8_accum(const uint4& u, float (&acc)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// d = 64, bf16: one 128-thread CTA per (head, tile).  Warp w sums rows [w*T/4, (w+1)*T/4) of the
// tile, lane = (row group r4 in 0..3, 16-byte chunk c in 0..7), every load of its rows in flight at
// once (8 per tensor at T = 128); the four warps' partial sums meet in shared memory and are added
// in warp order (deterministic).
__global__ void __launch_bounds__(128) pool_tiles_bf16_kernel(PoolArgs a) {
    __shared__ float part[3][4][64];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y, j = blockIdx.x;
    const int f = j / a.tpf, slot = j % a.tpf;
    const int n0 = slot * a.tile;
    const int nq = min(a.tile, a.tokens - n0);
    const int lo = min(nq, max(0, a.n_sink - n0));  // first key row inside the tile
    const int64_t row0 = (int64_t)h * a.frames * a.tokens + (int64_t)f * a.tokens + n0;
    const int c = lane & 7, r4 = lane >> 3;
    const int per_warp = a.tile / 4;  // 32 or 16 rows
    const int rw0 = warp * per_warp;
    const uint4* q4 = reinterpret_cast<const uint4*>(a.q) + row0 * 8 + c;
    const uint4* k4 = reinterpret_cast<const uint4*>(a.k) + row0 * 8 + c;
    const uint4* v4 = a.v_pool ? reinterpret_cast<const uint4*>(a.v) + row0 * 8 + c : nullptr;
    float sq[8] = {}, sk[8] = {}, sv[8] = {};
    uint4 uq[8], uk[8], uv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int r = rw0 + r4 + 4 * u;
        const bool in = 4 * u < per_warp && r < nq;
        uq[u] = in ? __ldg(q4 + (int64_t)r * 8) : make_uint4(0, 0, 0, 0);
        uk[u] = (in && r >= lo) ? __ldg(k4 + (int64_t)r * 8) : make_uint4(0, 0, 0, 0);
        uv[u] = (v4 && in && r >= lo) ? __ldg(v4 + (int64_t)r * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        bf16x8_accum(uq[u], sq);
        bf16x8_accum(uk[u], sk);
        if (v4) bf16x8_accum(uv[u], sv);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        sq[e] += __shfl_xor_sync(0xffffffffu, sq[e], 8);
        sq[e] += __shfl_xor_sync(0xffffffffu, sq[e], 16);
        sk[e] += __shfl_xor_sync(0xffffffffu, sk[e], 8);
        sk[e] += __shfl_xor_sync(0xffffffffu, sk[e], 16);
        sv[e] += __shfl_xor_sync(0xffffffffu, sv[e], 8);
        sv[e] += __shfl_xor_sync(0xffffffffu, sv[e], 16);
    }
    if (lane < 8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            part[0][warp][8 * c + e] = sq[e];
            part[1][warp][8 * c + e] = sk[e];
            part[2][warp][8 * c + e] = sv[e];
        }
    }
    __syncthreads();
    const int nk = nq - lo;
    if (threadIdx.x < 64) {
        const int d = threadIdx.x;
        const float iq = 1.0f / (float)nq;
        const float ik = nk > 0 ? 1.0f / (float)nk : 0.0f;
        const int64_t o = ((int64_t)h * a.nt + j) * 64 + d;
        a.q_pool[o] = (((part[0][0][d] + part[0][1][d]) + part[0][2][d]) + part[0][3][d]) * iq;
        a.k_pool[o] = (((part[1][0][d] + part[1][1][d]) + part[1][2][d]) + part[1][3][d]) * ik;
        if (a.v_pool) a.v_pool[o] = (((part[2][0][d] + part[2][1][d]) + part[2][2][d]) + part[2][3][d]) * ik;
    }
    if (h == 0 && threadIdx.x == 0) a.k_cnt[j] = nk;
    // sink rows of this tile (only tiles that start before n_sink hold any)
    if (lo > 0 && a.sink_k) {
        const int64_t srow0 = (int64_t)h * a.frames * a.n_sink + (int64_t)f * a.n_sink + n0;
        for (int idx = threadIdx.x; idx < lo * 8; idx += 128) {
            const int rr = idx >> 3, cc = idx & 7;
            reinterpret_cast<uint4*>(a.sink_k)[(srow0 + rr) * 8 + cc] =
                __ldg(reinterpret_cast<const uint4*>(a.k) + (row0 + rr) * 8 + cc);
            if (a.v && a.sink_v)
                reinterpret_cast<uint4*>(a.sink_v)[(srow0 + rr) * 8 + cc] =
                    __ldg(reinterpret_cast<const uint4*>(a.v) + (row0 + rr) * 8 + cc);
        }
    }
}

// d = 64, f32: lane = (row pair r2 in 0..1, 16-byte chunk c in 0..15).
__global__ void __launch_bounds__(256) pool_tiles_f32_kernel(PoolArgs a) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= a.bh * a.nt) return;
    const int h = warp / a.nt, j = warp % a.nt;
    const int f = j / a.tpf, slot = j % a.tpf;
    const int n0 = slot * a.tile;
    const int nq = min(a.tile, a.tokens - n0);
    const int lo = min(nq, max(0, a.n_sink - n0));
    const int64_t row0 = (int64_t)h * a.frames * a.tokens + (int64_t)f * a.tokens + n0;
    const int c = lane & 15, r2 = lane >> 4;
    const float4* q4 = reinterpret_cast<const float4*>(a.q) + row0 * 16 + c;
    const float4* k4 = reinterpret_cast<const float4*>(a.k) + row0 * 16 + c;
    const float4* v4 = a.v_pool ? reinterpret_cast<const float4*>(a.v) + row0 * 16 + c : nullptr;
    float4 sq = make_float4(0, 0, 0, 0), sk = sq, sv = sq;
    for (int r = r2; r < nq; r += 2) {
        const float4 x = __ldg(q4 + (int64_t)r * 16);
        sq.x += x.x; sq.y += x.y; sq.z += x.z; sq.w += x.w;
        if (r >= lo) {
            const float4 y = __ldg(k4 + (int64_t)r * 16);
            sk.x += y.x; sk.y += y.y; sk.z += y.z; sk.w += y.w;
            if (v4) {
                const float4 z = __ldg(v4 + (int64_t)r * 16);
                sv.x += z.x; sv.y += z.y; sv.z += z.z; sv.w += z.w;
            }
        }
    }
    sq.x += __shfl_xor_sync(0xffffffffu, sq.x, 16); sq.y += __shfl_xor_sync(0xffffffffu, sq.y, 16);
    sq.z += __shfl_xor_sync(0xffffffffu, sq.z, 16); sq.w += __shfl_xor_sync(0xffffffffu, sq.w, 16);
    sk.x += __shfl_xor_sync(0xffffffffu, sk.x, 16); sk.y += __shfl_xor_sync(0xffffffffu, sk.y, 16);
    sk.z += __shfl_xor_sync(0xffffffffu, sk.z, 16); sk.w += __shfl_xor_sync(0xffffffffu, sk.w, 16);
    sv.x += __shfl_xor_sync(0xffffffffu, sv.x, 16); sv.y += __shfl_xor_sync(0xffffffffu, sv.y, 16);
    sv.z += __shfl_xor_sync(0xffffffffu, sv.z, 16); sv.w += __shfl_xor_sync(0xffffffffu, sv.w, 16);
    const int nk = nq - lo;
    if (lane < 16) {
        const float iq = 1.0f / (float)nq;
        const float ik = nk > 0 ? 1.0f / (float)nk : 0.0f;
        const int64_t o = ((int64_t)h * a.nt + j) * 64 + 4 * c;
        *reinterpret_cast<float4*>(a.q_pool + o) = make_float4(sq.x * iq, sq.y * iq, sq.z * iq, sq.w * iq);
        *reinterpret_cast<float4*>(a.k_pool + o) = make_float4(sk.x * ik, sk.y * ik, sk.z * ik, sk.w * ik);
        if (a.v_pool)
            *reinterpret_cast<float4*>(a.v_pool + o) = make_float4(sv.x * ik, sv.y * ik, sv.z * ik, sv.w * ik);
    }
    if (h == 0 && lane == 0) a.k_cnt[j] = nk;
    if (lo > 0 && a.sink_k) {
        const int64_t srow0 = (int64_t)h * a.frames * a.n_sink + (int64_t)f * a.n_sink + n0;
        for (int idx = lane; idx < lo * 16; idx += 32) {
            const int rr = idx >> 4, cc = idx & 15;
            reinterpret_cast<float4*>(a.sink_k)[(srow0 + rr) * 16 + cc] =
                __ldg(reinterpret_cast<const float4*>(a.k) + (row0 + rr) * 16 + cc);
            if (a.v && a.sink_v)
                reinterpret_cast<float4*>(a.sink_v)[(srow0 + rr) * 16 + cc] =
                    __ldg(reinterpret_cast<const float4*>(a.v) + (row0 + rr) * 16 + cc);
        }
    }
}
