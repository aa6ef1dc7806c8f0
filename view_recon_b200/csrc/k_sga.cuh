// Subsampled global attention ("AVGGT: Rethinking Global Attention for Accelerating VGGT",
// technical summary 2.B.2, SGA): keys and values are subsampled on each frame's 2-D patch grid
// (one token per s_h x s_w window), every query and every special token is kept, each token's
// own key (the diagonal) is kept, and the discarded columns are represented by one mean
// key/value pair weighted by their count.
//
// On the device this is three steps around the dense tensor-core attention:
//   sga_gather_kernel   compacts the kept K/V rows of every frame into one key sequence of
//                       S * (n_special + ceil(grid_h/s_h) * ceil(grid_w/s_w)) rows per head and
//                       sums the discarded K/V rows of each quarter frame in fp32;
//   sga_sum_kernel      adds the partial sums into one sum per head (fixed order);
//   (attention)         every query over the compacted keys: O and the natural-log LSE;
//   sga_combine_kernel  per query row, folds in the diagonal (for a query whose own token was
//                       discarded) and the mean pair of the other discarded columns:
//                       LSE' = log(e^LSE + e^a_d + e^a_m),
//                       O'   = e^(LSE-LSE') O + e^(a_d-LSE') v_t + e^(a_m-LSE') v_mean,
//                       a_d = scale q.k_t, a_m = scale q.k_mean + ln(count).
#pragma once
#include "sa_device.cuh"

struct SgaGeo {
    int32_t frames, tokens, n_special, grid_h, grid_w, s_h, s_w;
    int32_t kh, kw;  // kept grid rows / columns per frame: ceil(grid_h / s_h), ceil(grid_w / s_w)
    int32_t kpf;     // kept tokens per frame: n_special + kh * kw
};

#define SGA_SPLIT 4  // CTAs per frame in the gather

struct SgaGatherArgs {
    const uint32_t* k;  // [bh][L][32] bf16 pairs
    const uint32_t* v;
    uint32_t* ksub;     // [bh][Lk][32]
    uint32_t* vsub;
    float* part;        // [bh][S * SGA_SPLIT][2][64] partial sums of the discarded K (0) and V (1) rows
    int32_t L, Lk;
    SgaGeo g;
};

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

__device__ __forceinline__ void acc_bf16x8(float (&s)[16], int off, const uint4& w) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        s[off + 2 * i] += __uint_as_float(u[i] << 16);
        s[off + 2 * i + 1] += __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

// SGA_SPLIT CTAs of 8 warps per (frame, head); CTA q takes every SGA_SPLIT-th kept row and a
// contiguous quarter of the frame's patch tokens.  For the discarded sums a warp covers 8
// consecutive tokens per step: lane l reads elements [16 (l & 3), 16 (l & 3) + 16) of token
// l >> 2 as two 16-byte words of K and two of V, so every lane keeps four loads in flight.
__global__ void __launch_bounds__(256) sga_gather_kernel(SgaGatherArgs a) {
    __shared__ float red[8][2][64];
    const SgaGeo& g = a.g;
    const int f = blockIdx.x, q = blockIdx.y, h = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t)h * a.L + (int64_t)f * g.tokens;
    const int64_t out0 = (int64_t)h * a.Lk + (int64_t)f * g.kpf;
    // kept rows: the special tokens, then the grid positions (r * s_h, c * s_w) row-major
    for (int e = q * 8 + warp; e < g.kpf; e += 8 * SGA_SPLIT) {
        int n = e;
        if (e >= g.n_special) {
            const int p = e - g.n_special, rr = p / g.kw, cc = p - rr * g.kw;
            n = g.n_special + rr * g.s_h * g.grid_w + cc * g.s_w;
        }
        a.ksub[(out0 + e) * 32 + lane] = __ldg(a.k + (row0 + n) * 32 + lane);
        a.vsub[(out0 + e) * 32 + lane] = __ldg(a.v + (row0 + n) * 32 + lane);
    }
    // discarded rows of this CTA's quarter of the patch grid
    const int np = g.grid_h * g.grid_w;
    const int per = (np + SGA_SPLIT - 1) / SGA_SPLIT;
    const int p_lo = q * per, p_hi = min(np, p_lo + per);
    const int sub = lane >> 2, quarter = lane & 3;
    float sk[16], sv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) sk[i] = sv[i] = 0.f;
    for (int p0 = p_lo + warp * 8; p0 < p_hi; p0 += 64) {
        const int p = p0 + sub;
        bool take = p < p_hi;
        if (take) {
            const int r = p / g.grid_w, c = p - r * g.grid_w;
            take = !((r % g.s_h) == 0 && (c % g.s_w) == 0);
        }
        if (take) {
            const uint4* kr = reinterpret_cast<const uint4*>(a.k + (row0 + g.n_special + p) * 32) + 2 * quarter;
            const uint4* vr = reinterpret_cast<const uint4*>(a.v + (row0 + g.n_special + p) * 32) + 2 * quarter;
            const uint4 k0 = __ldg(kr), k1 = __ldg(kr + 1), v0 = __ldg(vr), v1 = __ldg(vr + 1);
            acc_bf16x8(sk, 0, k0);
            acc_bf16x8(sk, 8, k1);
            acc_bf16x8(sv, 0, v0);
            acc_bf16x8(sv, 8, v1);
        }
    }
    // lanes with the same quarter hold partial sums of the same 16 elements
#pragma unroll
    for (int off = 4; off < 32; off <<= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], off);
            sv[i] += __shfl_xor_sync(0xffffffffu, sv[i], off);
        }
    if (lane < 4) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            red[warp][0][16 * lane + i] = sk[i];
            red[warp][1][16 * lane + i] = sv[i];
        }
    }
    __syncthreads();
    if (threadIdx.x < 128) {
        const int kv = threadIdx.x >> 6, e = threadIdx.x & 63;
        float t = 0.f;
        for (int w = 0; w < 8; ++w) t += red[w][kv][e];
        a.part[(((int64_t)h * g.frames + f) * SGA_SPLIT + q) * 128 + threadIdx.x] = t;
    }
}

// sums[h][0 or 1][64] = sum over the S * SGA_SPLIT partial sums of head h, in a fixed order; one
// CTA of 128 threads per head.
__global__ void __launch_bounds__(128) sga_sum_kernel(const float* part, float* sums, int32_t parts) {
    const int h = blockIdx.x, i = threadIdx.x;  // i = kv * 64 + e
    float s = 0.f;
    for (int f = 0; f < parts; ++f) s += part[((int64_t)h * parts + f) * 128 + i];
    sums[(int64_t)h * 128 + i] = s;
}

struct SgaCombineArgs {
    const uint32_t* q;  // [bh][L][32] bf16 pairs
    const uint32_t* k;
    const uint32_t* v;
    uint32_t* o;             // in: attention over the kept keys; out: the layer's output
    const float* lse_in;     // [bh][L] natural-log LSE of that attention
    float* lse_out;          // [bh][L] or null
    const float* sums;       // [bh][2][64] sums of all discarded K / V rows
    int64_t rows;            // bh * L
    int32_t L, n_disc;       // discarded tokens over all frames
    float scale;
    SgaGeo g;
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

#define SGA_ROWS_PER_WARP 2

__device__ __forceinline__ float half_sum(float x) {  // sum over the 16 lanes of a half-warp
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

__device__ __forceinline__ float4 bf16x4_to_f4(uint2 u) {
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xFFFF0000u));
}

// One half-warp per query row (two rows per warp, four elements per lane), so each warp
// instruction serves two rows and a dot product needs four shuffles.
__global__ void __launch_bounds__(256) sga_combine_kernel(SgaCombineArgs a) {
    const int lane = threadIdx.x & 31, hl = lane & 15;
    const int64_t row = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * 2 + (lane >> 4);
    const bool valid = row < a.rows;
    const int64_t rr = valid ? row : a.rows - 1;  // the tail's idle half mirrors the last row
    const SgaGeo& g = a.g;
    const int h = (int)(rr / a.L);
    const int t = (int)(rr - (int64_t)h * a.L);
    const int n = t % g.tokens;
    bool kept = n < g.n_special;
    if (!kept) {
        const int p = n - g.n_special, r = p / g.grid_w, c = p - r * g.grid_w;
        kept = (r % g.s_h) == 0 && (c % g.s_w) == 0;
    }
    const uint2* q2p = reinterpret_cast<const uint2*>(a.q) + rr * 16 + hl;
    uint2* o2p = reinterpret_cast<uint2*>(a.o) + rr * 16 + hl;
    const float4 q4 = bf16x4_to_f4(__ldg(q2p));
    const float4 o4 = bf16x4_to_f4(*o2p);
    const float lse = a.lse_in[rr];
    const float4* sk4 = reinterpret_cast<const float4*>(a.sums + (int64_t)h * 128);
    float4 km = __ldg(sk4 + hl), vm = __ldg(sk4 + 16 + hl);
    float4 vt = make_float4(0.f, 0.f, 0.f, 0.f);
    float a_d = -INFINITY;
    int cnt = a.n_disc;
    if (!kept) {  // the diagonal is kept on its own; the mean pair covers the other discarded columns
        const float4 kt = bf16x4_to_f4(__ldg(reinterpret_cast<const uint2*>(a.k) + rr * 16 + hl));
        vt = bf16x4_to_f4(__ldg(reinterpret_cast<const uint2*>(a.v) + rr * 16 + hl));
        a_d = q4.x * kt.x + q4.y * kt.y + q4.z * kt.z + q4.w * kt.w;
        km.x -= kt.x; km.y -= kt.y; km.z -= kt.z; km.w -= kt.w;
        vm.x -= vt.x; vm.y -= vt.y; vm.z -= vt.z; vm.w -= vt.w;
        cnt -= 1;
    }
    const float inv = cnt > 0 ? 1.0f / (float)cnt : 0.0f;
    const float dm = (q4.x * km.x + q4.y * km.y + q4.z * km.z + q4.w * km.w) * inv;
    // both half-warps reduce together (the two rows of a warp may differ in `kept`)
    const float sd = half_sum(kept ? 0.0f : a_d);
    const float sm = half_sum(dm);
    const float ad = kept ? -INFINITY : a.scale * sd;
    const float am = cnt > 0 ? a.scale * sm + logf((float)cnt) : -INFINITY;
    const float mx = fmaxf(lse, fmaxf(ad, am));
    const float w0 = expf(lse - mx), wd = expf(ad - mx), wm = expf(am - mx);
    const float tot = w0 + wd + wm;
    const float f0 = w0 / tot, fd = wd / tot, fm = wm * inv / tot;
    if (valid) {
        uint2 out;
        out.x = pack_bf16x2(f0 * o4.x + fd * vt.x + fm * vm.x, f0 * o4.y + fd * vt.y + fm * vm.y);
        out.y = pack_bf16x2(f0 * o4.z + fd * vt.z + fm * vm.z, f0 * o4.w + fd * vt.w + fm * vm.w);
        *o2p = out;
        if (a.lse_out && hl == 0) a.lse_out[row] = mx + logf(tot);
    }
}
