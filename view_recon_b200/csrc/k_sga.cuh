// Subsampled global attention ("AVGGT: Rethinking Global Attention for Accelerating VGGT",
// technical summary 2.B.2, SGA): keys and values are subsampled on each frame's 2-D patch grid
// (one token per s_h x s_w window), every query and every special token is kept, each token's
// own key (the diagonal) is kept, and the discarded columns are represented by one mean
// key/value pair weighted by their count.
//
// On the device this is three steps around the dense tensor-core attention:
//   sga_gather_kernel   compacts the kept K/V rows of every frame into one key sequence of
//                       S * (n_special + ceil(grid_h/s_h) * ceil(grid_w/s_w)) rows per head and
//                       sums each frame's discarded K/V rows in fp32;
//   sga_sum_kernel      adds the per-frame sums into one sum per head (fixed order);
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

struct SgaGatherArgs {
    const uint32_t* k;  // [bh][L][32] bf16 pairs
    const uint32_t* v;
    uint32_t* ksub;     // [bh][Lk][32]
    uint32_t* vsub;
    float* part;        // [bh][S][2][64] per-frame sums of the discarded K (0) and V (1) rows
    int32_t L, Lk;
    SgaGeo g;
};

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// One CTA of 8 warps per (frame, head).  A token row (64 bf16) is one 4-byte word per lane.
__global__ void __launch_bounds__(256) sga_gather_kernel(SgaGatherArgs a) {
    __shared__ float2 red[8][2][32];
    const SgaGeo& g = a.g;
    const int f = blockIdx.x, h = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t)h * a.L + (int64_t)f * g.tokens;
    const int64_t out0 = (int64_t)h * a.Lk + (int64_t)f * g.kpf;
    // kept rows: the special tokens, then the grid positions (r * s_h, c * s_w) row-major
    for (int e = warp; e < g.kpf; e += 8) {
        int n = e;
        if (e >= g.n_special) {
            const int p = e - g.n_special, rr = p / g.kw, cc = p - rr * g.kw;
            n = g.n_special + rr * g.s_h * g.grid_w + cc * g.s_w;
        }
        a.ksub[(out0 + e) * 32 + lane] = __ldg(a.k + (row0 + n) * 32 + lane);
        a.vsub[(out0 + e) * 32 + lane] = __ldg(a.v + (row0 + n) * 32 + lane);
    }
    // discarded rows: warp w sums grid rows w, w + 8, ...
    float2 sk = make_float2(0.f, 0.f), sv = make_float2(0.f, 0.f);
    for (int r = warp; r < g.grid_h; r += 8) {
        const bool row_on_grid = (r % g.s_h) == 0;
        const int64_t t0 = row0 + g.n_special + (int64_t)r * g.grid_w;
        int cm = 0;  // c mod s_w
        for (int c = 0; c < g.grid_w; ++c) {
            if (!(row_on_grid && cm == 0)) {
                const float2 kv = bf16x2_to_f2(__ldg(a.k + (t0 + c) * 32 + lane));
                const float2 vv = bf16x2_to_f2(__ldg(a.v + (t0 + c) * 32 + lane));
                sk.x += kv.x;
                sk.y += kv.y;
                sv.x += vv.x;
                sv.y += vv.y;
            }
            if (++cm == g.s_w) cm = 0;
        }
    }
    red[warp][0][lane] = sk;
    red[warp][1][lane] = sv;
    __syncthreads();
    if (warp < 2) {
        float2 s = make_float2(0.f, 0.f);
        for (int w = 0; w < 8; ++w) {
            s.x += red[w][warp][lane].x;
            s.y += red[w][warp][lane].y;
        }
        float* dst = a.part + (((int64_t)h * g.frames + f) * 2 + warp) * 64;
        dst[2 * lane] = s.x;
        dst[2 * lane + 1] = s.y;
    }
}

// sums[h][0 or 1][64] = sum over frames of part[h][f][0 or 1][64]; one CTA of 128 threads per head.
__global__ void __launch_bounds__(128) sga_sum_kernel(const float* part, float* sums, int32_t frames) {
    const int h = blockIdx.x, i = threadIdx.x;  // i = kv * 64 + e
    float s = 0.f;
    for (int f = 0; f < frames; ++f) s += part[((int64_t)h * frames + f) * 128 + i];
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

// One warp per query row.
__global__ void __launch_bounds__(256) sga_combine_kernel(SgaCombineArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= a.rows) return;
    const SgaGeo& g = a.g;
    const int h = (int)(row / a.L);
    const int t = (int)(row - (int64_t)h * a.L);
    const int n = t % g.tokens;
    bool kept = n < g.n_special;
    if (!kept) {
        const int p = n - g.n_special, r = p / g.grid_w, c = p - r * g.grid_w;
        kept = (r % g.s_h) == 0 && (c % g.s_w) == 0;
    }
    const float2 q2 = bf16x2_to_f2(__ldg(a.q + row * 32 + lane));
    const float2 o2 = bf16x2_to_f2(a.o[row * 32 + lane]);
    const float lse = a.lse_in[row];
    const float* sk = a.sums + (int64_t)h * 128;
    float2 km = make_float2(sk[2 * lane], sk[2 * lane + 1]);
    float2 vm = make_float2(sk[64 + 2 * lane], sk[64 + 2 * lane + 1]);
    float2 vt = make_float2(0.f, 0.f);
    float a_d = -INFINITY;
    int cnt = a.n_disc;
    if (!kept) {  // the diagonal is kept on its own; the mean pair covers the other discarded columns
        const float2 kt = bf16x2_to_f2(__ldg(a.k + row * 32 + lane));
        vt = bf16x2_to_f2(__ldg(a.v + row * 32 + lane));
        a_d = a.scale * warp_sum(q2.x * kt.x + q2.y * kt.y);
        km.x -= kt.x;
        km.y -= kt.y;
        vm.x -= vt.x;
        vm.y -= vt.y;
        cnt -= 1;
    }
    float a_m = -INFINITY;
    if (cnt > 0) {
        const float inv = 1.0f / (float)cnt;
        km.x *= inv;
        km.y *= inv;
        vm.x *= inv;
        vm.y *= inv;
        a_m = a.scale * warp_sum(q2.x * km.x + q2.y * km.y) + logf((float)cnt);
    }
    const float mx = fmaxf(lse, fmaxf(a_d, a_m));
    const float w0 = expf(lse - mx), wd = expf(a_d - mx), wm = expf(a_m - mx);
    const float tot = w0 + wd + wm;
    const float inv_tot = 1.0f / tot;
    const float ox = (w0 * o2.x + wd * vt.x + wm * vm.x) * inv_tot;
    const float oy = (w0 * o2.y + wd * vt.y + wm * vm.y) * inv_tot;
    a.o[row * 32 + lane] = pack_bf16x2(ox, oy);
    if (a.lse_out && lane == 0) a.lse_out[row] = mx + logf(tot);
}
