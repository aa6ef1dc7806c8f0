// Per-head budgets from an online statistic of the head's pooled scores ("SAF3R" abstract:
// sparsity differs from head to head and is adapted online, per head).
//
// For query tile i of head h, H_i is the entropy of softmax(temperature * s_ij) over the
// candidate tiles j (other frames, with at least one key row); the head's statistic is the
// mean perplexity P_h = (1/nt) sum_i exp(H_i) (0 for a tile without candidates) and its budget
//     k_h = min(k_hi, max(k_lo, floor(beta * P_h + 1/2))).
//
// head_stat_kernel: one 256-thread CTA per (128 query tiles, head) walks every 128-column block
// of key tiles.  The scores are f32 FMA chains over e ascending, in 8 x 8 register blocks; each thread keeps, for its 8 rows, the running triple
//     m = max x,  Z = sum exp(x - m),  A = sum (x - m) exp(x - m)        (x = temperature * s)
// so that H = ln Z - A / Z without a second pass.  The 16 threads sharing a row merge their
// triples in a fixed order and the row's perplexity exp(H) lands in the workspace.
// head_budget_kernel: one CTA per head sums its rows' perplexities in a fixed order (f64) and
// writes k_h (and P_h).  Both kernels are deterministic.
#pragma once
#include "sa_device.cuh"

struct BudgetArgs {
    const float* q_pool;  // [bh][nt][64]
    const float* k_pool;  // [bh][nt][64]
    float* row_perp;      // [bh][nt] workspace
    int32_t* k_per_head;  // [bh]
    float* perp_out;      // [bh] or null
    int32_t nt, tpf, tile, tokens, n_sink;
    float temperature, beta;
    int32_t k_lo, k_hi;
};

#define BUDGET_SMEM (2 * 64 * 128 * 4)

struct EntTriple {
    float m, z, a;
};

// Rescales the triple to a new maximum m_new >= t.m (m = -inf means empty).
__device__ __forceinline__ void ent_rescale(EntTriple& t, float m_new) {
    if (t.m == -INFINITY) {
        t.z = 0.0f;
        t.a = 0.0f;
    } else {
        const float d = t.m - m_new;  // <= 0
        const float f = expf(d);
        t.a = (t.a + d * t.z) * f;
        t.z *= f;
    }
    t.m = m_new;
}

__device__ __forceinline__ EntTriple ent_merge(EntTriple x, EntTriple y) {
    const float m = fmaxf(x.m, y.m);
    if (m == -INFINITY) return x;
    ent_rescale(x, m);
    ent_rescale(y, m);
    x.z += y.z;
    x.a += y.a;
    return x;
}

__device__ __forceinline__ bool slot_has_keys(int slot, int tile, int tokens, int n_sink) {
    const int n0 = slot * tile;
    const int nq = min(tile, tokens - n0);
    return nq > min(nq, max(0, n_sink - n0));
}

__global__ void __launch_bounds__(256) head_stat_kernel(BudgetArgs a) {
    extern __shared__ __align__(16) float bud_smem[];
    float* qT = bud_smem;             // [64 e][128 rows]
    float* kT = bud_smem + 64 * 128;  // [64 e][128 cols]
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int h = blockIdx.y;
    const int r_blk = blockIdx.x * 128;
    const float* qb = a.q_pool + (int64_t)h * a.nt * 64;
    const float* kb = a.k_pool + (int64_t)h * a.nt * 64;
    for (int idx = threadIdx.x; idx < 128 * 16; idx += 256) {
        const int r = idx & 127, c4 = idx >> 7;
        float4 x = make_float4(0, 0, 0, 0);
        if (r_blk + r < a.nt) x = __ldg(reinterpret_cast<const float4*>(qb + (int64_t)(r_blk + r) * 64) + c4);
        qT[(4 * c4 + 0) * 128 + r] = x.x;
        qT[(4 * c4 + 1) * 128 + r] = x.y;
        qT[(4 * c4 + 2) * 128 + r] = x.z;
        qT[(4 * c4 + 3) * 128 + r] = x.w;
    }
    int frame_of_row[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) frame_of_row[u] = (r_blk + ty * 8 + u) / a.tpf;
    EntTriple t[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) t[u] = {-INFINITY, 0.0f, 0.0f};

    for (int c_blk = 0; c_blk < a.nt; c_blk += 128) {
        __syncthreads();  // the previous block's kT reads are done
        for (int idx = threadIdx.x; idx < 128 * 16; idx += 256) {
            const int r = idx & 127, c4 = idx >> 7;
            float4 y = make_float4(0, 0, 0, 0);
            if (c_blk + r < a.nt) y = __ldg(reinterpret_cast<const float4*>(kb + (int64_t)(c_blk + r) * 64) + c4);
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
        // candidate columns of this thread: c = c_blk + tx * 8 + v
        int col_frame[8];
        bool col_ok[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int c = c_blk + tx * 8 + v;
            col_frame[v] = c / a.tpf;
            col_ok[v] = c < a.nt && slot_has_keys(c - col_frame[v] * a.tpf, a.tile, a.tokens, a.n_sink);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float xv[8];
            float mb = -INFINITY;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                xv[2 * p] = a.temperature * acc[u][p].x;
                xv[2 * p + 1] = a.temperature * acc[u][p].y;
            }
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const bool cand = col_ok[v] && col_frame[v] != frame_of_row[u];
                xv[v] = cand ? xv[v] : -INFINITY;
                mb = fmaxf(mb, xv[v]);
            }
            if (mb == -INFINITY) continue;
            if (mb > t[u].m) ent_rescale(t[u], mb);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                if (xv[v] == -INFINITY) continue;
                const float d = xv[v] - t[u].m;
                const float ev = expf(d);
                t[u].z += ev;
                t[u].a = fmaf(d, ev, t[u].a);
            }
        }
    }
    // merge the 16 column groups of every row: lanes tx = 0..15 of one half-warp, fixed order
#pragma unroll
    for (int u = 0; u < 8; ++u) {
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) {
            EntTriple o;
            o.m = __shfl_xor_sync(0xffffffffu, t[u].m, off);
            o.z = __shfl_xor_sync(0xffffffffu, t[u].z, off);
            o.a = __shfl_xor_sync(0xffffffffu, t[u].a, off);
            // both partners combine (lower tx first) so that they hold the same triple
            t[u] = (tx & off) ? ent_merge(o, t[u]) : ent_merge(t[u], o);
        }
    }
    if (tx == 0) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = r_blk + ty * 8 + u;
            if (i >= a.nt) continue;
            const float p = t[u].z > 0.0f ? expf(logf(t[u].z) - t[u].a / t[u].z) : 0.0f;
            a.row_perp[(int64_t)h * a.nt + i] = p;
        }
    }
}

__global__ void __launch_bounds__(256) head_budget_kernel(BudgetArgs a) {
    __shared__ double part[256];
    const int h = blockIdx.x;
    const float* rp = a.row_perp + (int64_t)h * a.nt;
    double s = 0.0;
    for (int i = threadIdx.x; i < a.nt; i += 256) s += (double)rp[i];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double perp = part[0] / (double)a.nt;
        double k = floor((double)a.beta * perp + 0.5);
        k = fmin((double)a.k_hi, fmax((double)a.k_lo, k));
        a.k_per_head[h] = (int32_t)k;
        if (a.perp_out) a.perp_out[h] = (float)perp;
    }
}
