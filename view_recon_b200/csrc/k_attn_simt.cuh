// Step 4 on CUDA cores: block-sparse (or dense) attention forward with an exact f32
// online softmax, one thread per query row.
//
// This instantiation serves the f32 workloads and tile = 64 (the tensor-core kernel is
// built for bf16 with tile = 128).  A CTA owns one query tile; key/value rows of every
// attended item (listed tile, sink chunk, landmark chunk) are staged in shared memory as
// f32, and each thread folds them into its running (max, sum, accumulator) one key at a
// time.  The attended set is the one the oracle defines: listed tiles' key rows, every
// frame's sink rows once, and in landmark mode one (mean K, mean V, +ln c_j) token per
// unlisted tile with c_j > 0 ("Zebra3D" abstract; "AVGGT" 2.B.2).
#pragma once
#include "sa_device.cuh"

struct AttnArgs {
    const void* q;
    const void* k;
    const void* v;
    const int32_t* kept_idx;
    const int32_t* kept_cnt;
    int32_t max_kept;
    const void* sink_k;
    const void* sink_v;
    int32_t landmark;
    const float* k_pool;
    const float* v_pool;
    const int32_t* k_cnt;
    void* o;
    float* lse;
    int32_t bh, frames, tokens, tile, n_sink, tpf, nt, L;
    int32_t dense;
    float scale;
};

template <typename T>
__device__ __forceinline__ float load_elem(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p, int64_t i) {
    return __ldg(p + i);
}
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void store_elem(T* p, int64_t i, float x);
template <>
__device__ __forceinline__ void store_elem<float>(float* p, int64_t i, float x) {
    p[i] = x;
}
template <>
__device__ __forceinline__ void store_elem<__nv_bfloat16>(__nv_bfloat16* p, int64_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

struct OnlineRow {
    float m, l;
    float acc[64];
};

__device__ __forceinline__ void online_fold(OnlineRow& st, float x, const float* vrow) {
    if (x == -INFINITY) return;
    if (x > st.m) {
        const float corr = st.m == -INFINITY ? 0.0f : expf(st.m - x);
        st.l = st.l * corr + 1.0f;
#pragma unroll
        for (int e = 0; e < 64; ++e) st.acc[e] = st.acc[e] * corr + vrow[e];
        st.m = x;
    } else {
        const float p = expf(x - st.m);
        st.l += p;
#pragma unroll
        for (int e = 0; e < 64; ++e) st.acc[e] = fmaf(p, vrow[e], st.acc[e]);
    }
}

// dynamic smem: ks[TILE][64], vs[TILE][64], bias[TILE] (f32), kept mask words
template <typename T, int TILE>
__global__ void __launch_bounds__(TILE) attn_simt_kernel(AttnArgs a) {
    extern __shared__ float sm[];
    float* ks = sm;
    float* vs = ks + TILE * 64;
    float* bias = vs + TILE * 64;
    uint32_t* mask = reinterpret_cast<uint32_t*>(bias + TILE);

    const int tid = threadIdx.x;
    const int nq_head = a.dense ? (a.L + TILE - 1) / TILE : a.nt;
    const int h = blockIdx.x / nq_head, i = blockIdx.x % nq_head;
    const T* Q = reinterpret_cast<const T*>(a.q) + (int64_t)h * a.L * 64;
    const T* K = reinterpret_cast<const T*>(a.k) + (int64_t)h * a.L * 64;
    const T* V = reinterpret_cast<const T*>(a.v) + (int64_t)h * a.L * 64;

    int64_t qrow0;
    int nq;
    if (a.dense) {
        qrow0 = (int64_t)i * TILE;
        nq = min(TILE, a.L - i * TILE);
    } else {
        const int f = i / a.tpf, slot = i % a.tpf;
        qrow0 = (int64_t)f * a.tokens + slot * TILE;
        nq = min(TILE, a.tokens - slot * TILE);
    }
    OnlineRow st;
    st.m = -INFINITY;
    st.l = 0.0f;
    float qv[64];
#pragma unroll
    for (int e = 0; e < 64; ++e) {
        st.acc[e] = 0.0f;
        qv[e] = tid < nq ? load_elem<T>(Q, (qrow0 + tid) * 64 + e) * a.scale : 0.0f;
    }

    // fold `count` staged rows (ks/vs/bias) into this thread's row
    auto fold_staged = [&](int count) {
        __syncthreads();
        if (tid < nq) {
            for (int t = 0; t < count; ++t) {
                const float b = bias[t];
                if (b == -INFINITY) continue;
                float x = 0.0f;
#pragma unroll
                for (int e = 0; e < 64; ++e) x = fmaf(qv[e], ks[t * 64 + e], x);
                online_fold(st, x + b, vs + t * 64);
            }
        }
        __syncthreads();
    };
    // stage `count` consecutive rows of a [rows][64] key/value array pair
    auto stage_rows = [&](const T* kb, const T* vb, int64_t row0, int count) {
        for (int idx = tid; idx < TILE * 64; idx += TILE) {
            const int r = idx >> 6, e = idx & 63;
            if (r < count) {
                ks[idx] = load_elem<T>(kb, (row0 + r) * 64 + e);
                vs[idx] = load_elem<T>(vb, (row0 + r) * 64 + e);
            }
        }
        if (tid < TILE) bias[tid] = tid < count ? 0.0f : -INFINITY;
    };

    if (a.dense) {
        for (int j0 = 0; j0 < a.L; j0 += TILE) {
            const int cnt = min(TILE, a.L - j0);
            stage_rows(K, V, j0, cnt);
            fold_staged(cnt);
        }
    } else {
        const int64_t li = (int64_t)h * a.nt + i;
        const int cnt = max(0, min(a.kept_cnt[li], a.max_kept));
        const int32_t* list = a.kept_idx + li * a.max_kept;
        for (int n = 0; n < cnt; ++n) {
            const int j = list[n];
            if (j < 0 || j >= a.nt) {
                if (tid == 0) sa_flag_error(SA_ERR_BAD_LIST);
                continue;
            }
            const int f = j / a.tpf, slot = j % a.tpf;
            const int n0 = slot * TILE;
            const int nk = min(TILE, a.tokens - n0);
            const int lo = min(nk, max(0, a.n_sink - n0));
            stage_rows(K, V, (int64_t)f * a.tokens + n0 + lo, nk - lo);
            fold_staged(nk - lo);
        }
        const int n_sink_rows = a.frames * a.n_sink;
        if (n_sink_rows > 0) {
            const T* SK = reinterpret_cast<const T*>(a.sink_k) + (int64_t)h * n_sink_rows * 64;
            const T* SV = reinterpret_cast<const T*>(a.sink_v) + (int64_t)h * n_sink_rows * 64;
            for (int r0 = 0; r0 < n_sink_rows; r0 += TILE) {
                const int c = min(TILE, n_sink_rows - r0);
                stage_rows(SK, SV, r0, c);
                fold_staged(c);
            }
        }
        if (a.landmark) {
            const int words = (a.nt + 31) / 32;
            for (int w = tid; w < words; w += TILE) mask[w] = 0u;
            __syncthreads();
            for (int n = tid; n < cnt; n += TILE) {
                const int j = list[n];
                if (j >= 0 && j < a.nt) atomicOr(&mask[j >> 5], 1u << (j & 31));
            }
            __syncthreads();
            const float* KP = a.k_pool + (int64_t)h * a.nt * 64;
            const float* VP = a.v_pool + (int64_t)h * a.nt * 64;
            for (int j0 = 0; j0 < a.nt; j0 += TILE) {
                for (int idx = tid; idx < TILE * 64; idx += TILE) {
                    const int r = idx >> 6, e = idx & 63;
                    if (j0 + r < a.nt) {
                        ks[idx] = __ldg(KP + (int64_t)(j0 + r) * 64 + e);
                        vs[idx] = __ldg(VP + (int64_t)(j0 + r) * 64 + e);
                    }
                }
                {
                    const int j = j0 + tid;
                    float b = -INFINITY;
                    if (j < a.nt && !((mask[j >> 5] >> (j & 31)) & 1u)) {
                        const int c = a.k_cnt[j];
                        if (c > 0) b = logf((float)c);
                    }
                    bias[tid] = b;
                }
                fold_staged(min(TILE, a.nt - j0));
            }
        }
    }

    if (tid < nq) {
        T* O = reinterpret_cast<T*>(a.o) + ((int64_t)h * a.L + qrow0 + tid) * 64;
        const float inv = st.l > 0.0f ? 1.0f / st.l : 0.0f;
#pragma unroll
        for (int e = 0; e < 64; ++e) store_elem<T>(O, e, st.acc[e] * inv);
        if (a.lse) a.lse[(int64_t)h * a.L + qrow0 + tid] = st.l > 0.0f ? st.m + logf(st.l) : -INFINITY;
    }
}
