// Sparse decode attention over the recalled tokens plus the sink and recent
// tokens, and the per-step append of one generated token.
//
// Attention is softmax(q K^T) V ("II.A LLM Inference and KV Cache" of
// "ClusterKV: Manipulating LLM KV Cache in Semantic Space for Recallable
// Compression", arXiv 2412.03213v2); only the selected tokens are attended
// ("III.A Problem Formulation and Design Rationale").
//
// Split-K flash decode: the attended list A of a problem (sinks, recalled,
// recent) is cut into chunks, one CTA per (chunk, problem); each CTA runs an
// fp32 online softmax over its rows for all G query heads sharing the KV head
// and writes an unnormalised partial; k_decode_combine merges the partials.
// A 16-lane half-warp owns one row at a time (16 bytes per lane: one 256-byte
// bf16 row per half-warp); each half-warp keeps U rows of K and V in flight.
#pragma once

#include "common.cuh"

namespace ckv {

constexpr int DEC_THREADS = 128;
constexpr int DEC_HALVES = DEC_THREADS / 16;  // 8 row streams per CTA
constexpr int DEC_U = 4;                      // rows in flight per half-warp

// rows of A: [0, S) | sel_idx[0, cnt) | tail_begin + [0, ntail)
__device__ __forceinline__ int dec_row(int j, int S, int cnt, int tb,
                                       const int32_t *__restrict__ sel) {
    if (j < S) return j;
    if (j < S + cnt) return sel[j - S];
    return tb + (j - S - cnt);
}

template <typename T, int G>
__global__ void __launch_bounds__(DEC_THREADS)
k_decode_split(const T *__restrict__ q, const T *__restrict__ K, const T *__restrict__ V,
               int64_t kvs, int kv_rows, int S, const int32_t *__restrict__ tail_b,
               const int32_t *__restrict__ tail_e, const int32_t *__restrict__ sel_idx,
               const int32_t *__restrict__ sel_cnt, int B, float qscale, int chunk,
               int nsplit, float *__restrict__ part_o, float2 *__restrict__ part_ml) {
    __shared__ float sm_o[DEC_HALVES][G][D];
    __shared__ float sm_m[DEC_HALVES][G];
    __shared__ float sm_l[DEC_HALVES][G];
    const int p = blockIdx.y, split = blockIdx.x;
    const int half = threadIdx.x >> 4, hl = threadIdx.x & 15;
    const int cnt = min(max(sel_cnt[p], 0), B);
    const int tb = tail_b[p];
    const int ntail = max(0, tail_e[p] - tb);
    const int n_att = S + cnt + ntail;
    const int j0 = split * chunk, j1 = min(n_att, j0 + chunk);
    // rows beyond the grid's capacity (a tail longer than max_tail) are reported
    if (split == 0 && threadIdx.x == 0 && n_att > nsplit * chunk) dev_flag(CKV_DEVERR_INDEX);
    const int32_t *sel = sel_idx + (size_t)p * B;
    const T *Kp = K + (int64_t)p * kvs + hl * 8;
    const T *Vp = V + (int64_t)p * kvs + hl * 8;

    float qf[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        Row8<T> r;
        r.load(q + ((size_t)p * G + g) * D + hl * 8);
        r.to_float(qf[g]);
#pragma unroll
        for (int t = 0; t < 8; ++t) qf[g][t] *= qscale;  // scale * log2(e)
    }
    float m[G], l[G], o[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) o[g][t] = 0.f;
    }

    // the trip count is uniform across the CTA (shuffles below use full masks)
    for (int jb = j0; jb < j1; jb += DEC_HALVES * DEC_U) {
        int row[DEC_U];
        bool ok[DEC_U];
#pragma unroll
        for (int u = 0; u < DEC_U; ++u) {
            const int j = jb + half + u * DEC_HALVES;
            ok[u] = j < j1;
            row[u] = ok[u] ? dec_row(j, S, cnt, tb, sel) : 0;
            if (ok[u] && (row[u] < 0 || row[u] >= kv_rows)) {
                ok[u] = false;
                if (hl == 0) dev_flag(CKV_DEVERR_INDEX);
            }
        }
        Row8<T> kr[DEC_U], vr[DEC_U];
#pragma unroll
        for (int u = 0; u < DEC_U; ++u) {
            if (ok[u]) {
                kr[u].load(Kp + (int64_t)row[u] * D);
                vr[u].load(Vp + (int64_t)row[u] * D);
            } else {
                kr[u].zero();
                vr[u].zero();
            }
        }
        float kf[DEC_U][8];
#pragma unroll
        for (int u = 0; u < DEC_U; ++u) kr[u].to_float(kf[u]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float lg[DEC_U];
            float mx = m[g];
#pragma unroll
            for (int u = 0; u < DEC_U; ++u) {
                float a = 0.f;
#pragma unroll
                for (int t = 0; t < 8; ++t) a = fmaf(qf[g][t], kf[u][t], a);
#pragma unroll
                for (int w = 8; w >= 1; w >>= 1) a += __shfl_xor_sync(FULL, a, w);
                lg[u] = ok[u] ? a : -INFINITY;
                mx = fmaxf(mx, lg[u]);
            }
            if (mx != -INFINITY) {
                const float corr = exp2f(m[g] - mx);
                l[g] *= corr;
#pragma unroll
                for (int t = 0; t < 8; ++t) o[g][t] *= corr;
#pragma unroll
                for (int u = 0; u < DEC_U; ++u) {
                    const float pu = exp2f(lg[u] - mx);
                    l[g] += pu;
                    float vf[8];
                    vr[u].to_float(vf);
#pragma unroll
                    for (int t = 0; t < 8; ++t) o[g][t] = fmaf(pu, vf[t], o[g][t]);
                }
                m[g] = mx;
            }
        }
    }
    // merge the 8 half-warp states of this CTA
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int t = 0; t < 8; ++t) sm_o[half][g][hl * 8 + t] = o[g][t];
        if (hl == 0) {
            sm_m[half][g] = m[g];
            sm_l[half][g] = l[g];
        }
    }
    __syncthreads();
    const int t = threadIdx.x;  // channel
    const size_t base = ((size_t)p * nsplit + split) * G;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int h = 0; h < DEC_HALVES; ++h) M = fmaxf(M, sm_m[h][g]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int h = 0; h < DEC_HALVES; ++h) {
                const float w = exp2f(sm_m[h][g] - M);
                L = fmaf(sm_l[h][g], w, L);
                O = fmaf(sm_o[h][g][t], w, O);
            }
        }
        part_o[(base + g) * D + t] = O;
        if (t == 0) part_ml[base + g] = make_float2(M, L);
    }
}

template <int G>
__global__ void __launch_bounds__(D)
k_decode_combine(const float *__restrict__ part_o, const float2 *__restrict__ part_ml, int nsplit,
                 float *__restrict__ out) {
    const int p = blockIdx.x, t = threadIdx.x;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
        for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part_ml[((size_t)p * nsplit + s) * G + g].x);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
            for (int s = 0; s < nsplit; ++s) {
                const size_t b = ((size_t)p * nsplit + s) * G + g;
                const float2 ml = part_ml[b];
                const float w = exp2f(ml.x - M);
                L = fmaf(ml.y, w, L);
                O = fmaf(part_o[b * D + t], w, O);
            }
        }
        out[((size_t)p * G + g) * D + t] = L > 0.f ? O / L : 0.f;
    }
}

// a9 append: one warp per problem
template <typename T>
__global__ void __launch_bounds__(32)
k_append(T *__restrict__ K, T *__restrict__ V, int64_t kvs, int kv_rows,
         const T *__restrict__ nk, const T *__restrict__ nv, int32_t *__restrict__ tail_end) {
    const int p = blockIdx.x, lane = threadIdx.x;
    const int pos = tail_end[p];
    __syncwarp();
    if (pos < 0 || pos >= kv_rows) {
        if (lane == 0) dev_flag(CKV_DEVERR_INDEX);
        return;
    }
    const size_t src = (size_t)p * D + lane * 4;
    const int64_t dst = (int64_t)p * kvs + (int64_t)pos * D + lane * 4;
    store4(K + dst, load4(nk + src));
    store4(V + dst, load4(nv + src));
    __syncwarp();
    if (lane == 0) tail_end[p] = pos + 1;
}

// ---------------------------------------------------------------------------
// Self-test of the timeout reporting: wait (bounded by the global timer) for a
// flag that nothing sets, then record a timeout in the device error word.
// ---------------------------------------------------------------------------
__device__ int g_selftest_flag;  // never set

__global__ void k_selftest_wait(unsigned long long limit_ns) {
    if (threadIdx.x != 0) return;
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    while (*reinterpret_cast<volatile int *>(&g_selftest_flag) == 0) {
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > limit_ns) {
            dev_flag(CKV_DEVERR_TIMEOUT);
            return;
        }
    }
}

}  // namespace ckv
