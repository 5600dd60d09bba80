// Decode-time cluster selection ("IV.C Selection and Indexing" of
// "ClusterKV: Manipulating LLM KV Cache in Semantic Space for Recallable
// Compression", arXiv 2412.03213v2): clusters are ranked by the query's
// attention weight to their centroids, and whole clusters are taken in that
// order until the token budget is met, the last one trimmed; the output is
// the token indices used to load K/V.
#pragma once

#include "common.cuh"

namespace ckv {

// ---------------------------------------------------------------------------
// a6 score: s_c = sum_g q_g . lp_c in one fixed fp32 order (lane l owns
// channels 4l..4l+3, fmaf chain from 0 in channel order, xor butterfly over
// 16, 8, 4, 2, 1, heads added in order). One warp per cluster, one 256-byte
// coalesced centroid row per warp (bf16).
// ---------------------------------------------------------------------------
template <typename T, int G>
__global__ void __launch_bounds__(256)
k_score(const T *__restrict__ q, const T *__restrict__ lp, const int32_t *__restrict__ ncl,
        int C_cap, float *__restrict__ s) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x * 8 + warp;
    const int p = blockIdx.y;
    const int nC = min(max(ncl[p], 0), C_cap);
    if (c >= nC) return;
    float4 qv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) qv[g] = load4(q + ((size_t)p * G + g) * D + lane * 4);
    const float4 m = load4(lp + ((size_t)p * C_cap + c) * D + lane * 4);
    float tot = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float a = 0.f;
        a = fmaf(qv[g].x, m.x, a);
        a = fmaf(qv[g].y, m.y, a);
        a = fmaf(qv[g].z, m.z, a);
        a = fmaf(qv[g].w, m.w, a);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) a = a + __shfl_xor_sync(FULL, a, o);
        tot = (g == 0) ? a : tot + a;
    }
    if (lane == 0) s[(size_t)p * C_cap + c] = tot;
}

// monotone map float -> uint32 (ascending); -0 is folded into +0
__device__ __forceinline__ uint32_t ordered_bits(float f) {
    if (f == 0.f) f = 0.f;
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// ---------------------------------------------------------------------------
// a7 rank + fill: one CTA per problem.
//   key_c = (descending score, ascending id) packed into 64 bits, so the
//   order is total; rank_c = #{c' : key_c' < key_c} (broadcast reads of the
//   key table); sizes in rank order are prefix-summed; each warp then copies
//   the perm segments of its ranks whose start lies below the budget,
//   trimming the one that crosses it.
// Shared memory: 16 bytes per cluster (key, order, start).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
k_rankfill(const float *__restrict__ s, const int32_t *__restrict__ ncl, int C_cap,
           const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm, int perm_cap,
           int B, int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_cnt) {
    extern __shared__ __align__(16) unsigned char smraw[];
    uint64_t *key = reinterpret_cast<uint64_t *>(smraw);          // [C_cap]
    int32_t *order = reinterpret_cast<int32_t *>(key + C_cap);    // [C_cap]
    int32_t *start = order + C_cap;                                // [C_cap]
    __shared__ int32_t wsum[32];
    const int p = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthr = blockDim.x;
    const int nC = min(max(ncl[p], 0), C_cap);
    const float *sp = s + (size_t)p * C_cap;
    const int32_t *off = offsets + (size_t)p * (C_cap + 1);
    const int32_t *pp = perm + (size_t)p * perm_cap;

    for (int c = tid; c < nC; c += nthr)
        key[c] = ((uint64_t)(~ordered_bits(sp[c])) << 32) | (uint32_t)c;
    __syncthreads();
    for (int c = tid; c < nC; c += nthr) {
        const uint64_t kc = key[c];
        int r = 0;
        for (int k = 0; k < nC; ++k) r += key[k] < kc;
        order[r] = c;
    }
    __syncthreads();
    // sizes in rank order, then a block exclusive scan (4 consecutive per thread)
    int v[4], loc = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int r = tid * 4 + u;
        int sz = 0;
        if (r < nC) {
            const int c = order[r];
            const int o0 = off[c], o1 = off[c + 1];
            if (o0 < 0 || o1 < o0 || o1 > perm_cap) dev_flag(CKV_DEVERR_OFFSETS);
            else sz = o1 - o0;
        }
        v[u] = sz;
        loc += sz;
    }
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < (nthr >> 5) ? wsum[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += t;
        }
        wsum[lane] = wi;  // inclusive prefix of warp totals
    }
    __syncthreads();
    const int total = wsum[(nthr >> 5) - 1];
    int run = (warp ? wsum[warp - 1] : 0) + incl - loc;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int r = tid * 4 + u;
        if (r < nC) start[r] = run;
        run += v[u];
    }
    __syncthreads();
    if (tid == 0) sel_cnt[p] = min(B, total);
    int32_t *out = sel_idx + (size_t)p * B;
    const int nwarps = nthr >> 5;
    for (int r = warp; r < nC; r += nwarps) {
        const int st = start[r];
        if (st >= B) break;  // starts are non-decreasing in rank
        const int c = order[r];
        const int o0 = off[c], o1 = off[c + 1];
        if (o0 < 0 || o1 < o0 || o1 > perm_cap) continue;
        const int take = min(o1 - o0, B - st);
        for (int k = lane; k < take; k += 32) out[st + k] = pp[o0 + k];
    }
}

}  // namespace ckv
