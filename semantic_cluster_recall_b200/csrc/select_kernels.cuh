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
//   order is total. The cluster at which the running size sum, in key order,
//   reaches the budget is found by a weighted radix select (8-bit digits from
//   the top of the key; the id half holds c < 2^16, so its two upper bytes are
//   skipped); the non-empty clusters up to it are compacted, and each one's
//   rank and first output slot come from counting the smaller keys and
//   summing their sizes; each warp then copies the perm segments of its ranks,
//   trimming the one that crosses the budget.
// Shared memory: 36 bytes per cluster.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
k_rankfill(const float *__restrict__ s, const int32_t *__restrict__ ncl, int C_cap,
           const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm, int perm_cap,
           int B, int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_cnt) {
    extern __shared__ __align__(16) unsigned char smraw[];
    uint64_t *key = reinterpret_cast<uint64_t *>(smraw);    // [C_cap]
    uint64_t *lkey = key + C_cap;                           // [C_cap] keys of the selected
    int32_t *csz = reinterpret_cast<int32_t *>(lkey + C_cap);  // [C_cap] sizes by id
    int32_t *lst = csz + C_cap;                             // [C_cap] selected ids
    int32_t *lsz = lst + C_cap;                             // [C_cap] their sizes
    int32_t *order = lsz + C_cap;                           // [C_cap] id by rank
    int32_t *start = order + C_cap;                         // [C_cap] first slot by rank
    __shared__ __align__(16) unsigned s_hw[2][256];         // size sum per digit
    __shared__ __align__(16) unsigned s_hn[2][256];         // cluster count per digit
    __shared__ int s_before, s_total, s_bin, s_cnt, s_m;
    const int p = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthr = blockDim.x;
    const int nC = min(max(ncl[p], 0), C_cap);
    const float *sp = s + (size_t)p * C_cap;
    const int32_t *off = offsets + (size_t)p * (C_cap + 1);
    const int32_t *pp = perm + (size_t)p * perm_cap;

    for (int c = tid; c < nC; c += nthr) {
        key[c] = ((uint64_t)(~ordered_bits(sp[c])) << 32) | (uint32_t)c;
        const int o0 = off[c], o1 = off[c + 1];
        int sz = 0;
        if (o0 < 0 || o1 < o0 || o1 > perm_cap) dev_flag(CKV_DEVERR_OFFSETS);
        else sz = o1 - o0;
        csz[c] = sz;
    }
    if (tid < 256) {
        s_hw[0][tid] = 0;
        s_hn[0][tid] = 0;
    }
    if (tid == 0) {
        s_m = 0;
        s_total = 0;
    }
    __syncthreads();

    uint64_t pre = 0, msk = 0;  // key bits fixed so far
    int need = B;               // budget still to reach inside the fixed prefix
    bool take_all = false;      // the sizes sum to less than the budget
    if (B > 0) {
        constexpr int NPASS = 6;
        for (int ps = 0; ps < NPASS; ++ps) {
            const int sh = ps < 4 ? 56 - 8 * ps : 8 * (NPASS - 1 - ps);
            unsigned *hw = s_hw[ps & 1], *hn = s_hn[ps & 1];
            for (int c = tid; c < nC; c += nthr) {
                const uint64_t k = key[c];
                if ((k & msk) == pre) {
                    const int dg = (int)((k >> sh) & 255);
                    atomicAdd(&hw[dg], (unsigned)csz[c]);
                    atomicAdd(&hn[dg], 1u);
                }
            }
            if (tid < 256) {  // the next pass's tables
                s_hw[(ps + 1) & 1][tid] = 0;
                s_hn[(ps + 1) & 1][tid] = 0;
            }
            __syncthreads();
            if (warp == 0) {
                // lane l owns digits 8l..8l+7: the first digit whose running
                // weight reaches `need` (valid offsets keep sums below 2^31)
                const uint4 wa = reinterpret_cast<const uint4 *>(hw)[lane * 2];
                const uint4 wb = reinterpret_cast<const uint4 *>(hw)[lane * 2 + 1];
                const unsigned wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                unsigned wl = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) wl += wv[i];
                unsigned incl = wl;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned t = __shfl_up_sync(FULL, incl, o);
                    if (lane >= o) incl += t;
                }
                if (ps == 0 && lane == 31) s_total = (int)incl;
                const unsigned hit = __ballot_sync(FULL, incl >= (unsigned)need);
                if (hit == 0) {
                    if (lane == 0) s_bin = -1;
                } else if (lane == __ffs(hit) - 1) {
                    unsigned before = incl - wl;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (before + wv[i] >= (unsigned)need) {
                            s_bin = lane * 8 + i;
                            s_before = (int)before;
                            s_cnt = (int)hn[lane * 8 + i];
                            break;
                        }
                        before += wv[i];
                    }
                }
            }
            __syncthreads();
            const int bin = s_bin;
            if (bin < 0) {
                take_all = true;
                break;
            }
            pre |= (uint64_t)bin << sh;
            msk |= 255ull << sh;
            need -= s_before;
            if (s_cnt == 1) break;
        }
        // the selected non-empty clusters, compacted
        for (int c0 = warp * 32; c0 < nC; c0 += nthr) {  // warp-uniform
            const int c = c0 + lane;
            uint64_t k = 0;
            int sz = 0;
            bool in = false;
            if (c < nC) {
                k = key[c];
                sz = csz[c];
                in = sz > 0 && (take_all || (k & msk) <= pre);
            }
            const unsigned bal = __ballot_sync(FULL, in);
            int base = 0;
            if (lane == 0 && bal) base = atomicAdd(&s_m, __popc(bal));
            base = __shfl_sync(FULL, base, 0);
            if (in) {
                const int i = base + __popc(bal & lanemask_lt());
                lst[i] = c;
                lkey[i] = k;
                lsz[i] = sz;
            }
        }
    }
    __syncthreads();
    const int nsel = s_m;
    for (int i = tid; i < nsel; i += nthr) {  // rank and first slot by counting
        const uint64_t ki = lkey[i];
        int r = 0, st = 0;
        for (int j = 0; j < nsel; ++j) {
            if (lkey[j] < ki) {
                ++r;
                st += lsz[j];
            }
        }
        order[r] = lst[i];
        start[r] = st;
    }
    __syncthreads();
    if (tid == 0) sel_cnt[p] = B > 0 ? min(B, s_total) : 0;
    int32_t *out = sel_idx + (size_t)p * B;
    const int nwarps = nthr >> 5;
    for (int r = warp; r < nsel; r += nwarps) {
        const int st = start[r];
        if (st >= B) continue;
        const int c = order[r];
        const int take = min(csz[c], B - st);
        const int o0 = off[c];
        for (int k = lane; k < take; k += 32) out[st + k] = pp[o0 + k];
    }
}

}  // namespace ckv
