// Fused decode step: cluster-granularity selection and sparse attention in one
// launch ("IV.C Selection and Indexing" and "II.A LLM Inference and KV Cache"
// of "ClusterKV: Manipulating LLM KV Cache in Semantic Space for Recallable
// Compression", arXiv 2412.03213v2).
//
// One thread-block cluster of NC CTAs per problem; the CTAs talk through
// distributed shared memory (DSMEM) and the hardware cluster barrier:
//   1. score   CTA r scores clusters c = r*8+warp (mod NC*8) in exactly the
//              fixed fp32 order of k_score and writes the 64-bit rank key
//              (descending score, ascending id) into every CTA's key table
//   -- cluster barrier
//   2. rank    CTA r ranks clusters c = r (mod NC), one warp per cluster,
//              the 32 lanes counting smaller keys, and writes
//              (order[rank] = c, size[rank] = n_c) into every CTA
//   -- cluster barrier
//   3. fill    every CTA prefix-sums the sizes in rank order (redundantly, no
//              leader round trip); sel_cnt = min(budget, total)
//   4. resolve CTA r owns rows [r*chunk, (r+1)*chunk) of the attended list
//              (sinks, recalled, recent); each recalled row finds its rank by
//              binary search and its position through offsets/perm; the
//              positions go to shared memory and to sel_idx (ABI output)
//   5. attend  split-K online softmax over the CTA's rows (half-warp per
//              256-byte row, U rows in flight per half-warp, U chosen so a
//              CTA's rows arrive in one batch at the usual shapes), merged
//              inside the CTA
//   -- partial (m, l, o) pushed into the leader CTA's shared memory
//   -- cluster barrier
//   6. combine the leader merges the NC partials and writes out
// The selection is bit-identical to ckv_select (same arithmetic, same order,
// same tie rules); attention agrees with ckv_sparse_decode up to fp32
// summation order.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "select_kernels.cuh"

namespace ckv {
namespace sd {

namespace cg = cooperative_groups;

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int HALVES = THREADS / 16;   // row streams
constexpr int NC_MAX = 8;              // CTAs per problem (portable cluster size)
constexpr int POS_MAX = 4096;          // attended rows per CTA

struct Args {
    const void *q;
    const void *lp;
    const int32_t *ncl;
    int C_cap;
    const int32_t *offsets;
    const int32_t *perm;
    int perm_cap;
    int B;
    const void *K;
    const void *V;
    int64_t kvs;
    int kv_rows;
    int S;
    const int32_t *tail_b;
    const int32_t *tail_e;
    float qscale;  // attention scale * log2(e)
    int chunk;     // attended rows per CTA
    int32_t *sel_idx;
    int32_t *sel_cnt;
    float *out;
};

// dynamic shared memory layout (bytes), sized by C_cap, G and chunk
struct Layout {
    size_t keys, order, size, start, offs, pos, mo, ml, part, total;
};

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~(size_t)15; }

__host__ __device__ inline Layout layout(int C_cap, int G, int chunk, int nc) {
    Layout L;
    size_t o = 0;
    L.keys = o;   o += al16((size_t)C_cap * 8);
    L.order = o;  o += al16((size_t)C_cap * 4);
    L.size = o;   o += al16((size_t)C_cap * 4);
    L.start = o;  o += al16((size_t)(C_cap + 1) * 4);
    L.offs = o;   o += al16((size_t)(C_cap + 1) * 4);     // the problem's offsets row
    L.pos = o;    o += al16((size_t)chunk * 4);
    L.mo = o;     o += al16((size_t)HALVES * D * 4);          // per-g merge of the row streams
    L.ml = o;     o += al16((size_t)HALVES * 2 * 4);
    L.part = o;   o += al16((size_t)nc * G * (D + 2) * 4);    // leader: partials of the cluster
    L.total = o;
    return L;
}

template <typename T, int G, int U>
__global__ void __launch_bounds__(THREADS)
k_select_decode(const Args a) {
    cg::cluster_group cl = cg::this_cluster();
    const int nc = (int)cl.num_blocks();
    const int rank = (int)cl.block_rank();
    const int p = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    extern __shared__ __align__(16) unsigned char smem[];
    const Layout LY = layout(a.C_cap, G, a.chunk, nc);
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem + LY.keys);
    int32_t *order = reinterpret_cast<int32_t *>(smem + LY.order);
    int32_t *rsz = reinterpret_cast<int32_t *>(smem + LY.size);
    int32_t *start = reinterpret_cast<int32_t *>(smem + LY.start);
    int32_t *off_s = reinterpret_cast<int32_t *>(smem + LY.offs);
    int32_t *pos_s = reinterpret_cast<int32_t *>(smem + LY.pos);
    float *mo = reinterpret_cast<float *>(smem + LY.mo);
    float *mml = reinterpret_cast<float *>(smem + LY.ml);
    float *part = reinterpret_cast<float *>(smem + LY.part);
    __shared__ int wsum[WARPS];

    const int nC = min(max(a.ncl[p], 0), a.C_cap);
    const int32_t *off = a.offsets + (size_t)p * (a.C_cap + 1);
    const int32_t *pp = a.perm + (size_t)p * a.perm_cap;
    const T *qp = reinterpret_cast<const T *>(a.q) + (size_t)p * G * D;

    // the problem's offsets row, needed by ranking and by position lookup
    for (int i = tid; i <= nC; i += THREADS) off_s[i] = off[i];
    cl.sync();  // every CTA of the cluster is running before any DSMEM access

    // ---- 1. score (fixed fp32 order), keys broadcast to every CTA ----
    {
        float4 qv[G];
#pragma unroll
        for (int g = 0; g < G; ++g) qv[g] = load4(qp + g * D + lane * 4);
        const T *lpp = reinterpret_cast<const T *>(a.lp) + (size_t)p * a.C_cap * D + lane * 4;
        const int cstride = nc * WARPS;
        constexpr int SB = 8;  // centroid rows in flight per warp
        for (int cb = rank * WARPS + warp; cb < nC; cb += cstride * SB) {
            float4 mrow[SB];
#pragma unroll
            for (int u = 0; u < SB; ++u) {
                const int c = cb + u * cstride;
                mrow[u] = c < nC ? load4(lpp + (size_t)c * D) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < SB; ++u) {
                const int c = cb + u * cstride;
                if (c >= nC) break;  // warp-uniform
                float tot = 0.f;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float sc = 0.f;
                    sc = fmaf(qv[g].x, mrow[u].x, sc);
                    sc = fmaf(qv[g].y, mrow[u].y, sc);
                    sc = fmaf(qv[g].z, mrow[u].z, sc);
                    sc = fmaf(qv[g].w, mrow[u].w, sc);
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) sc = sc + __shfl_xor_sync(FULL, sc, o);
                    tot = (g == 0) ? sc : tot + sc;
                }
                const uint64_t key = ((uint64_t)(~ordered_bits(tot)) << 32) | (uint32_t)c;
                if (lane < nc) *cl.map_shared_rank(&keys[c], lane) = key;
            }
        }
    }
    cl.sync();

    // ---- 2. rank own clusters (c = rank mod nc): one warp per cluster ----
    for (int c = rank + warp * nc; c < nC; c += WARPS * nc) {  // warp-uniform
        const uint64_t kc = keys[c];
        int n0 = 0, n1 = 0, n2 = 0, n3 = 0;  // independent partial counts
        int k = lane;
        for (; k + 96 < nC; k += 128) {
            n0 += keys[k] < kc;
            n1 += keys[k + 32] < kc;
            n2 += keys[k + 64] < kc;
            n3 += keys[k + 96] < kc;
        }
        for (; k < nC; k += 32) n0 += keys[k] < kc;
        const int r = __reduce_add_sync(FULL, n0 + n1 + n2 + n3);
        int sz = 0;
        const int o0 = off_s[c], o1 = off_s[c + 1];
        if (o0 < 0 || o1 < o0 || o1 > a.perm_cap) {
            if (lane == 0) dev_flag(CKV_DEVERR_OFFSETS);
        } else {
            sz = o1 - o0;
        }
        if (lane < nc) {  // every CTA gets (order, size)
            *cl.map_shared_rank(&order[r], lane) = c;
            *cl.map_shared_rank(&rsz[r], lane) = sz;
        }
    }
    cl.sync();

    // ---- 3. fill: exclusive scan of sizes in rank order (every CTA) ----
    {
        const int per = (nC + THREADS - 1) / THREADS;
        const int b = tid * per, e = min(nC, b + per);
        int loc = 0;
        for (int r = b; r < e; ++r) loc += rsz[r];
        int incl = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int wpre = 0;
        for (int w = 0; w < warp; ++w) wpre += wsum[w];
        int run = wpre + incl - loc;
        for (int r = b; r < e; ++r) {
            start[r] = run;
            run += rsz[r];
        }
        if (tid == THREADS - 1) start[nC] = run;  // total
        __syncthreads();
    }
    const int total = start[nC];
    const int cnt = min(a.B, total);
    if (rank == 0 && tid == 0) a.sel_cnt[p] = cnt;

    // ---- 4. resolve this CTA's rows of the attended list ----
    const int tb = a.tail_b[p];
    const int ntail = max(0, a.tail_e[p] - tb);
    const int n_att = a.S + cnt + ntail;
    if (rank == 0 && tid == 0 && n_att > nc * a.chunk) dev_flag(CKV_DEVERR_INDEX);
    const int j0 = rank * a.chunk, j1 = min(n_att, j0 + a.chunk);
    for (int j = j0 + tid; j < j1; j += THREADS) {
        int row;
        if (j < a.S) {
            row = j;
        } else if (j < a.S + cnt) {
            const int k = j - a.S;
            // last rank r with start[r] <= k (a non-empty cluster)
            int lo = 0, hi = nC - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (start[mid] <= k) lo = mid;
                else hi = mid - 1;
            }
            const int c = order[lo];
            const int slot = off_s[c] + (k - start[lo]);
            row = (slot >= 0 && slot < a.perm_cap) ? pp[slot] : -1;
            a.sel_idx[(size_t)p * a.B + k] = row;
        } else {
            row = tb + (j - a.S - cnt);
        }
        if (row < 0 || row >= a.kv_rows) {
            dev_flag(CKV_DEVERR_INDEX);
            row = -1;
        }
        pos_s[j - j0] = row;
    }
    __syncthreads();

    // ---- 5. attention over the CTA's rows ----
    const int half = tid >> 4, hl = tid & 15;
    const T *Kp = reinterpret_cast<const T *>(a.K) + (int64_t)p * a.kvs + hl * 8;
    const T *Vp = reinterpret_cast<const T *>(a.V) + (int64_t)p * a.kvs + hl * 8;
    float qf[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        Row8<T> r;
        r.load(qp + g * D + hl * 8);
        r.to_float(qf[g]);
#pragma unroll
        for (int t = 0; t < 8; ++t) qf[g][t] *= a.qscale;
    }
    float m[G], l[G], o[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) o[g][t] = 0.f;
    }
    const int nrows = max(0, j1 - j0);
    for (int jb = 0; jb < nrows; jb += HALVES * U) {  // uniform trip count
        int row[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = jb + half + u * HALVES;
            row[u] = j < nrows ? pos_s[j] : -1;
        }
        Row8<T> kr[U], vr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (row[u] >= 0) {
                kr[u].load(Kp + (int64_t)row[u] * D);
                vr[u].load(Vp + (int64_t)row[u] * D);
            } else {
                kr[u].zero();
                vr[u].zero();
            }
        }
        float lg[G][U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float kf[8];
            kr[u].to_float(kf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float sc = 0.f;
#pragma unroll
                for (int t = 0; t < 8; ++t) sc = fmaf(qf[g][t], kf[t], sc);
                lg[g][u] = sc;
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int u = 0; u < U; ++u) {
#pragma unroll
                for (int w = 8; w >= 1; w >>= 1) lg[g][u] += __shfl_xor_sync(FULL, lg[g][u], w);
                if (row[u] < 0) lg[g][u] = -INFINITY;
            }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float mx = m[g];
#pragma unroll
            for (int u = 0; u < U; ++u) mx = fmaxf(mx, lg[g][u]);
            if (mx != -INFINITY) {
                const float corr = exp2f(m[g] - mx);
                l[g] *= corr;
#pragma unroll
                for (int t = 0; t < 8; ++t) o[g][t] *= corr;
                m[g] = mx;
#pragma unroll
                for (int u = 0; u < U; ++u) lg[g][u] = exp2f(lg[g][u] - mx);
            } else {
#pragma unroll
                for (int u = 0; u < U; ++u) lg[g][u] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float vf[8];
            vr[u].to_float(vf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                l[g] += lg[g][u];
#pragma unroll
                for (int t = 0; t < 8; ++t) o[g][t] = fmaf(lg[g][u], vf[t], o[g][t]);
            }
        }
    }
    // merge the row streams of this CTA, one query head at a time, and push
    // the CTA's partial into the leader's shared memory
    float *lead_part = cl.map_shared_rank(part, 0);
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int t = 0; t < 8; ++t) mo[half * D + hl * 8 + t] = o[g][t];
        if (hl == 0) {
            mml[half * 2 + 0] = m[g];
            mml[half * 2 + 1] = l[g];
        }
        __syncthreads();
        if (tid < D) {
            float M = -INFINITY;
#pragma unroll
            for (int h = 0; h < HALVES; ++h) M = fmaxf(M, mml[h * 2]);
            float Lsum = 0.f, O = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int h = 0; h < HALVES; ++h) {
                    const float w = exp2f(mml[h * 2] - M);
                    Lsum = fmaf(mml[h * 2 + 1], w, Lsum);
                    O = fmaf(mo[h * D + tid], w, O);
                }
            }
            float *dst = lead_part + (size_t)(rank * G + g) * (D + 2);
            dst[tid] = O;
            if (tid == 0) {
                dst[D] = M;
                dst[D + 1] = Lsum;
            }
        }
        __syncthreads();
    }
    cl.sync();

    // ---- 6. the leader combines the cluster's partials ----
    if (rank == 0 && tid < D) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float M = -INFINITY;
            for (int r = 0; r < nc; ++r) M = fmaxf(M, part[(size_t)(r * G + g) * (D + 2) + D]);
            float Lsum = 0.f, O = 0.f;
            if (M != -INFINITY) {
                for (int r = 0; r < nc; ++r) {
                    const float *src = part + (size_t)(r * G + g) * (D + 2);
                    const float w = exp2f(src[D] - M);
                    Lsum = fmaf(src[D + 1], w, Lsum);
                    O = fmaf(src[tid], w, O);
                }
            }
            a.out[((size_t)p * G + g) * D + tid] = Lsum > 0.f ? O / Lsum : 0.f;
        }
    }
}

}  // namespace sd
}  // namespace ckv
