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
//   2. select  every CTA finds, on its own copy of the keys, the cluster at
//              which the running size sum in rank order reaches the budget:
//              a weighted radix select (8-bit digits from the top of the key,
//              per-digit size sums and counts by 32-bit shared atomics, the
//              first digit whose running size sum reaches the budget kept)
//   3. fill    the non-empty clusters up to that key are compacted; each
//              one's rank and first row among them come from counting the
//              smaller keys and summing their sizes; sel_cnt =
//              min(budget, total). No cluster barrier: all CTAs agree
//   4. resolve CTA r owns rows [r*chunk, (r+1)*chunk) of the attended list
//              (sinks, recalled, recent); each recalled row finds its rank by
//              binary search over the selected clusters and its position
//              through offsets/perm (perm loads batched); the positions go to
//              shared memory and to sel_idx (ABI output)
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
    // cache of the clusters selected in the last R steps (null: no cache)
    int32_t *last_sel;     // [P][C_cap] last step that selected each cluster
    int step, R;
    int32_t *cache_stats;  // [P][4] hits, selected clusters, hit tokens, recalled tokens
    int32_t *miss_list;    // [P][C_cap] selected clusters not cached, rank order (or null)
};

// dynamic shared memory layout (bytes), sized by C_cap, G and chunk
struct Layout {
    size_t keys, lkey, csz, lst, order, size, start, offs, pos, mo, ml, part, total;
};

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~(size_t)15; }

__host__ __device__ inline Layout layout(int C_cap, int G, int chunk, int nc) {
    Layout L;
    size_t o = 0;
    L.keys = o;   o += al16((size_t)C_cap * 8);
    L.lkey = o;   o += al16((size_t)C_cap * 8);           // keys of the selected clusters
    L.csz = o;    o += al16((size_t)C_cap * 4);           // cluster sizes by id
    L.lst = o;    o += al16((size_t)C_cap * 4);           // selected cluster ids (unordered)
    L.order = o;  o += al16((size_t)C_cap * 4);
    L.size = o;   o += al16((size_t)C_cap * 4);           // sizes of the selected clusters
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
    // programmatic dependent launch: wait for the preceding kernel of the
    // stream before reading anything (its outputs may be this step's inputs),
    // then let the next kernel be launched at once, so its CTAs are placed
    // while this grid finishes (the gap between back-to-back steps). Both are
    // no-ops when the launch carries no such dependency.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    cg::cluster_group cl = cg::this_cluster();
    const int nc = (int)cl.num_blocks();
    const int rank = (int)cl.block_rank();
    const int p = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    extern __shared__ __align__(16) unsigned char smem[];
    const Layout LY = layout(a.C_cap, G, a.chunk, nc);
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem + LY.keys);
    uint64_t *lkey = reinterpret_cast<uint64_t *>(smem + LY.lkey);
    int32_t *csz = reinterpret_cast<int32_t *>(smem + LY.csz);
    int32_t *lst = reinterpret_cast<int32_t *>(smem + LY.lst);
    int32_t *order = reinterpret_cast<int32_t *>(smem + LY.order);
    int32_t *lsz = reinterpret_cast<int32_t *>(smem + LY.size);
    int32_t *start = reinterpret_cast<int32_t *>(smem + LY.start);
    int32_t *off_s = reinterpret_cast<int32_t *>(smem + LY.offs);
    int32_t *pos_s = reinterpret_cast<int32_t *>(smem + LY.pos);
    float *mo = reinterpret_cast<float *>(smem + LY.mo);
    float *mml = reinterpret_cast<float *>(smem + LY.ml);
    float *part = reinterpret_cast<float *>(smem + LY.part);
    __shared__ __align__(16) unsigned s_hw[2][256];  // size sum per digit
    __shared__ __align__(16) unsigned s_hn[2][256];  // cluster count per digit
    __shared__ int s_before, s_total, s_bin, s_cnt, s_m;
    __shared__ int s_wm[WARPS], s_hits, s_htok;

    const int nC = min(max(a.ncl[p], 0), a.C_cap);
    const int32_t *off = a.offsets + (size_t)p * (a.C_cap + 1);
    const int32_t *pp = a.perm + (size_t)p * a.perm_cap;
    const T *qp = reinterpret_cast<const T *>(a.q) + (size_t)p * G * D;

    // the problem's offsets row, needed by selection and by position lookup
    for (int i = tid; i <= nC; i += THREADS) off_s[i] = off[i];
    s_hw[0][tid] = 0;  // THREADS == 256
    s_hn[0][tid] = 0;
    if (tid == 0) s_m = 0;

    // ---- 1. score (fixed fp32 order), keys broadcast to every CTA. The
    // first batch of centroid rows is loaded and scored before the cluster
    // barrier (only the DSMEM writes must wait for it) ----
    {
        float4 qv[G];
#pragma unroll
        for (int g = 0; g < G; ++g) qv[g] = load4(qp + g * D + lane * 4);
        const T *lpp = reinterpret_cast<const T *>(a.lp) + (size_t)p * a.C_cap * D + lane * 4;
        const int cstride = nc * WARPS;
        constexpr int SB = 8;  // centroid rows in flight per warp
        uint64_t kk[SB];
        auto score_batch = [&](int cb) {
            float4 mrow[SB];
#pragma unroll
            for (int u = 0; u < SB; ++u) {
                const int c = cb + u * cstride;
                mrow[u] = c < nC ? load4(lpp + (size_t)c * D) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < SB; ++u) {
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
                kk[u] = ((uint64_t)(~ordered_bits(tot)) << 32) | (uint32_t)(cb + u * cstride);
            }
        };
        int cb = rank * WARPS + warp;
        score_batch(cb);
        cl.sync();  // every CTA of the cluster is running before any DSMEM access
        for (;;) {  // warp-uniform
#pragma unroll
            for (int u = 0; u < SB; ++u) {
                const int c = cb + u * cstride;
                if (c < nC && lane < nc) *cl.map_shared_rank(&keys[c], lane) = kk[u];
            }
            cb += cstride * SB;
            if (cb >= nC) break;
            score_batch(cb);
        }
    }
    cl.sync();

    // ---- 2. threshold: the cluster at which the running size sum, in rank
    // order, reaches the budget. Weighted radix select over the 64-bit keys,
    // 8-bit digits from the top; the id half holds c < 2^16, so its two upper
    // bytes are zero for every key and are skipped. Every CTA runs it on its
    // own copy of the key table. ----
    uint64_t pre = 0, msk = 0;  // key bits fixed so far
    int need = a.B;             // budget still to reach inside the fixed prefix
    bool take_all = false;      // the sizes sum to less than the budget
    if (a.B > 0) {
        constexpr int NPASS = 6;
        for (int ps = 0; ps < NPASS; ++ps) {
            const int sh = ps < 4 ? 56 - 8 * ps : 8 * (NPASS - 1 - ps);
            unsigned *hw = s_hw[ps & 1], *hn = s_hn[ps & 1];
            // plain 32-bit shared atomics: (weight, count) per digit
            for (int c = tid; c < nC; c += THREADS) {
                const uint64_t k = keys[c];
                int sz;
                if (ps == 0) {
                    const int o0 = off_s[c], o1 = off_s[c + 1];
                    sz = 0;
                    if (o0 < 0 || o1 < o0 || o1 > a.perm_cap) dev_flag(CKV_DEVERR_OFFSETS);
                    else sz = o1 - o0;
                    csz[c] = sz;
                } else {
                    sz = csz[c];
                }
                if ((k & msk) == pre) {
                    const int dg = (int)((k >> sh) & 255);
                    atomicAdd(&hw[dg], (unsigned)sz);
                    atomicAdd(&hn[dg], 1u);
                }
            }
            s_hw[(ps + 1) & 1][tid] = 0;  // the next pass's tables (THREADS == 256)
            s_hn[(ps + 1) & 1][tid] = 0;
            __syncthreads();
            if (warp == 0) {
                // lane l owns digits 8l..8l+7: the first digit whose running
                // weight reaches `need`. Valid offsets keep every sum below
                // perm_cap < 2^31.
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
    }
    const int total = a.B > 0 ? s_total : 0;
    const int cnt = min(a.B, total);
    if (rank == 0 && tid == 0) a.sel_cnt[p] = cnt;

    // ---- 3. the selected non-empty clusters (every key up to the threshold),
    // compacted, then each one's rank and start row among them by counting
    // the smaller keys (thread per selected cluster, broadcast reads) ----
    if (a.B > 0) {
        for (int c0 = warp * 32; c0 < nC; c0 += THREADS) {  // warp-uniform
            const int c = c0 + lane;
            uint64_t k = 0;
            int sz = 0;
            bool in = false;
            if (c < nC) {
                k = keys[c];
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
    for (int i = tid; i < nsel; i += THREADS) {
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

    // ---- cache accounting ("D. Caching KV of Selected Tokens"): a selected
    // cluster is a hit when one of the last R steps selected it; misses (the
    // clusters a tiered cache would load) are listed in rank order; then this
    // step is recorded. CTA 0 of the problem, thread per selected cluster ----
    if (a.last_sel && rank == 0) {  // CTA-uniform
        if (tid == 0) {
            s_hits = 0;
            s_htok = 0;
        }
        __syncthreads();
        int32_t *last = a.last_sel + (size_t)p * a.C_cap;
        int mbase = 0;
        for (int r0 = 0; r0 < nsel; r0 += THREADS) {
            const int r = r0 + tid;
            int c = -1;
            bool hit = false;
            int tk = 0;
            if (r < nsel) {
                c = order[r];
                tk = min(csz[c], cnt - start[r]);
                const int l = last[c];
                hit = a.R > 0 && l < a.step && l >= a.step - a.R;
                last[c] = a.step;
            }
            const unsigned miss = __ballot_sync(FULL, r < nsel && !hit);
            const int wh = __reduce_add_sync(FULL, hit ? 1 : 0);
            const int wt = __reduce_add_sync(FULL, hit ? tk : 0);
            if (lane == 0) {
                s_wm[warp] = __popc(miss);
                atomicAdd(&s_hits, wh);
                atomicAdd(&s_htok, wt);
            }
            __syncthreads();
            int wpre = 0, tot = 0;
#pragma unroll
            for (int w2 = 0; w2 < WARPS; ++w2) {
                wpre += w2 < warp ? s_wm[w2] : 0;
                tot += s_wm[w2];
            }
            if (a.miss_list && r < nsel && !hit)
                a.miss_list[(size_t)p * a.C_cap + mbase + wpre + __popc(miss & lanemask_lt())] = c;
            mbase += tot;
            __syncthreads();
        }
        if (tid == 0) {
            int32_t *cs = a.cache_stats + (size_t)p * 4;
            cs[0] = s_hits;
            cs[1] = nsel;
            cs[2] = s_htok;
            cs[3] = cnt;
        }
    }

    // ---- 4. resolve this CTA's rows of the attended list ----
    const int tb = a.tail_b[p];
    const int ntail = max(0, a.tail_e[p] - tb);
    const int n_att = a.S + cnt + ntail;
    if (rank == 0 && tid == 0 && n_att > nc * a.chunk) dev_flag(CKV_DEVERR_INDEX);
    const int j0 = rank * a.chunk, j1 = min(n_att, j0 + a.chunk);
    constexpr int RB = 4;  // rows per thread whose perm loads are in flight together
    for (int jb = j0 + tid; jb < j1; jb += THREADS * RB) {
        int slot[RB];
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int j = jb + u * THREADS;
            slot[u] = -1;
            if (j < j1 && j >= a.S && j < a.S + cnt) {
                const int k = j - a.S;
                // last rank r with start[r] <= k (every listed cluster is non-empty)
                int lo = 0, hi = nsel - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (start[mid] <= k) lo = mid;
                    else hi = mid - 1;
                }
                slot[u] = off_s[order[lo]] + (k - start[lo]);
            }
        }
        int row[RB];
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int j = jb + u * THREADS;
            if (j < a.S) row[u] = j;
            else if (j < a.S + cnt) row[u] = (slot[u] >= 0 && slot[u] < a.perm_cap) ? __ldg(pp + slot[u]) : -1;
            else row[u] = tb + (j - a.S - cnt);
        }
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int j = jb + u * THREADS;
            if (j >= j1) break;
            int r = row[u];
            if (j >= a.S && j < a.S + cnt) a.sel_idx[(size_t)p * a.B + (j - a.S)] = r;
            if (r < 0 || r >= a.kv_rows) {
                dev_flag(CKV_DEVERR_INDEX);
                r = -1;
            }
            pos_s[j - j0] = r;
        }
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
