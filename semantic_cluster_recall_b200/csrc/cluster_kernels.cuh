// Clustering kernels except the tensor-core assignment: strided seeding,
// the FFMA assignment (fp32 keys), the cluster index (stable counting sort)
// and the centroid update.
//
// Method: "ClusterKV: Manipulating LLM KV Cache in Semantic Space for
// Recallable Compression" (arXiv 2412.03213v2): cosine k-means over the keys
// ("III.B Clustering in the Semantic Space"); a custom kernel sums the keys of
// each cluster and counts them, then divides ("IV.B Semantic Clustering");
// cluster sizes, prefix sums and token indices sorted by cluster are stored
// for selection ("IV.C Selection and Indexing").
#pragma once

#include "common.cuh"

namespace ckv {

// Round a double to bf16 (round to nearest, ties to even) in one step, from
// the bit pattern: 8 significant bits are kept and the 45 dropped mantissa
// bits decide the rounding. Values below the fp32 normal range take the
// fp32 path (two roundings), which no centroid of unit-scale keys reaches.
__device__ __forceinline__ uint16_t bf16_bits_rn(double x) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(x);
    const unsigned sign = (unsigned)(b >> 63) << 15;
    const int e = (int)((b >> 52) & 0x7ff) - 1023;
    if (x != x) return (uint16_t)(sign | 0x7fc0u);
    if (e > 127) return (uint16_t)(sign | 0x7f80u);
    if (e < -126) return __bfloat16_as_ushort(__float2bfloat16_rn((float)x));
    const unsigned long long m = b & ((1ull << 52) - 1);
    unsigned keep = (unsigned)(m >> 45);              // 7 stored mantissa bits
    const unsigned long long rem = m & ((1ull << 45) - 1);
    const unsigned long long halfway = 1ull << 44;
    unsigned v = ((unsigned)(e + 127) << 7) | keep;   // exponent and mantissa
    if (rem > halfway || (rem == halfway && (keep & 1u))) v += 1;  // may carry into the exponent
    if (v >= 0x7f80u) v = 0x7f80u;                    // rounded past the largest finite
    return (uint16_t)(sign | v);
}

template <typename T>
__device__ __forceinline__ void store4_rn(T *p, const double (&v)[4]);

template <>
__device__ __forceinline__ void store4_rn<float>(float *p, const double (&v)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4((float)v[0], (float)v[1], (float)v[2], (float)v[3]);
}

template <>
__device__ __forceinline__ void store4_rn<bf16>(bf16 *p, const double (&v)[4]) {
    uint2 u;
    u.x = (uint32_t)bf16_bits_rn(v[0]) | ((uint32_t)bf16_bits_rn(v[1]) << 16);
    u.y = (uint32_t)bf16_bits_rn(v[2]) | ((uint32_t)bf16_bits_rn(v[3]) << 16);
    *reinterpret_cast<uint2 *>(p) = u;
}

// the values store4_rn stores, as doubles
template <typename T>
__device__ __forceinline__ void round4_rn(const double (&v)[4], double (&r)[4]);

template <>
__device__ __forceinline__ void round4_rn<float>(const double (&v)[4], double (&r)[4]) {
#pragma unroll
    for (int t = 0; t < 4; ++t) r[t] = (double)(float)v[t];
}

template <>
__device__ __forceinline__ void round4_rn<bf16>(const double (&v)[4], double (&r)[4]) {
#pragma unroll
    for (int t = 0; t < 4; ++t) r[t] = (double)__uint_as_float((uint32_t)bf16_bits_rn(v[t]) << 16);
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// a1 seeding: centroid c starts at the key of position tok_begin + c*floor(n/C).
// One warp per centroid; lane l owns channels 4l..4l+3. The unit copy is
// normalised in double and rounded to the storage type once.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
k_init(const T *__restrict__ keys, int64_t pstride, int tok_begin, int n, int C, int cbase,
       int C_cap, float *__restrict__ cent, T *__restrict__ hat, T *__restrict__ lp, int metric,
       float *__restrict__ bias, int bstride) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x * 8 + warp;
    const int p = blockIdx.y;
    if (c >= C) return;
    const int stride = n / C;
    const T *row = keys + (int64_t)p * pstride + (int64_t)(tok_begin + c * stride) * D;
    const float4 v = load4(row + lane * 4);
    const double mu[4] = {v.x, v.y, v.z, v.w};  // exact
    const double ss = warp_sum_d(mu[0] * mu[0] + mu[1] * mu[1] + mu[2] * mu[2] + mu[3] * mu[3]);
    const size_t o = ((size_t)p * C_cap + cbase + c) * D + lane * 4;
    store4(cent + o, v);
    store4(lp + o, v);
    if (metric != CKV_COSINE) {  // the assignment copy is the key itself
        store4(hat + o, v);
        if (metric == CKV_L2) {
            const double hb = 0.5 * ss;  // half the squared norm of the (exact) copy
            if (lane == 0) bias[(size_t)p * bstride + c] = (float)hb;
        }
        return;
    }
    double h[4] = {0.0, 0.0, 0.0, 0.0};
    if (ss > 0.0) {
        const double nrm = sqrt(ss);
#pragma unroll
        for (int t = 0; t < 4; ++t) h[t] = mu[t] / nrm;
    }
    store4_rn(hat + o, h);
}

// ---------------------------------------------------------------------------
// a2 assignment on CUDA cores (fp32 keys): labels = argmax_c k . hat_c.
// CTA tile: 64 keys x 64 centroids per pass over the centroids, 256 threads,
// each owning a 4x4 register tile; operands staged k-major in shared memory
// so each thread reads one float4 of keys and one of centroids per channel.
// Running (best, index) per key; ties keep the lowest centroid index.
// ---------------------------------------------------------------------------
constexpr int AS_TILE = 64;
constexpr int AS_SMEM = 2 * D * AS_TILE * 4;

template <typename T>
__global__ void __launch_bounds__(256)
k_assign_simt(const T *__restrict__ keys, int64_t pstride, int tok_begin, int n,
              const T *__restrict__ hat, int C, int cbase, int C_cap,
              int32_t *__restrict__ labels, int perm_base, int perm_cap,
              const float *__restrict__ bias, int bstride) {
    extern __shared__ __align__(16) float smf[];
    float *Ks = smf;                  // [D][64], channel-major
    float *Ms = smf + D * AS_TILE;    // [D][64]
    const int p = blockIdx.y;
    const int row0 = blockIdx.x * AS_TILE;
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const T *kp = keys + (int64_t)p * pstride + (int64_t)tok_begin * D;
    const T *hp = hat + ((size_t)p * C_cap + cbase) * D;

    for (int e = tid; e < AS_TILE * (D / 4); e += 256) {
        const int r = e & (AS_TILE - 1), t4 = e >> 6;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row0 + r < n) v = load4(kp + (int64_t)(row0 + r) * D + t4 * 4);
        Ks[(t4 * 4 + 0) * AS_TILE + r] = v.x;
        Ks[(t4 * 4 + 1) * AS_TILE + r] = v.y;
        Ks[(t4 * 4 + 2) * AS_TILE + r] = v.z;
        Ks[(t4 * 4 + 3) * AS_TILE + r] = v.w;
    }

    float best[4];
    int bidx[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        best[i] = -INFINITY;
        bidx[i] = 0;
    }

    for (int c0 = 0; c0 < C; c0 += AS_TILE) {
        __syncthreads();
        for (int e = tid; e < AS_TILE * (D / 4); e += 256) {
            const int r = e & (AS_TILE - 1), t4 = e >> 6;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c0 + r < C) v = load4(hp + (size_t)(c0 + r) * D + t4 * 4);
            Ms[(t4 * 4 + 0) * AS_TILE + r] = v.x;
            Ms[(t4 * 4 + 1) * AS_TILE + r] = v.y;
            Ms[(t4 * 4 + 2) * AS_TILE + r] = v.z;
            Ms[(t4 * 4 + 3) * AS_TILE + r] = v.w;
        }
        __syncthreads();
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
        for (int t = 0; t < D; ++t) {
            const float4 a = *reinterpret_cast<const float4 *>(&Ks[t * AS_TILE + ty * 4]);
            const float4 b = *reinterpret_cast<const float4 *>(&Ms[t * AS_TILE + tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w};
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + tx * 4 + j;
            if (c < C) {
                // L2: minus half the centroid's squared norm (k . m - |m|^2 / 2)
                const float bj = bias ? bias[(size_t)p * bstride + c] : 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float sc = acc[i][j] - bj;
                    if (sc > best[i]) {
                        best[i] = sc;
                        bidx[i] = c;
                    }
                }
            }
        }
    }
    // reduce over the 16 threads sharing these keys (lanes differing in tx)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(FULL, best[i], o);
            const int oi = __shfl_xor_sync(FULL, bidx[i], o);
            if (ov > best[i] || (ov == best[i] && oi < bidx[i])) {
                best[i] = ov;
                bidx[i] = oi;
            }
        }
    }
    if (tx == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = row0 + ty * 4 + i;
            if (r < n) labels[(size_t)p * perm_cap + perm_base + r] = cbase + bidx[i];
        }
    }
}

// ---------------------------------------------------------------------------
// a4 cluster index: stable counting sort of labels into offsets + perm.
// Tokens are cut into chunks of IDX_CHUNK (one CTA each, IDX_WTOK per warp).
// (1) k_index_hist: per-chunk counts per cluster -> hist[p][c][chunk]
// (2) k_index_scan: exclusive scan of hist in (cluster, chunk) order, which is
//     exactly the output slot of each chunk's first member of each cluster;
//     also the offsets
// (3) k_index_scatter: each warp walks its tokens in order; __match_any_sync
//     ranks equal labels within a 32-token step, so positions stay ascending
//     within every cluster (stable), with no atomics on the output.
// ---------------------------------------------------------------------------
constexpr int IDX_WARPS = 8;
constexpr int IDX_WTOK = 256;
constexpr int IDX_CHUNK = IDX_WARPS * IDX_WTOK;

__device__ __forceinline__ void idx_count_warp(const int32_t *__restrict__ lab, int n, int C,
                                               int cbase, int chunk, int warp, int lane,
                                               int32_t *cnt) {
    const int start = chunk * IDX_CHUNK + warp * IDX_WTOK;
    for (int s = 0; s < IDX_WTOK; s += 32) {
        const int i = start + s + lane;
        if (i < n) {
            const int l = lab[i] - cbase;
            if ((unsigned)l < (unsigned)C) atomicAdd(&cnt[warp * C + l], 1);
            else dev_flag(CKV_DEVERR_LABEL);
        }
    }
}

__global__ void __launch_bounds__(256)
k_index_hist(const int32_t *__restrict__ labels, int perm_base, int perm_cap, int n, int C,
             int cbase, int nchunks, int32_t *__restrict__ hist) {
    extern __shared__ int32_t cnt[];  // [IDX_WARPS][C]
    const int p = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < IDX_WARPS * C; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    idx_count_warp(labels + (size_t)p * perm_cap + perm_base, n, C, cbase, chunk, warp, lane, cnt);
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        int s = 0;
#pragma unroll
        for (int w = 0; w < IDX_WARPS; ++w) s += cnt[w * C + c];
        hist[((size_t)p * C + c) * nchunks + chunk] = s;
    }
}

__global__ void __launch_bounds__(1024)
k_index_scan(int32_t *__restrict__ hist, int C, int nchunks, int perm_base, int cbase, int C_cap,
             int32_t *__restrict__ offsets) {
    __shared__ int32_t wsum[32];
    const int p = blockIdx.x;
    const int E = C * nchunks;
    int32_t *h = hist + (size_t)p * E;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int b = threadIdx.x * per, e = min(E, b + per);
    int local = 0;
    for (int k = b; k < e; ++k) local += h[k];
    // block exclusive scan of the per-thread sums
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
        int vi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(FULL, vi, o);
            if (lane >= o) vi += u;
        }
        wsum[lane] = vi - v;  // exclusive prefix of warp totals
    }
    __syncthreads();
    int run = wsum[warp] + incl - local;
    int32_t *off = offsets + (size_t)p * (C_cap + 1) + cbase;
    for (int k = b; k < e; ++k) {
        const int v = h[k];
        h[k] = run;
        if (k % nchunks == 0) off[k / nchunks] = perm_base + run;
        run += v;
    }
    if (threadIdx.x == blockDim.x - 1) off[C] = perm_base + run;
}

__global__ void __launch_bounds__(256)
k_index_scatter(const int32_t *__restrict__ labels, int perm_base, int perm_cap, int tok_begin,
                int n, int C, int cbase, int nchunks, const int32_t *__restrict__ base,
                int32_t *__restrict__ perm) {
    extern __shared__ int32_t run[];  // [IDX_WARPS][C]
    const int p = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t *lab = labels + (size_t)p * perm_cap + perm_base;
    for (int e = threadIdx.x; e < IDX_WARPS * C; e += blockDim.x) run[e] = 0;
    __syncthreads();
    // count again (cheap) so every warp knows where its members of c start
    {
        const int start = chunk * IDX_CHUNK + warp * IDX_WTOK;
        for (int s = 0; s < IDX_WTOK; s += 32) {
            const int i = start + s + lane;
            if (i < n) {
                const int l = lab[i] - cbase;
                if ((unsigned)l < (unsigned)C) atomicAdd(&run[warp * C + l], 1);
            }
        }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        int acc = base[((size_t)p * C + c) * nchunks + chunk];
#pragma unroll
        for (int w = 0; w < IDX_WARPS; ++w) {
            const int t = run[w * C + c];
            run[w * C + c] = acc;
            acc += t;
        }
    }
    __syncthreads();
    int32_t *out = perm + (size_t)p * perm_cap + perm_base;
    int32_t *myrun = run + warp * C;
    const int start = chunk * IDX_CHUNK + warp * IDX_WTOK;
    for (int s = 0; s < IDX_WTOK; s += 32) {
        const int i = start + s + lane;
        int l = -1;
        if (i < n) l = lab[i] - cbase;
        const bool ok = i < n && (unsigned)l < (unsigned)C;
        const unsigned active = __ballot_sync(FULL, ok);
        if (ok) {
            const unsigned peers = __match_any_sync(active, l);
            const int rank = __popc(peers & lanemask_lt());
            const int pos = myrun[l] + rank;
            out[pos] = tok_begin + i;
            __syncwarp(active);
            if (rank == __popc(peers) - 1) myrun[l] = pos + 1;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// a3 centroid update: one warp per cluster gathers its member rows through
// perm; lane l owns channels 4l..4l+3 (one 256-byte bf16 row per warp load)
// and keeps UPD_ROWS rows in flight. Each channel is summed in double, one
// row at a time in perm order (ascending position), so the sum, the mean,
// and the rounded copies do not depend on the launch shape. Deterministic,
// no atomics.
// ---------------------------------------------------------------------------
constexpr int UPD_ROWS = 16;  // rows in flight per warp

// Raw bits of 4 consecutive elements (loaded first, converted later, so all
// loads of a batch are in flight together).
template <typename T>
struct Raw4;

template <>
struct Raw4<bf16> {
    uint2 u;
    __device__ __forceinline__ void load(const bf16 *p) { u = __ldg(reinterpret_cast<const uint2 *>(p)); }
    __device__ __forceinline__ void zero() { u = make_uint2(0, 0); }
    __device__ __forceinline__ void add_to(double (&acc)[4]) const {
        acc[0] += (double)__uint_as_float(u.x << 16);
        acc[1] += (double)__uint_as_float(u.x & 0xffff0000u);
        acc[2] += (double)__uint_as_float(u.y << 16);
        acc[3] += (double)__uint_as_float(u.y & 0xffff0000u);
    }
};

template <>
struct Raw4<float> {
    float4 f;
    __device__ __forceinline__ void load(const float *p) { f = __ldg(reinterpret_cast<const float4 *>(p)); }
    __device__ __forceinline__ void zero() { f = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void add_to(double (&acc)[4]) const {
        acc[0] += (double)f.x;
        acc[1] += (double)f.y;
        acc[2] += (double)f.z;
        acc[3] += (double)f.w;
    }
};

template <typename T>
__global__ void __launch_bounds__(256)
k_update(const T *__restrict__ keys, int64_t pstride, int tok_begin, int tok_end, int C,
         int cbase, int C_cap, const int32_t *__restrict__ offsets,
         const int32_t *__restrict__ perm, int perm_cap, float *__restrict__ cent,
         T *__restrict__ hat, T *__restrict__ lp, int32_t *__restrict__ sizes, int metric,
         float *__restrict__ bias, int bstride) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x * 8 + warp;
    const int p = blockIdx.y;
    if (c >= C) return;
    const int32_t *off = offsets + (size_t)p * (C_cap + 1) + cbase;
    const int o0 = off[c], o1 = off[c + 1];
    int32_t *sz = sizes + (size_t)p * C_cap + cbase + c;
    if (o0 < 0 || o1 < o0 || o1 > perm_cap) {
        if (lane == 0) {
            dev_flag(CKV_DEVERR_OFFSETS);
            *sz = 0;
        }
        return;
    }
    const T *kb = keys + (int64_t)p * pstride + lane * 4;
    const int32_t *pp = perm + (size_t)p * perm_cap;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int j0 = o0; j0 < o1; j0 += 32) {
        const int cnt = min(32, o1 - j0);
        const int pos = lane < cnt ? pp[j0 + lane] : -1;
        for (int k = 0; k < cnt; k += UPD_ROWS) {
            Raw4<T> r[UPD_ROWS];
#pragma unroll
            for (int u = 0; u < UPD_ROWS; ++u) {
                const int kk = k + u;  // < 32 always
                const int ps = __shfl_sync(FULL, pos, kk & 31);
                r[u].zero();
                if (kk < cnt) {
                    if (ps >= tok_begin && ps < tok_end) r[u].load(kb + (int64_t)ps * D);
                    else if (lane == 0) dev_flag(CKV_DEVERR_PERM);
                }
            }
#pragma unroll
            for (int u = 0; u < UPD_ROWS; ++u) r[u].add_to(acc);  // perm order; +0 is exact
        }
    }
    const int n = o1 - o0;
    if (lane == 0) *sz = n;
    if (n == 0) return;
    double mu[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) mu[t] = acc[t] / (double)n;
    const size_t o = ((size_t)p * C_cap + cbase + c) * D + lane * 4;
    if (metric != CKV_COSINE) {  // assignment copy = the mean rounded to storage
        double r[4];
        round4_rn<T>(mu, r);
        store4_rn<float>(cent + o, mu);
        store4_rn<T>(lp + o, mu);
        store4_rn<T>(hat + o, mu);
        if (metric == CKV_L2) {
            const double hb =
                0.5 * warp_sum_d(r[0] * r[0] + r[1] * r[1] + r[2] * r[2] + r[3] * r[3]);
            if (lane == 0) bias[(size_t)p * bstride + c] = (float)hb;
        }
        return;
    }
    const double ss = warp_sum_d(mu[0] * mu[0] + mu[1] * mu[1] + mu[2] * mu[2] + mu[3] * mu[3]);
    if (!(ss > 0.0)) return;
    const double nrm = sqrt(ss);
    double h[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) h[t] = mu[t] / nrm;
    store4_rn<float>(cent + o, mu);
    store4_rn<T>(lp + o, mu);
    store4_rn<T>(hat + o, h);
}

}  // namespace ckv
