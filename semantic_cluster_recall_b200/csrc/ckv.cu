// libckv: host side of the C ABI declared in include/ckv.h. Validates every
// argument before launching, picks launch shapes, and launches the sm_100a
// kernels of the *.cuh files on the caller's stream. Allocates nothing.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "cluster_kernels.cuh"
#include "assign_tc.cuh"
#include "select_kernels.cuh"
#include "decode_kernels.cuh"
#include "select_decode.cuh"

using namespace ckv;

namespace {

thread_local char g_err[512];

ckv_status fail(ckv_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

ckv_status ok() {
    g_err[0] = 0;
    return CKV_OK;
}

ckv_status launched(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(CKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return ok();
}

inline cudaStream_t S(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline bool aligned(const void *p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

constexpr int MAX_DEVICES = 64;

int sm_count() {
    static int cache[MAX_DEVICES] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= MAX_DEVICES) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Raise a kernel's dynamic shared memory limit once per device.
template <typename K>
cudaError_t smem_optin(K kernel, size_t bytes, int slot) {
    static std::mutex mu;
    static size_t done[64][MAX_DEVICES] = {{0}};
    if (bytes <= 48 * 1024) return cudaSuccess;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= MAX_DEVICES || slot < 0 || slot >= 64)
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    std::lock_guard<std::mutex> g(mu);
    if (done[slot][dev] >= bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done[slot][dev] = bytes;
    return e;
}

// slots for smem_optin (one per kernel instantiation that may exceed 48 KB)
enum { SLOT_ASSIGN_F32 = 0, SLOT_ASSIGN_BF16, SLOT_HIST, SLOT_SCATTER, SLOT_RANK, SLOT_ASSIGN_TC,
       SLOT_SD_BASE /* + 12 fused select-decode instantiations */ };

bool valid_dtype(ckv_dtype dt) { return dt == CKV_F32 || dt == CKV_BF16; }

#ifndef CKV_SD_PDL
#define CKV_SD_PDL 1  // fused steps launched as programmatic dependents
#endif

bool valid_metric(int m) { return m == CKV_COSINE || m == CKV_INNER || m == CKV_L2; }

int nchunks_of(int n) { return (n + IDX_CHUNK - 1) / IDX_CHUNK; }

// common checks of a clustering region
ckv_status check_region(const void *keys, ckv_dtype dt, int P, int64_t pstride, int d,
                        int tok_begin, int tok_end, int C, int cbase, int C_cap) {
    if (!keys) return fail(CKV_ERR_INVALID, "keys is null");
    if (!valid_dtype(dt)) return fail(CKV_ERR_INVALID, "unknown dtype %d", (int)dt);
    if (d != D) return fail(CKV_ERR_INVALID, "d must be 128 (got %d)", d);
    if (P < 1) return fail(CKV_ERR_INVALID, "P must be >= 1 (got %d)", P);
    if (P > 65535) return fail(CKV_ERR_INVALID, "P must be <= 65535 (got %d)", P);
    if (tok_begin < 0 || tok_end <= tok_begin)
        return fail(CKV_ERR_INVALID, "bad token range [%d, %d)", tok_begin, tok_end);
    if (pstride < (int64_t)tok_end * D)
        return fail(CKV_ERR_INVALID, "problem_stride %lld < tok_end * d", (long long)pstride);
    if (C < 1) return fail(CKV_ERR_INVALID, "C must be >= 1 (got %d)", C);
    if (cbase < 0 || C_cap < 1 || cbase + C > C_cap || C_cap > CKV_MAX_CLUSTERS)
        return fail(CKV_ERR_INVALID, "clusters [%d, %d) do not fit C_cap %d (max %d)", cbase,
                    cbase + C, C_cap, CKV_MAX_CLUSTERS);
    const size_t esz = dt == CKV_BF16 ? 2 : 4;
    if (!aligned(keys, 16) || ((size_t)pstride * esz) % 16)
        return fail(CKV_ERR_INVALID, "keys and problem_stride must be 16-byte aligned");
    return CKV_OK;
}

ckv_status check_perm(int n, int perm_base, int perm_cap) {
    if (perm_base < 0 || perm_cap < 1 || (int64_t)perm_base + n > perm_cap)
        return fail(CKV_ERR_INVALID, "perm slots [%d, %d) do not fit perm_cap %d", perm_base,
                    perm_base + n, perm_cap);
    return CKV_OK;
}

template <typename T>
ckv_status launch_init(const T *keys, int P, int64_t pstride, int tok_begin, int n, int C,
                       int cbase, int C_cap, float *cent, T *hat, T *lp, int metric, float *bias,
                       int bstride, cudaStream_t st) {
    dim3 grid((C + 7) / 8, P);
    k_init<T><<<grid, 256, 0, st>>>(keys, pstride, tok_begin, n, C, cbase, C_cap, cent, hat, lp,
                                    metric, bias, bstride);
    return launched("k_init");
}

ckv_status launch_assign_f32(const float *keys, int P, int64_t pstride, int tok_begin, int n,
                             const float *hat, int C, int cbase, int C_cap, int32_t *labels,
                             int perm_base, int perm_cap, const float *bias, int bstride,
                             cudaStream_t st) {
    cudaError_t e = smem_optin(k_assign_simt<float>, AS_SMEM, SLOT_ASSIGN_F32);
    if (e != cudaSuccess) return fail(CKV_ERR_CUDA, "smem opt-in: %s", cudaGetErrorString(e));
    dim3 grid((n + AS_TILE - 1) / AS_TILE, P);
    k_assign_simt<float><<<grid, 256, AS_SMEM, st>>>(keys, pstride, tok_begin, n, hat, C, cbase,
                                                     C_cap, labels, perm_base, perm_cap, bias,
                                                     bstride);
    return launched("k_assign_simt");
}

ckv_status launch_index(const int32_t *labels, int P, int tok_begin, int n, int C, int cbase,
                        int C_cap, int perm_base, int perm_cap, int32_t *offsets, int32_t *perm,
                        void *ws, cudaStream_t st) {
    const int nch = nchunks_of(n);
    int32_t *hist = reinterpret_cast<int32_t *>(ws);
    const size_t smem = (size_t)IDX_WARPS * C * sizeof(int32_t);
    cudaError_t e = smem_optin(k_index_hist, smem, SLOT_HIST);
    if (e == cudaSuccess) e = smem_optin(k_index_scatter, smem, SLOT_SCATTER);
    if (e != cudaSuccess) return fail(CKV_ERR_CUDA, "smem opt-in: %s", cudaGetErrorString(e));
    dim3 grid(nch, P);
    k_index_hist<<<grid, 256, smem, st>>>(labels, perm_base, perm_cap, n, C, cbase, nch, hist);
    ckv_status s = launched("k_index_hist");
    if (s) return s;
    k_index_scan<<<P, 1024, 0, st>>>(hist, C, nch, perm_base, cbase, C_cap, offsets);
    if ((s = launched("k_index_scan"))) return s;
    k_index_scatter<<<grid, 256, smem, st>>>(labels, perm_base, perm_cap, tok_begin, n, C, cbase,
                                             nch, hist, perm);
    return launched("k_index_scatter");
}

template <typename T>
ckv_status launch_update(const T *keys, int P, int64_t pstride, int tok_begin, int tok_end, int C,
                         int cbase, int C_cap, const int32_t *offsets, const int32_t *perm,
                         int perm_cap, float *cent, T *hat, T *lp, int32_t *sizes, int metric,
                         float *bias, int bstride, cudaStream_t st) {
    dim3 grid((C + 7) / 8, P);
    k_update<T><<<grid, 256, 0, st>>>(keys, pstride, tok_begin, tok_end, C, cbase, C_cap, offsets,
                                      perm, perm_cap, cent, hat, lp, sizes, metric, bias, bstride);
    return launched("k_update");
}

ckv_status launch_assign(const void *keys, ckv_dtype dt, int P, int64_t pstride, int tok_begin,
                         int n, const void *hat, int C, int cbase, int C_cap, int32_t *labels,
                         int perm_base, int perm_cap, cudaStream_t st, int max_sms,
                         const float *bias, int bstride) {
    if (dt == CKV_F32)
        return launch_assign_f32((const float *)keys, P, pstride, tok_begin, n, (const float *)hat,
                                 C, cbase, C_cap, labels, perm_base, perm_cap, bias, bstride, st);
    ckv_status s = launch_assign_bf16((const bf16 *)keys, P, pstride, tok_begin, n,
                                      (const bf16 *)hat, C, cbase, C_cap, labels, perm_base,
                                      perm_cap,
                                      max_sms > 0 && max_sms < sm_count() ? max_sms : sm_count(),
                                      bias, bstride, st);
    if (s) return fail(s, "tensor-core assignment launch failed (%s)",
                       cudaGetErrorString(cudaGetLastError()));
    return ok();
}

// partial-result slots of the decode workspace (chunks are >= 32 rows)
size_t decode_parts(int P, int G, int max_rows) {
    if (max_rows < 1) max_rows = 1;
    return (size_t)P * (size_t)((max_rows + 31) / 32) * (size_t)G;
}

// decode split heuristic: about 4 CTAs per SM in total, chunks of >= 32 rows
void decode_shape(int P, int max_rows, int sms, int *chunk, int *nsplit) {
    if (max_rows < 1) max_rows = 1;
    const int target = 4 * sms;
    int want = (target + P - 1) / P;
    if (want < 1) want = 1;
    int c = (max_rows + want - 1) / want;
    c = ((c + 15) / 16) * 16;
    if (c < 32) c = 32;
    *chunk = c;
    *nsplit = (max_rows + c - 1) / c;
}

// instantiations of the fused step: (kernel, smem_optin slot)
struct sd_kernel {
    const void *fn;
    int slot;
};

template <typename T, int G, int U>
sd_kernel sd_entry(int slot) {
    return {reinterpret_cast<const void *>(&sd::k_select_decode<T, G, U>), SLOT_SD_BASE + slot};
}

sd_kernel sd_pick(ckv_dtype dt, int G, int U) {
    if (dt == CKV_BF16) {
        if (G == 4) return U == 2 ? sd_entry<bf16, 4, 2>(10) : sd_entry<bf16, 4, 6>(0);
        if (G == 2) return U == 4 ? sd_entry<bf16, 2, 4>(1) : sd_entry<bf16, 2, 9>(2);
        return U == 4 ? sd_entry<bf16, 1, 4>(3) : sd_entry<bf16, 1, 9>(4);
    }
    if (G == 4) return U == 2 ? sd_entry<float, 4, 2>(11) : sd_entry<float, 4, 6>(5);
    if (G == 2) return U == 4 ? sd_entry<float, 2, 4>(6) : sd_entry<float, 2, 9>(7);
    return U == 4 ? sd_entry<float, 1, 4>(8) : sd_entry<float, 1, 9>(9);
}

cudaError_t sd_optin(const sd_kernel &k, size_t smem) {
    return smem_optin(k.fn, smem, k.slot);
}

// How many thread-block clusters of nc CTAs (smem bytes each) the device
// holds at once; cached per (device, instantiation, nc, smem).
cudaError_t sd_clusters_per_wave(const sd_kernel &k, int nc, size_t smem, int *out) {
    struct Entry {
        int dev, slot, nc;
        size_t smem;
        int fit;
    };
    static std::mutex mu;
    static Entry cache[256];
    static int n_cache = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> g(mu);
        for (int i = 0; i < n_cache; ++i)
            if (cache[i].dev == dev && cache[i].slot == k.slot && cache[i].nc == nc &&
                cache[i].smem == smem) {
                *out = cache[i].fit;
                return cudaSuccess;
            }
    }
    cudaError_t e = sd_optin(k, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc, 1, 1);
    cfg.blockDim = dim3(sd::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int fit = 0;
    e = cudaOccupancyMaxActiveClusters(&fit, k.fn, &cfg);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> g(mu);
    if (n_cache < 256) cache[n_cache++] = {dev, k.slot, nc, smem, fit};
    *out = fit;
    return cudaSuccess;
}

}  // namespace

extern "C" {

int ckv_version(void) { return 1; }

const char *ckv_status_string(int s) {
    switch (s) {
        case CKV_OK: return "ok";
        case CKV_ERR_INVALID: return "invalid argument";
        case CKV_ERR_CUDA: return "CUDA error";
        case CKV_ERR_TIMEOUT: return "device wait timed out";
        case CKV_ERR_UNSUPPORTED: return "unsupported";
        default: return "unknown status";
    }
}

const char *ckv_last_error(void) { return g_err; }

ckv_status ckv_device_error(unsigned int *flags, int clear, void *stream) {
    if (!flags) return fail(CKV_ERR_INVALID, "flags is null");
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_devflags, sizeof(v), 0,
                                              cudaMemcpyDeviceToHost, S(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
    if (e == cudaSuccess && clear) {
        const unsigned int z = 0;
        e = cudaMemcpyToSymbolAsync(g_devflags, &z, sizeof(z), 0, cudaMemcpyHostToDevice, S(stream));
        if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
    }
    if (e != cudaSuccess) return fail(CKV_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
    *flags = v;
    if (v & CKV_DEVERR_TIMEOUT) return fail(CKV_ERR_TIMEOUT, "a bounded device wait timed out");
    return ok();
}

size_t ckv_index_workspace_bytes(int P, int n_tok, int C) {
    if (P < 1 || n_tok < 1 || C < 1) return 0;
    return align256((size_t)P * C * nchunks_of(n_tok) * sizeof(int32_t));
}

size_t ckv_cluster_workspace_bytes(int P, int n_tok, int C) {
    return ckv_index_workspace_bytes(P, n_tok, C);
}

size_t ckv_cluster_ex_workspace_bytes(int P, int n_tok, int C, int metric) {
    const size_t w = ckv_index_workspace_bytes(P, n_tok, C);
    if (w == 0 || !valid_metric(metric)) return 0;
    return metric == CKV_L2 ? w + align256((size_t)P * C * sizeof(float)) : w;
}

ckv_status ckv_init_centroids(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                              int tok_begin, int tok_end, int C, int cluster_base, int C_cap,
                              float *centroids, void *centroids_hat, void *centroids_lp,
                              void *stream) {
    return ckv_init_centroids_ex(keys, dt, P, problem_stride, d, tok_begin, tok_end, C,
                                 cluster_base, C_cap, centroids, centroids_hat, centroids_lp,
                                 CKV_COSINE, nullptr, stream);
}

ckv_status ckv_init_centroids_ex(const void *keys, ckv_dtype dt, int P, int64_t problem_stride,
                                 int d, int tok_begin, int tok_end, int C, int cluster_base,
                                 int C_cap, float *centroids, void *centroids_hat,
                                 void *centroids_lp, int metric, float *bias, void *stream) {
    ckv_status s = check_region(keys, dt, P, problem_stride, d, tok_begin, tok_end, C,
                                cluster_base, C_cap);
    if (s) return s;
    const int n = tok_end - tok_begin;
    if (n < C) return fail(CKV_ERR_INVALID, "fewer tokens (%d) than clusters (%d)", n, C);
    if (!centroids || !centroids_hat || !centroids_lp)
        return fail(CKV_ERR_INVALID, "null centroid array");
    if (!valid_metric(metric)) return fail(CKV_ERR_INVALID, "unknown metric %d", metric);
    if (metric == CKV_L2 && !bias) return fail(CKV_ERR_INVALID, "L2 needs the bias array");
    float *b = metric == CKV_L2 ? bias + cluster_base : nullptr;
    if (dt == CKV_BF16)
        return launch_init((const bf16 *)keys, P, problem_stride, tok_begin, n, C, cluster_base,
                           C_cap, centroids, (bf16 *)centroids_hat, (bf16 *)centroids_lp, metric,
                           b, C_cap, S(stream));
    return launch_init((const float *)keys, P, problem_stride, tok_begin, n, C, cluster_base, C_cap,
                       centroids, (float *)centroids_hat, (float *)centroids_lp, metric, b, C_cap,
                       S(stream));
}

ckv_status ckv_assign(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                      int tok_begin, int tok_end, const void *centroids_hat, int C,
                      int cluster_base, int C_cap, int32_t *labels, int perm_base, int perm_cap,
                      void *stream) {
    return ckv_assign_ex(keys, dt, P, problem_stride, d, tok_begin, tok_end, centroids_hat, C,
                         cluster_base, C_cap, labels, perm_base, perm_cap, nullptr, stream);
}

ckv_status ckv_assign_ex(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                         int tok_begin, int tok_end, const void *centroids_hat, int C,
                         int cluster_base, int C_cap, int32_t *labels, int perm_base,
                         int perm_cap, const float *bias, void *stream) {
    ckv_status s = check_region(keys, dt, P, problem_stride, d, tok_begin, tok_end, C,
                                cluster_base, C_cap);
    if (s) return s;
    const int n = tok_end - tok_begin;
    if (!centroids_hat || !labels) return fail(CKV_ERR_INVALID, "null centroids_hat or labels");
    if ((s = check_perm(n, perm_base, perm_cap))) return s;
    if (!aligned(centroids_hat, 16)) return fail(CKV_ERR_INVALID, "centroids_hat misaligned");
    if (bias && !aligned(bias, 4)) return fail(CKV_ERR_INVALID, "bias misaligned");
    return launch_assign(keys, dt, P, problem_stride, tok_begin, n, centroids_hat, C, cluster_base,
                         C_cap, labels, perm_base, perm_cap, S(stream), 0,
                         bias ? bias + cluster_base : nullptr, C_cap);
}

ckv_status ckv_index(const int32_t *labels, int P, int tok_begin, int tok_end, int C,
                     int cluster_base, int C_cap, int perm_base, int perm_cap, int32_t *offsets,
                     int32_t *perm, void *workspace, size_t ws_bytes, void *stream) {
    if (!labels || !offsets || !perm) return fail(CKV_ERR_INVALID, "null labels/offsets/perm");
    if (P < 1 || P > 65535) return fail(CKV_ERR_INVALID, "bad P %d", P);
    if (tok_begin < 0 || tok_end <= tok_begin)
        return fail(CKV_ERR_INVALID, "bad token range [%d, %d)", tok_begin, tok_end);
    const int n = tok_end - tok_begin;
    if (C < 1 || cluster_base < 0 || cluster_base + C > C_cap || C_cap > CKV_MAX_CLUSTERS)
        return fail(CKV_ERR_INVALID, "bad clusters C=%d base=%d C_cap=%d", C, cluster_base, C_cap);
    ckv_status s = check_perm(n, perm_base, perm_cap);
    if (s) return s;
    if (!workspace || ws_bytes < ckv_index_workspace_bytes(P, n, C) || !aligned(workspace, 256))
        return fail(CKV_ERR_INVALID, "workspace too small or not 256-byte aligned");
    return launch_index(labels, P, tok_begin, n, C, cluster_base, C_cap, perm_base, perm_cap,
                        offsets, perm, workspace, S(stream));
}

ckv_status ckv_update(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                      int tok_begin, int tok_end, int C, int cluster_base, int C_cap,
                      const int32_t *offsets, const int32_t *perm, int perm_cap,
                      float *centroids, void *centroids_hat, void *centroids_lp, int32_t *sizes,
                      void *stream) {
    return ckv_update_ex(keys, dt, P, problem_stride, d, tok_begin, tok_end, C, cluster_base,
                         C_cap, offsets, perm, perm_cap, centroids, centroids_hat, centroids_lp,
                         sizes, CKV_COSINE, nullptr, stream);
}

namespace {
ckv_status update_impl(const void *keys, ckv_dtype dt, int P, int64_t problem_stride,
                       int tok_begin, int tok_end, int C, int cluster_base, int C_cap,
                       const int32_t *offsets, const int32_t *perm, int perm_cap,
                       float *centroids, void *centroids_hat, void *centroids_lp, int32_t *sizes,
                       int metric, float *bias, int bstride, cudaStream_t st) {
    if (dt == CKV_BF16)
        return launch_update((const bf16 *)keys, P, problem_stride, tok_begin, tok_end, C,
                             cluster_base, C_cap, offsets, perm, perm_cap, centroids,
                             (bf16 *)centroids_hat, (bf16 *)centroids_lp, sizes, metric, bias,
                             bstride, st);
    return launch_update((const float *)keys, P, problem_stride, tok_begin, tok_end, C,
                         cluster_base, C_cap, offsets, perm, perm_cap, centroids,
                         (float *)centroids_hat, (float *)centroids_lp, sizes, metric, bias,
                         bstride, st);
}
}  // namespace

ckv_status ckv_update_ex(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                         int tok_begin, int tok_end, int C, int cluster_base, int C_cap,
                         const int32_t *offsets, const int32_t *perm, int perm_cap,
                         float *centroids, void *centroids_hat, void *centroids_lp,
                         int32_t *sizes, int metric, float *bias, void *stream) {
    ckv_status s = check_region(keys, dt, P, problem_stride, d, tok_begin, tok_end, C,
                                cluster_base, C_cap);
    if (s) return s;
    if (!offsets || !perm || !centroids || !centroids_hat || !centroids_lp || !sizes)
        return fail(CKV_ERR_INVALID, "null pointer argument");
    if (perm_cap < 1) return fail(CKV_ERR_INVALID, "bad perm_cap %d", perm_cap);
    if (!valid_metric(metric)) return fail(CKV_ERR_INVALID, "unknown metric %d", metric);
    if (metric == CKV_L2 && !bias) return fail(CKV_ERR_INVALID, "L2 needs the bias array");
    return update_impl(keys, dt, P, problem_stride, tok_begin, tok_end, C, cluster_base, C_cap,
                       offsets, perm, perm_cap, centroids, centroids_hat, centroids_lp, sizes,
                       metric, metric == CKV_L2 ? bias + cluster_base : nullptr, C_cap, S(stream));
}

ckv_status ckv_cluster(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                       int tok_begin, int tok_end, int C, int iters, int cluster_base,
                       int perm_base, int C_cap, int perm_cap, float *centroids,
                       void *centroids_hat, void *centroids_lp, int32_t *labels, int32_t *sizes,
                       int32_t *offsets, int32_t *perm, void *workspace, size_t ws_bytes,
                       void *stream) {
    return ckv_cluster_ex(keys, dt, P, problem_stride, d, tok_begin, tok_end, C, iters,
                          cluster_base, perm_base, C_cap, perm_cap, centroids, centroids_hat,
                          centroids_lp, labels, sizes, offsets, perm, workspace, ws_bytes,
                          CKV_COSINE, 0, stream);
}

ckv_status ckv_cluster_ex(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                          int tok_begin, int tok_end, int C, int iters, int cluster_base,
                          int perm_base, int C_cap, int perm_cap, float *centroids,
                          void *centroids_hat, void *centroids_lp, int32_t *labels,
                          int32_t *sizes, int32_t *offsets, int32_t *perm, void *workspace,
                          size_t ws_bytes, int metric, int max_sms, void *stream) {
    if (max_sms < 0) return fail(CKV_ERR_INVALID, "max_sms must be >= 0 (got %d)", max_sms);
    if (!valid_metric(metric)) return fail(CKV_ERR_INVALID, "unknown metric %d", metric);
    ckv_status s = check_region(keys, dt, P, problem_stride, d, tok_begin, tok_end, C,
                                cluster_base, C_cap);
    if (s) return s;
    const int n = tok_end - tok_begin;
    if (n < C) return fail(CKV_ERR_INVALID, "fewer tokens (%d) than clusters (%d)", n, C);
    if (iters < 1) return fail(CKV_ERR_INVALID, "iters must be >= 1 (got %d)", iters);
    if (!centroids || !centroids_hat || !centroids_lp || !labels || !sizes || !offsets || !perm)
        return fail(CKV_ERR_INVALID, "null output array");
    if ((s = check_perm(n, perm_base, perm_cap))) return s;
    if (!workspace || ws_bytes < ckv_cluster_ex_workspace_bytes(P, n, C, metric) ||
        !aligned(workspace, 256))
        return fail(CKV_ERR_INVALID, "workspace too small or not 256-byte aligned");
    if (!aligned(centroids_hat, 16) || !aligned(centroids_lp, 16) || !aligned(centroids, 16))
        return fail(CKV_ERR_INVALID, "centroid arrays must be 16-byte aligned");
    cudaStream_t st = S(stream);
    // L2: half the squared norm of each assignment copy, [P][C] after the histograms
    float *bias = metric == CKV_L2
                      ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                  ckv_index_workspace_bytes(P, n, C))
                      : nullptr;
    if (dt == CKV_BF16)
        s = launch_init((const bf16 *)keys, P, problem_stride, tok_begin, n, C, cluster_base, C_cap,
                        centroids, (bf16 *)centroids_hat, (bf16 *)centroids_lp, metric, bias, C,
                        st);
    else
        s = launch_init((const float *)keys, P, problem_stride, tok_begin, n, C, cluster_base,
                        C_cap, centroids, (float *)centroids_hat, (float *)centroids_lp, metric,
                        bias, C, st);
    if (s) return s;
    for (int it = 0; it < iters; ++it) {
        if ((s = launch_assign(keys, dt, P, problem_stride, tok_begin, n, centroids_hat, C,
                               cluster_base, C_cap, labels, perm_base, perm_cap, st, max_sms, bias,
                               C)))
            return s;
        if ((s = launch_index(labels, P, tok_begin, n, C, cluster_base, C_cap, perm_base, perm_cap,
                              offsets, perm, workspace, st)))
            return s;
        if ((s = update_impl(keys, dt, P, problem_stride, tok_begin, tok_end, C, cluster_base,
                             C_cap, offsets, perm, perm_cap, centroids, centroids_hat,
                             centroids_lp, sizes, metric, bias, C, st)))
            return s;
    }
    return ok();
}

size_t ckv_select_workspace_bytes(int P, int C_cap) {
    if (P < 1 || C_cap < 1) return 0;
    return align256((size_t)P * C_cap * sizeof(float));
}

ckv_status ckv_select(const void *q, ckv_dtype dt, int P, int G, int d, const void *centroids_lp,
                      const int32_t *n_clusters, int C_cap, const int32_t *offsets,
                      const int32_t *perm, int perm_cap, int budget, int32_t *sel_idx,
                      int32_t *sel_cnt, void *workspace, size_t ws_bytes, void *stream) {
    if (!q || !centroids_lp || !n_clusters || !offsets || !perm || !sel_cnt)
        return fail(CKV_ERR_INVALID, "null pointer argument");
    if (budget > 0 && !sel_idx) return fail(CKV_ERR_INVALID, "sel_idx is null");
    if (!valid_dtype(dt)) return fail(CKV_ERR_INVALID, "unknown dtype %d", (int)dt);
    if (d != D) return fail(CKV_ERR_INVALID, "d must be 128 (got %d)", d);
    if (P < 1 || P > 65535) return fail(CKV_ERR_INVALID, "bad P %d", P);
    if (G < 1 || G > 8) return fail(CKV_ERR_INVALID, "G must be in [1, 8] (got %d)", G);
    if (C_cap < 1 || C_cap > CKV_MAX_CLUSTERS) return fail(CKV_ERR_INVALID, "bad C_cap %d", C_cap);
    if (perm_cap < 1) return fail(CKV_ERR_INVALID, "bad perm_cap %d", perm_cap);
    if (budget < 0) return fail(CKV_ERR_INVALID, "budget must be >= 0 (got %d)", budget);
    if (!workspace || ws_bytes < ckv_select_workspace_bytes(P, C_cap) || !aligned(workspace, 256))
        return fail(CKV_ERR_INVALID, "workspace too small or not 256-byte aligned");
    if (!aligned(q, 16) || !aligned(centroids_lp, 16))
        return fail(CKV_ERR_INVALID, "q and centroids_lp must be 16-byte aligned");
    cudaStream_t st = S(stream);
    float *scores = reinterpret_cast<float *>(workspace);
    dim3 g1((C_cap + 7) / 8, P);
#define CKV_SCORE(T, GG) k_score<T, GG><<<g1, 256, 0, st>>>((const T *)q, (const T *)centroids_lp, n_clusters, C_cap, scores)
#define CKV_SCORE_G(T)                    \
    switch (G) {                          \
        case 1: CKV_SCORE(T, 1); break;   \
        case 2: CKV_SCORE(T, 2); break;   \
        case 3: CKV_SCORE(T, 3); break;   \
        case 4: CKV_SCORE(T, 4); break;   \
        case 5: CKV_SCORE(T, 5); break;   \
        case 6: CKV_SCORE(T, 6); break;   \
        case 7: CKV_SCORE(T, 7); break;   \
        default: CKV_SCORE(T, 8); break;  \
    }
    if (dt == CKV_BF16) {
        CKV_SCORE_G(bf16)
    } else {
        CKV_SCORE_G(float)
    }
#undef CKV_SCORE_G
#undef CKV_SCORE
    ckv_status s = launched("k_score");
    if (s) return s;
    const size_t smem = (size_t)C_cap * 36;
    cudaError_t e = smem_optin(k_rankfill, smem, SLOT_RANK);
    if (e != cudaSuccess) return fail(CKV_ERR_CUDA, "smem opt-in: %s", cudaGetErrorString(e));
    k_rankfill<<<P, 1024, smem, st>>>(scores, n_clusters, C_cap, offsets, perm, perm_cap, budget,
                                       sel_idx, sel_cnt);
    return launched("k_rankfill");
}

ckv_status ckv_select_decode(const void *q, ckv_dtype dt, int P, int G, int d,
                             const void *centroids_lp, const int32_t *n_clusters, int C_cap,
                             const int32_t *offsets, const int32_t *perm, int perm_cap,
                             int budget, int32_t *sel_idx, int32_t *sel_cnt, const void *K,
                             const void *V, int64_t kv_problem_stride, int kv_rows, int sink,
                             const int32_t *tail_begin, const int32_t *tail_end, int max_tail,
                             float scale, float *out, void *stream) {
    return ckv_select_decode_cached(q, dt, P, G, d, centroids_lp, n_clusters, C_cap, offsets,
                                    perm, perm_cap, budget, sel_idx, sel_cnt, K, V,
                                    kv_problem_stride, kv_rows, sink, tail_begin, tail_end,
                                    max_tail, scale, out, nullptr, 0, 0, nullptr, nullptr,
                                    stream);
}

ckv_status ckv_select_decode_cached(const void *q, ckv_dtype dt, int P, int G, int d,
                                    const void *centroids_lp, const int32_t *n_clusters,
                                    int C_cap, const int32_t *offsets, const int32_t *perm,
                                    int perm_cap, int budget, int32_t *sel_idx, int32_t *sel_cnt,
                                    const void *K, const void *V, int64_t kv_problem_stride,
                                    int kv_rows, int sink, const int32_t *tail_begin,
                                    const int32_t *tail_end, int max_tail, float scale,
                                    float *out, int32_t *last_sel, int step, int R,
                                    int32_t *cache_stats, int32_t *miss_list, void *stream) {
    if (last_sel && (!cache_stats || R < 0))
        return fail(CKV_ERR_INVALID, "a cache needs cache_stats and R >= 0");
    if (!q || !centroids_lp || !n_clusters || !offsets || !perm || !sel_cnt || !K || !V ||
        !tail_begin || !tail_end || !out)
        return fail(CKV_ERR_INVALID, "null pointer argument");
    if (budget > 0 && !sel_idx) return fail(CKV_ERR_INVALID, "sel_idx is null");
    if (!valid_dtype(dt)) return fail(CKV_ERR_INVALID, "unknown dtype %d", (int)dt);
    if (d != D) return fail(CKV_ERR_INVALID, "d must be 128 (got %d)", d);
    if (P < 1 || P > 65535) return fail(CKV_ERR_INVALID, "bad P %d", P);
    if (G != 1 && G != 2 && G != 4)
        return fail(CKV_ERR_UNSUPPORTED, "fused step supports G = 1, 2, 4 (got %d)", G);
    if (C_cap < 1 || C_cap > CKV_MAX_CLUSTERS) return fail(CKV_ERR_INVALID, "bad C_cap %d", C_cap);
    if (perm_cap < 1) return fail(CKV_ERR_INVALID, "bad perm_cap %d", perm_cap);
    if (budget < 0 || max_tail < 0) return fail(CKV_ERR_INVALID, "negative budget or max_tail");
    if (kv_rows < 1 || kv_problem_stride < (int64_t)kv_rows * D)
        return fail(CKV_ERR_INVALID, "kv_problem_stride < kv_rows * d");
    if (sink < 0 || sink > kv_rows) return fail(CKV_ERR_INVALID, "bad sink %d", sink);
    if (!(scale > 0.f) || !isfinite(scale)) return fail(CKV_ERR_INVALID, "bad scale");
    const size_t esz = dt == CKV_BF16 ? 2 : 4;
    if (!aligned(q, 16) || !aligned(centroids_lp, 16) || !aligned(K, 16) || !aligned(V, 16) ||
        ((size_t)kv_problem_stride * esz) % 16)
        return fail(CKV_ERR_INVALID, "q, centroids_lp, K, V and the problem stride must be 16-byte aligned");
    const int64_t max_rows64 = (int64_t)sink + budget + max_tail;
    if (max_rows64 > (1 << 30)) return fail(CKV_ERR_INVALID, "too many attended rows");
    const int max_rows = max_rows64 < 1 ? 1 : (int)max_rows64;
    // CTAs per problem (nc) and rows in flight per half-warp (U): the largest
    // cluster size whose launch fits the GPU in one wave (all P clusters
    // resident at once), with U chosen so that a CTA's rows arrive in one
    // batch at the usual shapes. When not even one CTA per problem fits in a
    // wave (many problems), one CTA per problem with fewer rows in flight and
    // registers, so that more CTAs share an SM and their selection phases
    // overlap each other's gathers.
    int nc = 0, U = 0, chunk = 0;
    size_t smem = 0;
    sd_kernel kern = {nullptr, 0};
    cudaError_t e = cudaSuccess;
    for (int cand = sd::NC_MAX; cand >= 1; cand >>= 1) {
        const int ch = (max_rows + cand - 1) / cand;
        if (ch > sd::POS_MAX) break;
        const int u = (G == 4) ? 6 : (ch <= 16 * 4 ? 4 : 9);
        const sd_kernel k = sd_pick(dt, G, u);
        const size_t sm = sd::layout(C_cap, G, ch, cand).total;
        int fit = 0;
        if (sd_clusters_per_wave(k, cand, sm, &fit) != cudaSuccess) {
            cudaGetLastError();  // not a launchable shape: try fewer CTAs per problem
            fit = 0;
        }
        if (fit >= P || cand == 1) {
            nc = cand; chunk = ch; smem = sm; U = u; kern = k;
            if (fit < P && cand == 1) {  // more than one wave even at one CTA per problem
                U = (G == 4) ? 2 : 4;
                kern = sd_pick(dt, G, U);
            }
            break;
        }
    }
    if (nc == 0) {  // the rows do not fit one CTA: the smallest nc that holds them
        nc = (max_rows + sd::POS_MAX - 1) / sd::POS_MAX;
        nc = nc <= 2 ? nc : (nc <= 4 ? 4 : 8);
        chunk = (max_rows + nc - 1) / nc;
        if (chunk > sd::POS_MAX)
            return fail(CKV_ERR_UNSUPPORTED, "fused step supports up to %d attended rows per problem",
                        sd::NC_MAX * sd::POS_MAX);
        U = (G == 4) ? 6 : 9;
        kern = sd_pick(dt, G, U);
        smem = sd::layout(C_cap, G, chunk, nc).total;
    }
    sd::Args a;
    a.q = q;
    a.lp = centroids_lp;
    a.ncl = n_clusters;
    a.C_cap = C_cap;
    a.offsets = offsets;
    a.perm = perm;
    a.perm_cap = perm_cap;
    a.B = budget;
    a.K = K;
    a.V = V;
    a.kvs = kv_problem_stride;
    a.kv_rows = kv_rows;
    a.S = sink;
    a.tail_b = tail_begin;
    a.tail_e = tail_end;
    a.qscale = scale * 1.4426950408889634f;
    a.chunk = chunk;
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.out = out;
    a.last_sel = last_sel;
    a.step = step;
    a.R = R;
    a.cache_stats = cache_stats;
    a.miss_list = miss_list;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc, P, 1);
    cfg.blockDim = dim3(sd::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = S(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = CKV_SD_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = sd_optin(kern, smem);
    if (e == cudaSuccess) {
        void *args[] = {&a};
        e = cudaLaunchKernelExC(&cfg, kern.fn, args);
    }
    if (e != cudaSuccess) return fail(CKV_ERR_CUDA, "k_select_decode: %s", cudaGetErrorString(e));
    return launched("k_select_decode");
}

size_t ckv_decode_workspace_bytes(int P, int G, int d, int max_rows) {
    if (P < 1 || G < 1 || d != D) return 0;
    const size_t parts = decode_parts(P, G, max_rows);
    return align256(parts * D * sizeof(float)) + align256(parts * sizeof(float2));
}

ckv_status ckv_sparse_decode(const void *q, const void *K, const void *V, ckv_dtype dt, int P,
                             int G, int d, int64_t kv_problem_stride, int kv_rows, int sink,
                             const int32_t *tail_begin, const int32_t *tail_end, int max_tail,
                             const int32_t *sel_idx, const int32_t *sel_cnt, int budget,
                             float scale, float *out, void *workspace, size_t ws_bytes,
                             void *stream) {
    if (!q || !K || !V || !tail_begin || !tail_end || !sel_cnt || !out)
        return fail(CKV_ERR_INVALID, "null pointer argument");
    if (budget > 0 && !sel_idx) return fail(CKV_ERR_INVALID, "sel_idx is null");
    if (!valid_dtype(dt)) return fail(CKV_ERR_INVALID, "unknown dtype %d", (int)dt);
    if (d != D) return fail(CKV_ERR_INVALID, "d must be 128 (got %d)", d);
    if (P < 1 || P > 65535) return fail(CKV_ERR_INVALID, "bad P %d", P);
    if (G < 1 || G > 8 || (G & (G - 1)))
        return fail(CKV_ERR_INVALID, "G must be 1, 2, 4 or 8 (got %d)", G);
    if (kv_rows < 1 || kv_problem_stride < (int64_t)kv_rows * D)
        return fail(CKV_ERR_INVALID, "kv_problem_stride < kv_rows * d");
    if (sink < 0 || sink > kv_rows) return fail(CKV_ERR_INVALID, "bad sink %d", sink);
    if (budget < 0 || max_tail < 0) return fail(CKV_ERR_INVALID, "negative budget or max_tail");
    if (!(scale > 0.f) || !isfinite(scale)) return fail(CKV_ERR_INVALID, "bad scale");
    const size_t esz = dt == CKV_BF16 ? 2 : 4;
    if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) ||
        ((size_t)kv_problem_stride * esz) % 16)
        return fail(CKV_ERR_INVALID, "q, K, V and the problem stride must be 16-byte aligned");
    const int64_t max_rows64 = (int64_t)sink + budget + max_tail;
    if (max_rows64 > (1 << 30)) return fail(CKV_ERR_INVALID, "too many attended rows");
    const int max_rows = (int)max_rows64;
    if (!workspace || ws_bytes < ckv_decode_workspace_bytes(P, G, d, max_rows) ||
        !aligned(workspace, 256))
        return fail(CKV_ERR_INVALID, "workspace too small or not 256-byte aligned");
    int chunk, nsplit;
    decode_shape(P, max_rows, sm_count(), &chunk, &nsplit);
    const size_t parts = decode_parts(P, G, max_rows);
    float *part_o = reinterpret_cast<float *>(workspace);
    float2 *part_ml = reinterpret_cast<float2 *>(reinterpret_cast<char *>(workspace) +
                                                 align256(parts * D * sizeof(float)));
    const float qscale = scale * 1.4426950408889634f;  // exp(x) = exp2(x * log2(e))
    cudaStream_t st = S(stream);
    dim3 grid(nsplit, P);
#define CKV_DEC(T, GG)                                                                           \
    do {                                                                                         \
        k_decode_split<T, GG><<<grid, DEC_THREADS, 0, st>>>(                                     \
            (const T *)q, (const T *)K, (const T *)V, kv_problem_stride, kv_rows, sink,          \
            tail_begin, tail_end, sel_idx, sel_cnt, budget, qscale, chunk, nsplit, part_o,       \
            part_ml);                                                                            \
        k_decode_combine<GG><<<P, D, 0, st>>>(part_o, part_ml, nsplit, out);                     \
    } while (0)
#define CKV_DEC_G(T)                     \
    switch (G) {                         \
        case 1: CKV_DEC(T, 1); break;    \
        case 2: CKV_DEC(T, 2); break;    \
        case 4: CKV_DEC(T, 4); break;    \
        default: CKV_DEC(T, 8); break;   \
    }
    if (dt == CKV_BF16) {
        CKV_DEC_G(bf16)
    } else {
        CKV_DEC_G(float)
    }
#undef CKV_DEC_G
#undef CKV_DEC
    return launched("k_decode");
}

ckv_status ckv_append(void *K, void *V, ckv_dtype dt, int P, int d, int64_t kv_problem_stride,
                      int kv_rows, const void *new_k, const void *new_v, int32_t *tail_end,
                      void *stream) {
    if (!K || !V || !new_k || !new_v || !tail_end)
        return fail(CKV_ERR_INVALID, "null pointer argument");
    if (!valid_dtype(dt)) return fail(CKV_ERR_INVALID, "unknown dtype %d", (int)dt);
    if (d != D) return fail(CKV_ERR_INVALID, "d must be 128 (got %d)", d);
    if (P < 1 || P > 65535) return fail(CKV_ERR_INVALID, "bad P %d", P);
    if (kv_rows < 1 || kv_problem_stride < (int64_t)kv_rows * D)
        return fail(CKV_ERR_INVALID, "kv_problem_stride < kv_rows * d");
    const size_t esz = dt == CKV_BF16 ? 2 : 4;
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(new_k, 16) || !aligned(new_v, 16) ||
        ((size_t)kv_problem_stride * esz) % 16)
        return fail(CKV_ERR_INVALID, "buffers must be 16-byte aligned");
    cudaStream_t st = S(stream);
    if (dt == CKV_BF16)
        k_append<bf16><<<P, 32, 0, st>>>((bf16 *)K, (bf16 *)V, kv_problem_stride, kv_rows,
                                         (const bf16 *)new_k, (const bf16 *)new_v, tail_end);
    else
        k_append<float><<<P, 32, 0, st>>>((float *)K, (float *)V, kv_problem_stride, kv_rows,
                                          (const float *)new_k, (const float *)new_v, tail_end);
    return launched("k_append");
}

ckv_status ckv_selftest_timeout(unsigned int limit_us, void *stream) {
    if (limit_us > 1000000u) return fail(CKV_ERR_INVALID, "limit_us must be <= 1000000");
    k_selftest_wait<<<1, 32, 0, S(stream)>>>((unsigned long long)limit_us * 1000ull);
    return launched("k_selftest_wait");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free sparse decode: the split-K partials live in a fixed array
// inside the library instead of a caller workspace. See ckv.h
// (ckv_sparse_decode_noalloc) for who needs this and its limits.
// ---------------------------------------------------------------------------

// One copy per device that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_decode_scratch[CKV_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mu;
void *g_noalloc_addr[MAX_DEVICES] = {nullptr};

// Device address of the fixed scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
ckv_status noalloc_scratch(void **addr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(CKV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= MAX_DEVICES) return fail(CKV_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_decode_scratch);
        if (e != cudaSuccess || !ptr)
            return fail(CKV_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        g_noalloc_addr[dev] = ptr;
    }
    *addr = g_noalloc_addr[dev];
    return CKV_OK;
}

}  // namespace

extern "C" size_t ckv_sparse_decode_noalloc_scratch_bytes(int P, int G, int d, int max_rows) {
    if (P < 1 || G < 1 || d != D) return 0;
    int chunk, nsplit;
    decode_shape(P, max_rows, sm_count(), &chunk, &nsplit);
    const size_t parts = (size_t)P * nsplit * G;
    return align256(parts * D * sizeof(float)) + align256(parts * sizeof(float2));
}

extern "C" ckv_status ckv_sparse_decode_noalloc(const void *q, const void *K, const void *V,
                                                ckv_dtype dt, int P, int G, int d,
                                                int64_t kv_problem_stride, int kv_rows, int sink,
                                                const int32_t *tail_begin,
                                                const int32_t *tail_end, int max_tail,
                                                const int32_t *sel_idx, const int32_t *sel_cnt,
                                                int budget, float scale, float *out,
                                                void *stream) {
    if (!q || !K || !V || !tail_begin || !tail_end || !sel_cnt || !out)
        return fail(CKV_ERR_INVALID, "null pointer argument");
    if (budget > 0 && !sel_idx) return fail(CKV_ERR_INVALID, "sel_idx is null");
    if (!valid_dtype(dt)) return fail(CKV_ERR_INVALID, "unknown dtype %d", (int)dt);
    if (d != D) return fail(CKV_ERR_INVALID, "d must be 128 (got %d)", d);
    if (P < 1 || P > 65535) return fail(CKV_ERR_INVALID, "bad P %d", P);
    if (G < 1 || G > 8 || (G & (G - 1)))
        return fail(CKV_ERR_INVALID, "G must be 1, 2, 4 or 8 (got %d)", G);
    if (kv_rows < 1 || kv_problem_stride < (int64_t)kv_rows * D)
        return fail(CKV_ERR_INVALID, "kv_problem_stride < kv_rows * d");
    if (sink < 0 || sink > kv_rows) return fail(CKV_ERR_INVALID, "bad sink %d", sink);
    if (budget < 0 || max_tail < 0) return fail(CKV_ERR_INVALID, "negative budget or max_tail");
    if (!(scale > 0.f) || !isfinite(scale)) return fail(CKV_ERR_INVALID, "bad scale");
    const size_t esz = dt == CKV_BF16 ? 2 : 4;
    if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) ||
        ((size_t)kv_problem_stride * esz) % 16)
        return fail(CKV_ERR_INVALID, "q, K, V and the problem stride must be 16-byte aligned");
    const int64_t max_rows64 = (int64_t)sink + budget + max_tail;
    if (max_rows64 > (1 << 30)) return fail(CKV_ERR_INVALID, "too many attended rows");
    const int max_rows = (int)max_rows64;
    int chunk, nsplit;
    decode_shape(P, max_rows, sm_count(), &chunk, &nsplit);
    const size_t parts = (size_t)P * nsplit * G;
    const size_t o_bytes = align256(parts * D * sizeof(float));
    const size_t need = o_bytes + align256(parts * sizeof(float2));
    if (need > (size_t)CKV_NOALLOC_SCRATCH_BYTES)
        return fail(CKV_ERR_INVALID,
                    "this decode needs %zu bytes of scratch, more than the fixed %zu bytes of "
                    "ckv_sparse_decode_noalloc; use ckv_sparse_decode with a workspace",
                    need, (size_t)CKV_NOALLOC_SCRATCH_BYTES);
    void *scratch = nullptr;
    ckv_status s = noalloc_scratch(&scratch);
    if (s) return s;
    float *part_o = reinterpret_cast<float *>(scratch);
    float2 *part_ml = reinterpret_cast<float2 *>(reinterpret_cast<char *>(scratch) + o_bytes);
    const float qscale = scale * 1.4426950408889634f;
    cudaStream_t st = S(stream);
    dim3 grid(nsplit, P);
#define CKV_DEC_NA(T, GG)                                                                        \
    do {                                                                                         \
        k_decode_split<T, GG><<<grid, DEC_THREADS, 0, st>>>(                                     \
            (const T *)q, (const T *)K, (const T *)V, kv_problem_stride, kv_rows, sink,          \
            tail_begin, tail_end, sel_idx, sel_cnt, budget, qscale, chunk, nsplit, part_o,       \
            part_ml);                                                                            \
        k_decode_combine<GG><<<P, D, 0, st>>>(part_o, part_ml, nsplit, out);                     \
    } while (0)
#define CKV_DEC_NA_G(T)                     \
    switch (G) {                            \
        case 1: CKV_DEC_NA(T, 1); break;    \
        case 2: CKV_DEC_NA(T, 2); break;    \
        case 4: CKV_DEC_NA(T, 4); break;    \
        default: CKV_DEC_NA(T, 8); break;   \
    }
    if (dt == CKV_BF16) {
        CKV_DEC_NA_G(bf16)
    } else {
        CKV_DEC_NA_G(float)
    }
#undef CKV_DEC_NA_G
#undef CKV_DEC_NA
    return launched("k_decode (noalloc)");
}
