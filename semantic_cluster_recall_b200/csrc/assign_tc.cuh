// a2 assignment for bf16 keys on the sm_100a tensor cores.
//
// labels[i] = argmax_c k_i . hat_c: the key-centroid similarity of cosine
// k-means ("III.B Clustering in the Semantic Space" of "ClusterKV:
// Manipulating LLM KV Cache in Semantic Space for Recallable Compression",
// arXiv 2412.03213v2) is a [n x 128] x [128 x C] contraction per problem,
// followed by a row argmax. The paper runs it with library kernels; here it
// is one persistent kernel:
//
//   warp 8 (1 lane)   TMA producer: 128-key tiles (two 64-column halves,
//                     128-byte swizzle) into a ring of KST stages, and the
//                     centroid chunks (resident per problem when they fit in
//                     shared memory, otherwise streamed through 2 slots)
//   warp 9 (1 lane)   MMA issuer: tcgen05.mma kind::f16, M = 128 keys,
//                     N = one centroid chunk (<= 256), K = 128 in 8 steps,
//                     bf16 x bf16 -> fp32 into one of two TMEM accumulators
//   warps 0-7         epilogue: warps w and w+4 share TMEM lane quarter w,
//                     so each key row (TMEM lane) has two threads, each
//                     reading half of the chunk's columns with tcgen05.ld and
//                     keeping four independent running (max, argmax) chains
//                     (instruction-level parallelism); the chains and the two
//                     halves are merged per tile with ties to the lowest
//                     centroid index, and the label is written
//
// Two 256-column TMEM accumulators let the MMA of the next chunk overlap the
// epilogue of the current one. Tiles are split into contiguous ranges, one
// per CTA (one CTA per SM), so a CTA reloads resident centroids only when its
// range crosses into the next problem. Every mbarrier wait is bounded: on
// timeout the kernel sets CKV_DEVERR_TIMEOUT, stops all roles, waits for its
// own copies and MMAs, frees TMEM and returns.
#pragma once

#include <cuda.h>  // CUtensorMap and its enums (the driver entry point is looked up at run time)

#include "common.cuh"

namespace ckv {
namespace tc {

constexpr int BM = 128;                          // key rows per tile (MMA M)
constexpr int KEY_HALF_BYTES = BM * 128;         // 128 rows x 64 bf16
constexpr int KEY_STAGE_BYTES = 2 * KEY_HALF_BYTES;
constexpr int ACC_COLS = 256;                    // TMEM columns per accumulator
constexpr int TMEM_COLS = 512;
#ifndef CKV_TC_EPI_PARTS
#define CKV_TC_EPI_PARTS 4      // epilogue threads per key row
#endif
#ifndef CKV_TC_CHAINS
#define CKV_TC_CHAINS 4         // independent (max, argmax) chains per thread
#endif
#ifndef CKV_TC_SUSPEND_NS
#define CKV_TC_SUSPEND_NS 0     // mbarrier try_wait suspend-time hint (0: none)
#endif
constexpr int EPI_PARTS = CKV_TC_EPI_PARTS;
constexpr int CHAINS = CKV_TC_CHAINS;
constexpr int EPI_WARPS = 4 * EPI_PARTS;         // EPI_PARTS warps per TMEM lane quarter
constexpr int MAXG = (16 + EPI_PARTS - 1) / EPI_PARTS;  // 16-column groups per part (chunk <= 256)
constexpr int PRODUCER_WARP = EPI_WARPS;
constexpr int MMA_WARP = EPI_WARPS + 1;
constexpr int NTHREADS = (EPI_WARPS + 2) * 32;
constexpr int NBAR = 32;                         // mbarrier slots reserved
constexpr int EPI_SMEM = 2 * (EPI_PARTS - 1) * BM * 8;  // partial results, 2 buffers
constexpr int SMEM_OPTIN_MAX = 232448;           // 227 KB per CTA
constexpr int SMEM_MIN = 120 * 1024;             // keeps one CTA per SM (TMEM is not shared)
constexpr unsigned long long TIMEOUT_NS = 2000000000ull;
constexpr unsigned long long DRAIN_NS = 200000000ull;

struct Args {
    int n, tok_begin, C, cbase, perm_base, perm_cap;
    int tpp;             // tiles per problem
    int total;           // tiles over all problems
    int nch, ch_rows;    // centroid chunks and rows per chunk (multiple of 16, <= 256)
    int32_t *labels;
    const float *bias;   // problem p's cluster c at bias[p * bstride + c] (L2), or null
    int bstride;
    int bias_vec4;       // bias rows start 16-byte aligned
};

// ---- PTX wrappers ------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
#if CKV_TC_SUSPEND_NS > 0
    // the thread may sleep until the phase completes (or the hint elapses)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"((uint32_t)CKV_TC_SUSPEND_NS)
        : "memory");
#else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
#endif
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of the given parity; false if another role aborted or
// the wait timed out (then this role raises the abort flag and the error bit).
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > TIMEOUT_NS) {
            *abort_flag = 1;
            dev_flag(CKV_DEVERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag (used to drain own async work).
__device__ __noinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_ns();
    while (!mbar_try(bar, parity)) {
        if (global_ns() - t0 > DRAIN_NS) {
            dev_flag(CKV_DEVERR_TIMEOUT);
            return;
        }
    }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane; the values are
// valid only after tmem_wait_ld().
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, float (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
          "=f"(v[7]), "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]),
          "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), sm_100
// descriptor version 1. The leading byte offset is unused in this layout.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: D fp32, A and B bf16, both K-major, N and M.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ---- the kernel ----------------------------------------------------------------

// 16 consecutive bias values (L1-cached; every lane of a warp reads the same ones)
__device__ __forceinline__ void load_bias16(const float *b, int vec4, float (&o)[16]) {
    if (vec4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 t = __ldg(reinterpret_cast<const float4 *>(b) + q);
            o[4 * q] = t.x;
            o[4 * q + 1] = t.y;
            o[4 * q + 2] = t.z;
            o[4 * q + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = __ldg(b + i);
    }
}

// BIASM: 0 no bias; 1 bias read from global memory (L1); 2 bias cached per
// epilogue warp in shared memory
template <bool RESIDENT, int KST, int BIASM>
__global__ void __launch_bounds__(NTHREADS, 1)
k_assign_tc(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmc,
            const Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nslot = RESIDENT ? a.nch : 2;
    const uint32_t ch_half = (uint32_t)a.ch_rows * 128u;
    const uint32_t ch_bytes = 2u * ch_half;
    unsigned char *keys_s = sm;
    unsigned char *cent_s = sm + KST * KEY_STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(cent_s + (size_t)nslot * ch_bytes);
    // barrier slots
    uint64_t *keys_full = bars;                // [KST]
    uint64_t *keys_empty = bars + KST;         // [KST]
    uint64_t *cent_full = bars + 2 * KST;      // [2]
    uint64_t *cent_empty = bars + 2 * KST + 2; // [2]
    uint64_t *acc_full = bars + 2 * KST + 4;   // [2]
    uint64_t *acc_empty = bars + 2 * KST + 6;  // [2]
    uint64_t *drain = bars + 2 * KST + 8;      // [1]
    uint64_t *red_full = bars + 2 * KST + 9;   // [2] other parts' partials are written
    uint64_t *red_empty = bars + 2 * KST + 11; // [2] part 0 has read them
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + NBAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    float *red_v = reinterpret_cast<float *>(bars + NBAR + 1);           // [2][PARTS-1][BM]
    int *red_i = reinterpret_cast<int *>(red_v + 2 * (EPI_PARTS - 1) * BM);
    // per epilogue warp: the bias of its columns of every chunk, [nch][MAXG * 16]
    float *wbias_all = reinterpret_cast<float *>(
        (reinterpret_cast<uintptr_t>(red_i + 2 * (EPI_PARTS - 1) * BM) + 15) & ~uintptr_t(15));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < KST; ++s) {
            mbar_init(smem_u32(&keys_full[s]), 1);
            mbar_init(smem_u32(&keys_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&cent_full[s]), 1);
            mbar_init(smem_u32(&cent_empty[s]), 1);
            mbar_init(smem_u32(&acc_full[s]), 1);
            mbar_init(smem_u32(&acc_empty[s]), EPI_WARPS * 32);
            mbar_init(smem_u32(&red_full[s]), (EPI_PARTS - 1) * 4 * 32 > 0 ? (EPI_PARTS - 1) * 4 * 32 : 1);
            mbar_init(smem_u32(&red_empty[s]), 4 * 32);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_holder)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int t_begin = (int)((long long)a.total * blockIdx.x / gridDim.x);
    const int t_end = (int)((long long)a.total * (blockIdx.x + 1) / gridDim.x);

    if (warp == PRODUCER_WARP) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int last_r[KST];
            for (int s = 0; s < KST; ++s) last_r[s] = -1;
            int last_c[2] = {-1, -1};
            int it = 0, pl = 0, g = 0, cur = -1;
            bool ok = true;
            for (int tile = t_begin; tile < t_end && ok; ++tile) {
                const int p = tile / a.tpp, t = tile - p * a.tpp;
                if (RESIDENT && p != cur) {
                    ok = mbar_wait(smem_u32(&cent_empty[0]), (pl & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    const uint32_t fb = smem_u32(&cent_full[0]);
                    mbar_expect_tx(fb, (uint32_t)a.nch * ch_bytes);
                    for (int j = 0; j < a.nch; ++j)
                        for (int h = 0; h < 2; ++h)
                            tma_load_3d(smem_u32(cent_s + (size_t)j * ch_bytes + h * ch_half), &tmc,
                                        fb, h * 64, a.cbase + j * a.ch_rows, p);
                    last_c[0] = pl;
                    ++pl;
                    cur = p;
                }
                const int s = it % KST, r = it / KST;
                ok = mbar_wait(smem_u32(&keys_empty[s]), (r & 1) ^ 1, abort_flag);
                if (!ok) break;
                const uint32_t kb = smem_u32(&keys_full[s]);
                mbar_expect_tx(kb, KEY_STAGE_BYTES);
                for (int h = 0; h < 2; ++h)
                    tma_load_3d(smem_u32(keys_s + s * KEY_STAGE_BYTES + h * KEY_HALF_BYTES), &tmk,
                                kb, h * 64, a.tok_begin + t * BM, p);
                last_r[s] = r;
                ++it;
                if (!RESIDENT) {
                    for (int j = 0; j < a.nch; ++j, ++g) {
                        const int sl = g & 1, rr = g >> 1;
                        ok = mbar_wait(smem_u32(&cent_empty[sl]), (rr & 1) ^ 1, abort_flag);
                        if (!ok) break;
                        const uint32_t fb = smem_u32(&cent_full[sl]);
                        mbar_expect_tx(fb, ch_bytes);
                        for (int h = 0; h < 2; ++h)
                            tma_load_3d(smem_u32(cent_s + (size_t)sl * ch_bytes + h * ch_half),
                                        &tmc, fb, h * 64, a.cbase + j * a.ch_rows, p);
                        last_c[sl] = rr;
                    }
                }
            }
            // every copy this thread issued has landed before the CTA can exit
            for (int s = 0; s < KST; ++s)
                if (last_r[s] >= 0) mbar_drain(smem_u32(&keys_full[s]), last_r[s] & 1);
            for (int s = 0; s < 2; ++s)
                if (last_c[s] >= 0) mbar_drain(smem_u32(&cent_full[s]), last_c[s] & 1);
        }
    } else if (warp == MMA_WARP) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, a.ch_rows);
            int it = 0, pl = 0, g = 0, acc = 0, cur = -1;
            bool ok = true, issued = false;
            for (int tile = t_begin; tile < t_end && ok; ++tile) {
                const int p = tile / a.tpp;
                if (RESIDENT && p != cur) {
                    ok = mbar_wait(smem_u32(&cent_full[0]), pl & 1, abort_flag);
                    if (!ok) break;
                    ++pl;
                    cur = p;
                }
                const int s = it % KST, r = it / KST;
                ok = mbar_wait(smem_u32(&keys_full[s]), r & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t ka = smem_u32(keys_s + s * KEY_STAGE_BYTES);
                for (int j = 0; j < a.nch; ++j) {
                    uint32_t ca;
                    int sl = 0;
                    if (RESIDENT) {
                        ca = smem_u32(cent_s + (size_t)j * ch_bytes);
                    } else {
                        sl = g & 1;
                        ok = mbar_wait(smem_u32(&cent_full[sl]), (g >> 1) & 1, abort_flag);
                        if (!ok) break;
                        ca = smem_u32(cent_s + (size_t)sl * ch_bytes);
                    }
                    const int buf = acc & 1;
                    ok = mbar_wait(smem_u32(&acc_empty[buf]), ((acc >> 1) & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(buf * ACC_COLS);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t koff = (uint32_t)(k >> 2) * KEY_HALF_BYTES + (k & 3) * 32;
                        const uint32_t coff = (uint32_t)(k >> 2) * ch_half + (k & 3) * 32;
                        tc_mma(d, sdesc(ka + koff), sdesc(ca + coff), idesc, k > 0 ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit(smem_u32(&acc_full[buf]));
                    if (!RESIDENT) {
                        tc_commit(smem_u32(&cent_empty[sl]));
                        ++g;
                    }
                    ++acc;
                }
                if (!ok) break;
                tc_commit(smem_u32(&keys_empty[s]));
                ++it;
                if (RESIDENT) {
                    const int nt = tile + 1;
                    if (nt >= t_end || nt / a.tpp != p) tc_commit(smem_u32(&cent_empty[0]));
                }
            }
            if (issued) {  // all MMAs issued by this thread have completed
                tc_commit(smem_u32(drain));
                mbar_drain(smem_u32(drain), 0);
            }
        }
    } else {
        // ------------- epilogue: EPI_PARTS threads per key row (one per warp part) -------------
        const int quarter = warp & 3, part = warp >> 2;
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const int ngroups = a.ch_rows / 16;               // 16-column groups per chunk
        const int gper = (ngroups + EPI_PARTS - 1) / EPI_PARTS;  // <= MAXG
        const int g_lo = min(ngroups, part * gper), g_hi = min(ngroups, g_lo + gper);
        int acc = 0, nt = 0;
        bool ok = true;
        float *wbias = wbias_all + (size_t)warp * a.nch * (MAXG * 16);
        int bias_p = -1;  // problem whose bias this warp holds
        for (int tile = t_begin; tile < t_end && ok; ++tile, ++nt) {
            const int p = tile / a.tpp, t = tile - p * a.tpp;
            const float *bp = BIASM ? a.bias + (size_t)p * a.bstride : nullptr;
            if (BIASM == 2 && p != bias_p) {  // this warp's columns, every chunk
                __syncwarp();
                for (int e = lane; e < a.nch * MAXG * 16; e += 32) {
                    const int j = e / (MAXG * 16), r = e - j * (MAXG * 16);
                    const int g = g_lo + r / 16, col = g * 16 + (r & 15);
                    const int cc = j * a.ch_rows + col;
                    wbias[e] = (g < g_hi && cc < a.C) ? __ldg(bp + cc) : 0.f;
                }
                __syncwarp();
                bias_p = p;
            }
            float best[CHAINS];
            int bidx[CHAINS];
#pragma unroll
            for (int k = 0; k < CHAINS; ++k) {
                best[k] = -INFINITY;
                bidx[k] = 0x7fffffff;
            }
            for (int j = 0; j < a.nch; ++j) {
                const int buf = acc & 1;
                ok = mbar_wait(smem_u32(&acc_full[buf]), (acc >> 1) & 1, abort_flag);
                ok = __all_sync(FULL, ok);  // tcgen05.ld below needs the whole warp
                if (!ok) break;
                tc_fence_after();
                const int c0 = j * a.ch_rows;
                const int lim = min(a.ch_rows, a.C - c0);  // valid columns of this chunk
                const uint32_t col_base = lane_base + (uint32_t)(buf * ACC_COLS);
                // copy this thread's slice of the chunk to registers and hand the
                // accumulator back to the MMA warp at once; the argmax runs after
                float v[MAXG][16];
#pragma unroll
                for (int u = 0; u < MAXG; ++u)
                    if (g_lo + u < g_hi) tmem_ld16_nowait(col_base + (g_lo + u) * 16, v[u]);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(smem_u32(&acc_empty[buf]));
#pragma unroll
                for (int u = 0; u < MAXG; ++u) {
                    const int gc = (g_lo + u) * 16;
                    if (g_lo + u < g_hi && gc < lim) {
                        // L2: scores minus half the centroid's squared norm
                        if (BIASM == 2) {  // from this warp's cached copy, 4 at a time
                            const float4 *wb = reinterpret_cast<const float4 *>(
                                wbias + j * (MAXG * 16) + u * 16);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 b4 = wb[q];
                                v[u][4 * q] -= b4.x;
                                v[u][4 * q + 1] -= b4.y;
                                v[u][4 * q + 2] -= b4.z;
                                v[u][4 * q + 3] -= b4.w;
                            }
                        }
                        float bcol[16];
                        if (BIASM == 1) {
                            if (gc + 16 <= lim) {
                                load_bias16(bp + c0 + gc, a.bias_vec4, bcol);
                            } else {
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    bcol[i] = gc + i < lim ? __ldg(bp + c0 + gc + i) : 0.f;
                            }
                        }
                        if (gc + 16 <= lim) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int k = (u * 16 + i) % CHAINS;
                                const float sc = BIASM == 1 ? v[u][i] - bcol[i] : v[u][i];
                                const bool take = sc > best[k];
                                best[k] = take ? sc : best[k];
                                bidx[k] = take ? c0 + gc + i : bidx[k];
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int k = (u * 16 + i) % CHAINS;
                                const float sc = BIASM == 1 ? v[u][i] - bcol[i] : v[u][i];
                                const bool take = (gc + i < lim) && sc > best[k];
                                best[k] = take ? sc : best[k];
                                bidx[k] = take ? c0 + gc + i : bidx[k];
                            }
                        }
                    }
                }
                ++acc;
            }
            if (!ok) break;
            // merge the chains: larger value, then lower index
            float bv = best[0];
            int bi = bidx[0];
#pragma unroll
            for (int k = 1; k < CHAINS; ++k)
                if (best[k] > bv || (best[k] == bv && bidx[k] < bi)) {
                    bv = best[k];
                    bi = bidx[k];
                }
            // merge the parts of the row (bounded mbarrier handshake)
            const int rb = nt & 1;
            if (part > 0) {
                ok = mbar_wait(smem_u32(&red_empty[rb]), ((nt >> 1) & 1) ^ 1, abort_flag);
                if (!ok) break;
                const int slot = (rb * (EPI_PARTS - 1) + part - 1) * BM + row_in_tile;
                red_v[slot] = bv;
                red_i[slot] = bi;
                mbar_arrive(smem_u32(&red_full[rb]));
            } else {
                if (EPI_PARTS > 1) {
                    ok = mbar_wait(smem_u32(&red_full[rb]), (nt >> 1) & 1, abort_flag);
                    if (!ok) break;
#pragma unroll
                    for (int q = 1; q < EPI_PARTS; ++q) {
                        const int slot = (rb * (EPI_PARTS - 1) + q - 1) * BM + row_in_tile;
                        const float ov = red_v[slot];
                        const int oi = red_i[slot];
                        if (ov > bv || (ov == bv && oi < bi)) {
                            bv = ov;
                            bi = oi;
                        }
                    }
                    mbar_arrive(smem_u32(&red_empty[rb]));
                }
                const int row = t * BM + row_in_tile;
                if (bi == 0x7fffffff) bi = 0;  // no valid column (cannot happen for C >= 1)
                if (row < a.n)
                    a.labels[(size_t)p * a.perm_cap + a.perm_base + row] = a.cbase + bi;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace tc

// ---- host side ---------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        tried = true;
    }
    return fn;
}

// 3-D bf16 tensor map [P][rows][128] with a {64, box_rows, 1} box, 128-byte swizzle.
inline bool make_map_bf16(CUtensorMap *m, const void *base, int P, long long rows,
                          long long problem_stride_elems, int box_rows) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)P};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)problem_stride_elems * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TcPlan {
    bool resident;
    int nch, ch_rows;
    size_t smem;
};

inline size_t tc_smem_bytes(bool resident, int kst, int nch, int ch_rows) {
    const size_t slots = resident ? (size_t)nch : 2;
    size_t s = 1024 /* alignment slack */ + (size_t)kst * tc::KEY_STAGE_BYTES +
               slots * 2 * (size_t)ch_rows * 128 + tc::NBAR * 8 + 8 /* TMEM address, flag */ +
               tc::EPI_SMEM;
    return s < (size_t)tc::SMEM_MIN ? (size_t)tc::SMEM_MIN : s;
}

inline TcPlan tc_plan(int C) {
    TcPlan pl;
    pl.nch = (C + 255) / 256;
    const int per = (C + pl.nch - 1) / pl.nch;
    pl.ch_rows = ((per + 15) / 16) * 16;
    pl.resident = tc_smem_bytes(true, 3, pl.nch, pl.ch_rows) <= (size_t)tc::SMEM_OPTIN_MAX;
    pl.smem = pl.resident ? tc_smem_bytes(true, 3, pl.nch, pl.ch_rows)
                          : tc_smem_bytes(false, 2, pl.nch, pl.ch_rows);
    return pl;
}

inline ckv_status launch_assign_bf16(const bf16 *keys, int P, int64_t pstride, int tok_begin,
                                     int n, const bf16 *hat, int C, int cbase, int C_cap,
                                     int32_t *labels, int perm_base, int perm_cap, int sms,
                                     const float *bias, int bstride, cudaStream_t st) {
    CUtensorMap mk, mc;
    const TcPlan pl = tc_plan(C);
    if (!make_map_bf16(&mk, keys, P, pstride / 128, pstride, tc::BM)) return CKV_ERR_CUDA;
    if (!make_map_bf16(&mc, hat, P, C_cap, (long long)C_cap * 128, pl.ch_rows))
        return CKV_ERR_CUDA;
    tc::Args a;
    a.n = n;
    a.tok_begin = tok_begin;
    a.C = C;
    a.cbase = cbase;
    a.perm_base = perm_base;
    a.perm_cap = perm_cap;
    a.tpp = (n + tc::BM - 1) / tc::BM;
    a.total = P * a.tpp;
    a.nch = pl.nch;
    a.ch_rows = pl.ch_rows;
    a.labels = labels;
    a.bias = bias;
    a.bstride = bstride;
    a.bias_vec4 = (bstride % 4 == 0 && ((uintptr_t)bias & 15) == 0) ? 1 : 0;
    // L2: cache the bias per epilogue warp when shared memory allows
    size_t smem = pl.smem;
    const size_t bias_bytes = (size_t)tc::EPI_WARPS * pl.nch * tc::MAXG * 16 * sizeof(float) + 16;
    const bool bias_smem = bias && pl.smem + bias_bytes <= (size_t)tc::SMEM_OPTIN_MAX;
    if (bias_smem) smem += bias_bytes;
    const int grid = a.total < sms ? a.total : sms;
    cudaError_t e;
#define CKV_TC_LAUNCH(RES, KS, BI)                                                        \
    do {                                                                                  \
        e = cudaFuncSetAttribute(tc::k_assign_tc<RES, KS, BI>,                            \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);    \
        if (e != cudaSuccess) return CKV_ERR_CUDA;                                        \
        tc::k_assign_tc<RES, KS, BI><<<grid, tc::NTHREADS, smem, st>>>(mk, mc, a);        \
    } while (0)
    if (pl.resident) {
        if (bias_smem) CKV_TC_LAUNCH(true, 3, 2);
        else if (bias) CKV_TC_LAUNCH(true, 3, 1);
        else CKV_TC_LAUNCH(true, 3, 0);
    } else {
        if (bias_smem) CKV_TC_LAUNCH(false, 2, 2);
        else if (bias) CKV_TC_LAUNCH(false, 2, 1);
        else CKV_TC_LAUNCH(false, 2, 0);
    }
#undef CKV_TC_LAUNCH
    return cudaGetLastError() == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

}  // namespace ckv
