// bf16 assignment dispatch.
#pragma once

#include "cluster_kernels.cuh"

namespace ckv {

inline ckv_status launch_assign_bf16(const bf16 *keys, int P, int64_t pstride, int tok_begin,
                                     int n, const bf16 *hat, int C, int cbase, int C_cap,
                                     int32_t *labels, int perm_base, int perm_cap,
                                     cudaStream_t st) {
    if (cudaFuncSetAttribute(k_assign_simt<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AS_SMEM) != cudaSuccess)
        return CKV_ERR_CUDA;
    dim3 grid((n + AS_TILE - 1) / AS_TILE, P);
    k_assign_simt<bf16><<<grid, 256, AS_SMEM, st>>>(keys, pstride, tok_begin, n, hat, C, cbase,
                                                    C_cap, labels, perm_base, perm_cap);
    return cudaGetLastError() == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

}  // namespace ckv
