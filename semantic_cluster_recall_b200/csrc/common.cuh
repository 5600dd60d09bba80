// Shared device helpers for libckv (sm_100a). Single translation unit: ckv.cu
// includes every kernel header after this one.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ckv.h"

namespace ckv {

constexpr int D = 128;            // head dimension (the only one supported)
constexpr unsigned FULL = 0xffffffffu;

typedef __nv_bfloat16 bf16;

// Device error word: out-of-range data is skipped and reported here instead
// of being dereferenced.
__device__ unsigned int g_devflags;

__device__ __forceinline__ void dev_flag(unsigned bits) { atomicOr(&g_devflags, bits); }

// ---- 4-element loads / stores (one lane owns 4 consecutive channels) ------

__device__ __forceinline__ float4 load4(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}

__device__ __forceinline__ float4 load4(const bf16 *p) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    float4 f;
    f.x = __uint_as_float(u.x << 16);
    f.y = __uint_as_float(u.x & 0xffff0000u);
    f.z = __uint_as_float(u.y << 16);
    f.w = __uint_as_float(u.y & 0xffff0000u);
    return f;
}

__device__ __forceinline__ void store4(float *p, float4 v) {
    *reinterpret_cast<float4 *>(p) = v;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t a = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo));
    uint32_t b = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return a | (b << 16);
}

__device__ __forceinline__ void store4(bf16 *p, float4 v) {
    uint2 u;
    u.x = pack_bf16x2(v.x, v.y);
    u.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2 *>(p) = u;
}

// ---- 8-element loads (one lane owns 8 consecutive channels) ---------------

__device__ __forceinline__ void unpack8(uint4 u, float (&f)[8]) {
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xffff0000u);
    f[4] = __uint_as_float(u.z << 16);
    f[5] = __uint_as_float(u.z & 0xffff0000u);
    f[6] = __uint_as_float(u.w << 16);
    f[7] = __uint_as_float(u.w & 0xffff0000u);
}

template <typename T>
struct Row8;  // raw registers holding 8 elements of one row

template <>
struct Row8<bf16> {
    uint4 u;
    __device__ __forceinline__ void load(const bf16 *p) {
        u = __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ void load_shared(const bf16 *p) {
        u = *reinterpret_cast<const uint4 *>(p);
    }
    __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void to_float(float (&f)[8]) const { unpack8(u, f); }
};

template <>
struct Row8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = __ldg(reinterpret_cast<const float4 *>(p));
        b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    }
    __device__ __forceinline__ void load_shared(const float *p) {
        a = reinterpret_cast<const float4 *>(p)[0];
        b = reinterpret_cast<const float4 *>(p)[1];
    }
    __device__ __forceinline__ void zero() {
        a = make_float4(0.f, 0.f, 0.f, 0.f);
        b = a;
    }
    __device__ __forceinline__ void to_float(float (&f)[8]) const {
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace ckv
