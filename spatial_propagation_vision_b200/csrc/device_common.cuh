// Device helpers shared by the Prop2D kernels: element conversion, async
// global->shared copies and the fused row-stochastic normalisation.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace gspn {

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Two fp32 values rounded to bf16 (round to nearest even) in one 32-bit word:
// x in the low half, y in the high half.
__device__ __forceinline__ uint32_t pack_bf16x2(float2 v) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(v.x, v.y);
    return *reinterpret_cast<const uint32_t *>(&b);
}

// ---------------------------------------------------------------------------
// hardware approximations: 2^x and 1/x (flush-to-zero), byte permutation
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Byte permutation of (x, 0): bf16 half of a word -> fp32 bits.
__device__ __forceinline__ uint32_t prmt0(uint32_t x, uint32_t sel) {
    uint32_t y;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(y) : "r"(x), "r"(sel));
    return y;
}

// ---------------------------------------------------------------------------
// async copies (cp.async, sm_80+): global -> shared, completion tracked per
// thread with commit/wait groups.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// L2 prefetch through the TMA engine
// ---------------------------------------------------------------------------
// Bulk prefetch of [src, src + bytes) into L2 (TMA engine); src 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// ---------------------------------------------------------------------------
// Plain normalisation (the general kernel's): w_k = sigmoid(z_k) / max(sum
// over on-grid k' of sigmoid(z_k'), 1e-6)  (Sec. 5.1 "Fused CUDA
// normalization": sigmoid, local sum, clamp, divide); off-grid slots weigh 0.
// ---------------------------------------------------------------------------
struct W3 { float w0, w1, w2; };

__device__ __forceinline__ W3 normalise_plain(float z0, float z1, float z2, bool v0, bool v2) {
    float s0 = v0 ? 1.0f / (1.0f + expf(-z0)) : 0.0f;
    float s1 = 1.0f / (1.0f + expf(-z1));
    float s2 = v2 ? 1.0f / (1.0f + expf(-z2)) : 0.0f;
    float S = fmaxf(s0 + s1 + s2, 1e-6f);
    W3 r;
    r.w0 = s0 / S;
    r.w1 = s1 / S;
    r.w2 = s2 / S;
    return r;
}

}  // namespace gspn
