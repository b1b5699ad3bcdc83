// Device helpers shared by the Prop2D kernels: element conversion, async
// global->shared copies and the fused row-stochastic normalisation.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace gspn {

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
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
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// bulk (TMA engine, non-tensor) copies global -> shared completed on an
// mbarrier, and the mbarrier operations around them.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(mbar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t mbar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
                 " selp.u32 %0, 1, 0, p;\n}" : "=r"(ok) : "r"(mbar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(mbar) : "memory");
}
// Bulk prefetch of [src, src + bytes) into L2 (TMA engine); src 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bit set in the library's device status word (a __device__ variable of the
// API translation unit whose address every launch passes in) by a kernel
// whose bounded wait for an asynchronous copy gave up; read and cleared by
// gspn_device_status().
constexpr unsigned int kStatusCopyTimeout = 1u;
constexpr long long kMaxWaitPolls = 1LL << 26;

// Wait for phase `parity` of an mbarrier, polling at most kMaxWaitPolls
// times; on timeout record it and return false (the caller carries on
// with whatever the buffer holds, so the launch still terminates).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t mbar, uint32_t parity, unsigned int *status) {
    for (long long i = 0; i < kMaxWaitPolls; ++i)
        if (mbar_try_wait(mbar, parity)) return true;
    atomicOr(status, kStatusCopyTimeout);
    return false;
}

__device__ __forceinline__ void red_add_shared_if(uint32_t addr, float v, bool pred) {
    // No memory clobber: these only add into the output plane, which is read
    // back after a barrier (itself ordered against every volatile asm here).
    asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %2, 0;\n @p red.shared.add.f32 [%0], %1;\n}"
                 ::"r"(addr), "f"(v), "r"(static_cast<uint32_t>(pred)));
}

// Copy the 4-byte words [w0, w0 + nwords) of a global buffer to shared
// memory, one warp cooperating.  `gsrc` is 4-byte aligned; `sdst` is the
// shared address that receives gsrc's first byte and has the same address
// modulo 16, so the aligned middle moves in 16-byte pieces.
__device__ __forceinline__ void warp_copy_words(uint32_t sdst, const char *gsrc, int nbytes,
                                                int lane) {
    const uintptr_t g = reinterpret_cast<uintptr_t>(gsrc);
    const int head = static_cast<int>(((16 - (g & 15)) & 15));      // bytes before 16B boundary
    const int h = head < nbytes ? head : nbytes;
    // head words
    for (int b = lane * 4; b < h; b += 128) cp_async_4(sdst + b, gsrc + b);
    const int body = (nbytes - h) & ~15;
    for (int b = h + lane * 16; b < h + body; b += 32 * 16) cp_async_16(sdst + b, gsrc + b);
    for (int b = h + body + lane * 4; b < nbytes; b += 128) cp_async_4(sdst + b, gsrc + b);
}

// ---------------------------------------------------------------------------
// Fused normalisation: w_k = sigmoid(z_k) / max(sum over on-grid k' of
// sigmoid(z_k'), 1e-6)  (Sec. 5.1 "Fused CUDA normalization": sigmoid, local
// sum, clamp, divide).
//
// Fast form: with a_k = 1 + exp(-z_k), sigmoid(z_k) = 1 / a_k, and
//   w_k = P_k / (P_0 + P_1 + P_2),   P_k = product of a_j over on-grid j != k,
// which needs three exponentials and one reciprocal.  An off-grid slot takes
// a_k = 1 and P_k = 0.  The clamp can only bind when every on-grid logit is
// below about -13.8, and the products overflow only when two logits are
// below about -44; both make the denominator exceed 1e11, in which case the
// plain form is evaluated instead.
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

// Returns false when the fast form is out of its safe range (caller then uses
// normalise_plain).  Weights are always written.
__device__ __forceinline__ bool normalise_fast(float z0, float z1, float z2, bool v0, bool v2,
                                               W3 &w) {
    float a0 = v0 ? 1.0f + __expf(-z0) : 1.0f;
    float a1 = 1.0f + __expf(-z1);
    float a2 = v2 ? 1.0f + __expf(-z2) : 1.0f;
    float p0 = v0 ? a1 * a2 : 0.0f;
    float p1 = a0 * a2;
    float p2 = v2 ? a0 * a1 : 0.0f;
    float D = p0 + p1 + p2;
    float r = __fdividef(1.0f, D);
    w.w0 = p0 * r;
    w.w1 = p1 * r;
    w.w2 = p2 * r;
    return D <= 1e11f;
}

}  // namespace gspn
