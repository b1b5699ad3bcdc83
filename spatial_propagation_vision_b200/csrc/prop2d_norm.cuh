// Normalised weights of the compact multi-channel mode, computed once per
// (batch, direction, position) and read by the scans of every channel
// ("Scaling Parallel Sequence Models to Foundation-Scale Vision Encoders",
// Sec. 4.2 "Channel-shared weights and the attention view": one w field per
// position shared across channels; Sec. 5.1 "Fused CUDA normalization":
// sigmoid, local sum over the on-grid neighbours, clamp, divide).
//
// Input:  logits [B][4][1][3][H][W] (the share_w layout), dtype T.
// Output: [B][4][1][3][H][W] of WT (fp32 for fp32 inputs, fp16 for bf16
//         inputs), slot 0 = w0, slot 1 = w0 + w1 + w2, slot 2 = w2.
// Storing the sum instead of w1 lets the scan form w1 as a difference, so
// the three weights it uses sum to the stored sum exactly: 1, unless the
// clamp bound (then sum s_k / eps < 1).  Off-grid slots get weight 0 and
// their logits are not read.  Only the directions in `dirs` are written.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace gspn {

struct NormParams {
    const void *wl;   // logits, share_w layout
    void *ws;         // normalised weights, same layout
    int B, H, W, dirs;
};

template <typename T> __device__ __forceinline__ float norm_in(const T *p);
template <> __device__ __forceinline__ float norm_in<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float norm_in<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
}
template <typename WT> __device__ __forceinline__ WT norm_out(float v);
template <> __device__ __forceinline__ float norm_out<float>(float v) { return v; }
template <> __device__ __forceinline__ __half norm_out<__half>(float v) { return __float2half_rn(v); }

// sigmoid(z) = 1 / (1 + e^-z), saturating to 0 or 1 for large |z|.
__device__ __forceinline__ float norm_sigmoid(float z) { return 1.0f / (1.0f + expf(-z)); }

// Grid-stride over (b, d) planes (y) and the positions of a plane (x).  Row
// lines (d = 0, 1) have their neighbour slots along W (j-1, j, j+1); column
// lines (d = 2, 3) along H.
template <typename T, typename WT>
__global__ void prop2d_norm_kernel(const NormParams p) {
    const int HW = p.H * p.W;
    const T *wl = static_cast<const T *>(p.wl);
    WT *ws = static_cast<WT *>(p.ws);
    for (long long bd = blockIdx.y; bd < 4LL * p.B; bd += gridDim.y) {
        const int d = static_cast<int>(bd % 4);
        if (!((p.dirs >> d) & 1)) continue;
        const int M = d < 2 ? p.W : p.H;
        const T *z = wl + bd * 3 * HW;
        WT *w = ws + bd * 3 * HW;
        for (int pos = blockIdx.x * blockDim.x + threadIdx.x; pos < HW; pos += gridDim.x * blockDim.x) {
            const int i = pos / p.W, j = pos - i * p.W;
            const int q = d < 2 ? j : i;
            const float s0 = q > 0 ? norm_sigmoid(norm_in<T>(z + pos)) : 0.0f;
            const float s1 = norm_sigmoid(norm_in<T>(z + static_cast<long long>(HW) + pos));
            const float s2 = q + 1 < M ? norm_sigmoid(norm_in<T>(z + 2LL * HW + pos)) : 0.0f;
            const float sum = (s0 + s1) + s2;
            const float S = fmaxf(sum, 1e-6f);
            w[pos] = norm_out<WT>(s0 / S);
            w[static_cast<long long>(HW) + pos] = norm_out<WT>(sum >= 1e-6f ? 1.0f : sum / S);
            w[2LL * HW + pos] = norm_out<WT>(s2 / S);
        }
    }
}

}  // namespace gspn
