// Launch of the cluster-split kernel (prop2d_split.cuh): one cluster of four
// CTAs per (batch, channel) plane.
#include "launch.h"
#include "prop2d_split.cuh"

namespace gspn_host {

namespace {

template <typename T, int R>
cudaError_t launch_split_t(const gspn::SplitParams &sp, int smem, cudaStream_t stream, LaunchInfo &li) {
    auto kern = gspn::prop2d_split_kernel<T, R>;
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(reinterpret_cast<const void *>(kern), gspn::kSplitThreads, smem, per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long grid = static_cast<long long>(sp.B) * sp.Cc * gspn::kSplitCluster;
    kern<<<static_cast<unsigned>(grid), gspn::kSplitThreads, smem, stream>>>(sp);
    li.launches = 1;
    li.grid = static_cast<int>(grid);
    li.block = gspn::kSplitThreads;
    li.smem = smem;
    li.path = "split";
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_split_r(int R, const gspn::SplitParams &sp, int smem, cudaStream_t s, LaunchInfo &li) {
    switch (R) {
        case 1: return launch_split_t<T, 1>(sp, smem, s, li);
        case 2: return launch_split_t<T, 2>(sp, smem, s, li);
        case 3: return launch_split_t<T, 3>(sp, smem, s, li);
        case 4: return launch_split_t<T, 4>(sp, smem, s, li);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
const void *split_kernel_ptr(int R) {
    switch (R) {
        case 1: return reinterpret_cast<const void *>(gspn::prop2d_split_kernel<T, 1>);
        case 2: return reinterpret_cast<const void *>(gspn::prop2d_split_kernel<T, 2>);
        case 3: return reinterpret_cast<const void *>(gspn::prop2d_split_kernel<T, 3>);
        case 4: return reinterpret_cast<const void *>(gspn::prop2d_split_kernel<T, 4>);
        default: return nullptr;
    }
}

}  // namespace

cudaError_t split_occupancy(int R, bool bf16, int smem, int &per_sm) {
    const void *k = bf16 ? split_kernel_ptr<__nv_bfloat16>(R) : split_kernel_ptr<float>(R);
    if (!k) return cudaErrorInvalidValue;
    return kernel_occupancy(k, gspn::kSplitThreads, smem, per_sm);
}

cudaError_t launch_split(int R, bool bf16, const gspn::SplitParams &sp, int smem, cudaStream_t s,
                         LaunchInfo &li) {
    return bf16 ? launch_split_r<__nv_bfloat16>(R, sp, smem, s, li) : launch_split_r<float>(R, sp, smem, s, li);
}

}  // namespace gspn_host
