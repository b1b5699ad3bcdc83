// Launch of the Prop2D backward kernel (prop2d_bwd.cuh), both element types.
#include "launch.h"

namespace gspn_host {

template <typename T, int R>
static cudaError_t launch_bwd_t(const gspn::BwdParams &bp, int smem, const DeviceProps &dp, int cap,
                                cudaStream_t stream, LaunchInfo &li) {
    auto kern = gspn::prop2d_bwd_kernel<T, R>;
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(reinterpret_cast<const void *>(kern), gspn::kBwdThreads, smem, per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (cap > 0 && per_sm > cap) per_sm = cap;
    long long grid = static_cast<long long>(dp.sms) * per_sm;
    const long long planes = static_cast<long long>(bp.B) * bp.Cc;
    if (grid > planes) grid = planes;
    kern<<<static_cast<unsigned>(grid), gspn::kBwdThreads, smem, stream>>>(bp);
    li.launches = 1;
    li.grid = static_cast<int>(grid);
    li.block = gspn::kBwdThreads;
    li.smem = smem;
    li.path = "bwd";
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_bwd_r(const gspn::BwdParams &bp, int smem, const DeviceProps &dp, int cap,
                                cudaStream_t s, LaunchInfo &li) {
    switch (bp.R) {
        case 1: return launch_bwd_t<T, 1>(bp, smem, dp, cap, s, li);
        case 2: return launch_bwd_t<T, 2>(bp, smem, dp, cap, s, li);
        case 3: return launch_bwd_t<T, 3>(bp, smem, dp, cap, s, li);
        case 4: return launch_bwd_t<T, 4>(bp, smem, dp, cap, s, li);
        case 5: return launch_bwd_t<T, 5>(bp, smem, dp, cap, s, li);
        case 6: return launch_bwd_t<T, 6>(bp, smem, dp, cap, s, li);
        case 7: return launch_bwd_t<T, 7>(bp, smem, dp, cap, s, li);
        case 8: return launch_bwd_t<T, 8>(bp, smem, dp, cap, s, li);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_bwd(const gspn::BwdParams &bp, bool bf16, int smem, const DeviceProps &dp, int cap,
                       cudaStream_t s, LaunchInfo &li) {
    return bf16 ? launch_bwd_r<__nv_bfloat16>(bp, smem, dp, cap, s, li)
                : launch_bwd_r<float>(bp, smem, dp, cap, s, li);
}

}  // namespace gspn_host
