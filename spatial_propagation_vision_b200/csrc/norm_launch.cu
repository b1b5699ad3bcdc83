// Launch of the compact mode's weight normalisation (prop2d_norm.cuh).
#include "launch.h"

namespace gspn_host {

cudaError_t launch_norm(const gspn::NormParams &np, bool bf16, const DeviceProps &dp, cudaStream_t s) {
    constexpr int kBlock = 256;
    const int HW = np.H * np.W;
    int gx = (HW + kBlock - 1) / kBlock;
    const long long planes = 4LL * np.B;
    // about eight blocks per SM in all
    const int gy = static_cast<int>(planes < 65535 ? planes : 65535);
    const long long want = 8LL * dp.sms;
    if (static_cast<long long>(gx) * gy > want) gx = static_cast<int>(want / gy > 1 ? want / gy : 1);
    const dim3 grid(gx, gy);
    if (bf16) gspn::prop2d_norm_kernel<__nv_bfloat16, __half><<<grid, kBlock, 0, s>>>(np);
    else gspn::prop2d_norm_kernel<float, float><<<grid, kBlock, 0, s>>>(np);
    return cudaGetLastError();
}

}  // namespace gspn_host
