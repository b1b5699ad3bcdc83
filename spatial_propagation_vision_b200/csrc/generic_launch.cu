// Launch of the general Prop2D kernel (both element types).
#include "launch.h"

namespace gspn_host {

template <typename T>
static cudaError_t launch_generic_t(const gspn::GenericParams &gp0, const DeviceProps &dp,
                                    cudaStream_t stream, bool &fits, LaunchInfo &li) {
    gspn::GenericParams gp = gp0;
    const int YP = gp.W | 1;
    gp.y_pitch = YP;
    gp.hline = round_up(gp.H > gp.W ? gp.H : gp.W, 4);
    const int hbytes = 4 * 2 * gp.hline * 4;
    const int cap = dp.smem_optin;
    int band_rows = (cap - hbytes) / (YP * 4);
    fits = band_rows >= 1;
    if (!fits) return cudaSuccess;
    if (band_rows > gp.H) band_rows = gp.H;
    gp.band_rows = band_rows;
    gp.bands = (gp.H + band_rows - 1) / band_rows;
    gp.n_items = gp.B * gp.Cc * gp.bands;
    const int smem = round_up(band_rows * YP * 4, 16) + hbytes;
    auto kern = gspn::prop2d_generic_kernel<T>;
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(reinterpret_cast<const void *>(kern), gspn::kGenericThreads, smem, per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(dp.sms) * per_sm;
    if (grid > gp.n_items) grid = gp.n_items;
    kern<<<static_cast<unsigned>(grid), gspn::kGenericThreads, smem, stream>>>(gp);
    li.launches = 1;
    li.grid = static_cast<int>(grid);
    li.block = gspn::kGenericThreads;
    li.smem = smem;
    li.path = "generic";
    return cudaGetLastError();
}

cudaError_t launch_generic(const gspn::GenericParams &gp, bool bf16, const DeviceProps &dp,
                           cudaStream_t stream, bool &fits, LaunchInfo &li) {
    return bf16 ? launch_generic_t<__nv_bfloat16>(gp, dp, stream, fits, li)
                : launch_generic_t<float>(gp, dp, stream, fits, li);
}

}  // namespace gspn_host
