// Launch of one variant of the direction kernel; included by the
// translation units that instantiate the variants.
#pragma once

#include "launch.h"

namespace gspn_host {

template <typename T, int R, int MODE, bool PRE>
cudaError_t launch_dir_t(const DirPlan &pl, const DeviceProps &dp, cudaStream_t stream, LaunchInfo &li) {
    auto kern = gspn::prop2d_dir_kernel<T, R, MODE, PRE>;
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(reinterpret_cast<const void *>(kern), gspn::kDirThreads, pl.smem, per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(dp.sms) * per_sm;
    if (grid > pl.p.n_items) grid = pl.p.n_items;
    kern<<<static_cast<unsigned>(grid), gspn::kDirThreads, pl.smem, stream>>>(pl.p);
    li.launches = 1;
    li.grid = static_cast<int>(grid);
    li.block = gspn::kDirThreads;
    li.smem = pl.smem;
    li.path = MODE == gspn::kYGlobal   ? "dir-yglobal"
              : MODE == gspn::kYBanded ? "dir-banded"
              : MODE == gspn::kYShared ? "dir-shared"
              : MODE == gspn::kYHalf   ? "dir-half"
                                       : "dir";
    return cudaGetLastError();
}

template <typename T, int MODE, bool PRE>
cudaError_t launch_dir_r(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li) {
    switch (R) {
        case 1: return launch_dir_t<T, 1, MODE, PRE>(pl, dp, s, li);
        case 2: return launch_dir_t<T, 2, MODE, PRE>(pl, dp, s, li);
        case 3: return launch_dir_t<T, 3, MODE, PRE>(pl, dp, s, li);
        case 4: return launch_dir_t<T, 4, MODE, PRE>(pl, dp, s, li);
        case 5: return launch_dir_t<T, 5, MODE, PRE>(pl, dp, s, li);
        case 6: return launch_dir_t<T, 6, MODE, PRE>(pl, dp, s, li);
        case 7: return launch_dir_t<T, 7, MODE, PRE>(pl, dp, s, li);
        case 8: return launch_dir_t<T, 8, MODE, PRE>(pl, dp, s, li);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gspn_host
