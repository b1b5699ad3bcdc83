// Launch of the sweep-pair kernel (prop2d_pair.cuh); included by the
// translation units that instantiate it for one element type.
#pragma once

#include "launch.h"

namespace gspn_host {

template <typename T, int RP, int NS>
cudaError_t launch_pair_t(const gspn::PairParams &pp, int smem, const DeviceProps &dp,
                          cudaStream_t stream, LaunchInfo &li) {
    auto kern = gspn::prop2d_pair_kernel<T, RP, NS>;
    int per_sm = 0;
    cudaError_t e = kernel_occupancy(reinterpret_cast<const void *>(kern), gspn::kPairThreads, smem, per_sm);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(dp.sms) * per_sm;
    if (grid > pp.n_items) grid = pp.n_items;
    kern<<<static_cast<unsigned>(grid), gspn::kPairThreads, smem, stream>>>(pp);
    li.launches = 1;
    li.grid = static_cast<int>(grid);
    li.block = gspn::kPairThreads;
    li.smem = smem;
    li.path = "pair";
    return cudaGetLastError();
}

// Positions per lane: RP pairs and NS singles (line capacity 32 RP + 16 NS).
template <typename T>
cudaError_t launch_pair_r(int RP, int NS, const gspn::PairParams &pp, int smem,
                          const DeviceProps &dp, cudaStream_t s, LaunchInfo &li) {
    switch (RP * 2 + (NS - 1)) {
        case 0: return launch_pair_t<T, 0, 1>(pp, smem, dp, s, li);
        case 1: return launch_pair_t<T, 0, 2>(pp, smem, dp, s, li);
        case 2: return launch_pair_t<T, 1, 1>(pp, smem, dp, s, li);
        case 3: return launch_pair_t<T, 1, 2>(pp, smem, dp, s, li);
        case 4: return launch_pair_t<T, 2, 1>(pp, smem, dp, s, li);
        case 5: return launch_pair_t<T, 2, 2>(pp, smem, dp, s, li);
        case 6: return launch_pair_t<T, 3, 1>(pp, smem, dp, s, li);
        case 7: return launch_pair_t<T, 3, 2>(pp, smem, dp, s, li);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gspn_host
