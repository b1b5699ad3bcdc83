// Direction kernel variant: element type __nv_bfloat16, output mode kYHalf,
// weights normalised in the scan.
#include "dir_launch.cuh"

namespace gspn_host {

cudaError_t launch_dir_bf16_half(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li) {
    return launch_dir_r<__nv_bfloat16, gspn::kYHalf, false>(R, pl, dp, s, li);
}

}  // namespace gspn_host
