// Direction kernel variant: element type float, output mode kYBanded,
// weights normalised in the scan.
#include "dir_launch.cuh"

namespace gspn_host {

cudaError_t launch_dir_f32_banded(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li) {
    return launch_dir_r<float, gspn::kYBanded, false>(R, pl, dp, s, li);
}

}  // namespace gspn_host
