// Direction kernel variant: element type float, output mode kYGlobal,
// weights normalised ahead (compact mode).
#include "dir_launch.cuh"

namespace gspn_host {

cudaError_t launch_dir_f32_global_pre(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li) {
    return launch_dir_r<float, gspn::kYGlobal, true>(R, pl, dp, s, li);
}

}  // namespace gspn_host
