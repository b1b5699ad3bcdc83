// Direction kernel variant: element type float, output mode kYSmem,
// weights normalised ahead (compact mode).
#include "dir_launch.cuh"

namespace gspn_host {

cudaError_t launch_dir_f32_smem_pre(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li) {
    return launch_dir_r<float, gspn::kYSmem, true>(R, pl, dp, s, li);
}

}  // namespace gspn_host
