// Sweep-pair kernel, fp32 inputs and output.
#include "pair_launch.cuh"

namespace gspn_host {

cudaError_t launch_pair_f32(int RP, int NS, const gspn::PairParams &pp, int smem,
                            const DeviceProps &dp, cudaStream_t s, LaunchInfo &li) {
    return launch_pair_r<float>(RP, NS, pp, smem, dp, s, li);
}

}  // namespace gspn_host
