// Sweep-pair kernel, bf16 inputs and output.
#include "pair_launch.cuh"

namespace gspn_host {

cudaError_t launch_pair_bf16(int RP, int NS, const gspn::PairParams &pp, int smem,
                             const DeviceProps &dp, cudaStream_t s, LaunchInfo &li) {
    return launch_pair_r<__nv_bfloat16>(RP, NS, pp, smem, dp, s, li);
}

}  // namespace gspn_host
