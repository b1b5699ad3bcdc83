// Host-side plumbing shared by the library's translation units: launch
// geometry, device properties and the per-variant launch functions.  Each
// (element type, output mode) variant of the direction kernel is compiled
// in its own translation unit so the library builds in parallel.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "prop2d_dir.cuh"
#include "prop2d_generic.cuh"
#include "prop2d_norm.cuh"
#include "prop2d_pair.cuh"
#include "prop2d_bwd.cuh"
#include "prop2d_split.cuh"

namespace gspn_host {

// What the last gspn_prop2d_fwd call on this host thread launched.
struct LaunchInfo {
    int launches = 0, grid = 0, block = 0, smem = 0;
    const char *path = "none";
};

struct DeviceProps {
    int sms = 0, smem_optin = 0, smem_per_sm = 0, major = 0, minor = 0, l2_bytes = 0;
};

// Launch geometry of the direction kernel.
struct DirPlan {
    bool y_global = false;
    bool y_shared = false;   // one plane, shared-memory atomics
    bool y_half = false;     // two bf16 planes of pair words, no atomics
    int smem = 0;
    gspn::DirParams p{};
};

inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Direction kernel, one function per (element type, output mode, weights
// normalised in the scan or ahead: _pre); R is the positions per lane (1..8).
cudaError_t launch_dir_f32_smem(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_f32_smem_pre(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_f32_global(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_f32_global_pre(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_f32_shared(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_f32_shared_pre(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_bf16_banded(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_bf16_banded_pre(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_bf16_shared(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_bf16_shared_pre(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_bf16_half(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_dir_bf16_half_pre(int R, const DirPlan &pl, const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);

// Sweep-pair kernel: RP position pairs and NS single positions per lane.
cudaError_t launch_pair_bf16(int RP, int NS, const gspn::PairParams &pp, int smem,
                             const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);
cudaError_t launch_pair_f32(int RP, int NS, const gspn::PairParams &pp, int smem,
                            const DeviceProps &dp, cudaStream_t s, LaunchInfo &li);

// Resident CTAs per SM of `kernel` with `smem` bytes of dynamic shared
// memory; sets the kernel's shared-memory limit.  Both are cached per
// (device, kernel, smem), so repeated calls make no runtime queries.
cudaError_t kernel_occupancy(const void *kernel, int threads, int smem, int &per_sm);

// Backward kernel (fp32 gradients); the caller zeroed the gradient buffers.
// `cap` > 0 limits the resident CTAs per SM.
cudaError_t launch_bwd(const gspn::BwdParams &bp, bool bf16, int smem, const DeviceProps &dp, int cap,
                       cudaStream_t s, LaunchInfo &li);

// Normalised weights of the compact mode into the workspace (one launch).
cudaError_t launch_norm(const gspn::NormParams &np, bool bf16, const DeviceProps &dp, cudaStream_t s);

// Cluster-split kernel: one cluster of four CTAs (one per direction) per
// plane; R positions per lane (1..4).
cudaError_t launch_split(int R, bool bf16, const gspn::SplitParams &sp, int smem, cudaStream_t s,
                         LaunchInfo &li);
// Resident CTAs per SM of that kernel with `smem` bytes (cached).
cudaError_t split_occupancy(int R, bool bf16, int smem, int &per_sm);

// General kernel; `fits` is false when even one output row does not fit.
cudaError_t launch_generic(const gspn::GenericParams &gp, bool bf16, const DeviceProps &dp,
                           cudaStream_t stream, bool &fits, LaunchInfo &li);

}  // namespace gspn_host
