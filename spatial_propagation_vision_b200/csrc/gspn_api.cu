// C ABI of libgspn.so (declared in include/gspn.h): argument checks, launch
// planning and dispatch to the Prop2D kernels.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "gspn.h"
#include "prop2d_fused.cuh"
#include "prop2d_generic.cuh"

namespace {

using gspn::FusedParams;
using gspn::GenericParams;

struct LaunchInfo {
    int launches = 0, grid = 0, block = 0, smem = 0;
    const char *path = "none";
};
thread_local LaunchInfo g_last;

constexpr int kMaxFusedLine = 256;      // longest line (H or W) the fused kernel holds in registers
constexpr int kMaxGenericLine = 4096;   // longest line the general kernel accepts

struct DeviceProps {
    int sms = 0, smem_optin = 0, smem_per_sm = 0, major = 0, minor = 0;
};

cudaError_t device_props(DeviceProps &dp) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static DeviceProps cache[64];
    static bool have[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && have[dev]) { dp = cache[dev]; return cudaSuccess; }
    if ((e = cudaDeviceGetAttribute(&dp.sms, cudaDevAttrMultiProcessorCount, dev))) return e;
    if ((e = cudaDeviceGetAttribute(&dp.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev))) return e;
    if ((e = cudaDeviceGetAttribute(&dp.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev))) return e;
    if ((e = cudaDeviceGetAttribute(&dp.major, cudaDevAttrComputeCapabilityMajor, dev))) return e;
    if ((e = cudaDeviceGetAttribute(&dp.minor, cudaDevAttrComputeCapabilityMinor, dev))) return e;
    if (dev < 64) { cache[dev] = dp; have[dev] = true; }
    return cudaSuccess;
}

inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Launch geometry of the fused kernel.
struct FusedPlan {
    bool ok = false;
    bool y_global = false;
    int smem = 0;
    FusedParams p{};
};

// Shared-memory bytes of one tensor slot for the row directions.
int row_slot_bytes(int t_row, int W, int es) { return round_up(t_row * W * es + 16, 16); }
// ... and for the column directions (rows of pw words, one extra word every 32 rows).
int col_slot_bytes(int H, int pw, int R) {
    return round_up((H * pw + ((R % 2 == 0) ? H / 32 + 1 : 0)) * 4, 16);
}

// Choose chunk sizes and the output mode so that the CTA fits `cap` bytes.
bool plan_fused_fit(FusedPlan &pl, int cap, int H, int W, int dirs, int es, int R,
                    bool allow_yg, int min_seg_bytes) {
    const bool any_row = dirs & 3, any_col = dirs & 12;
    const int n_row = ((dirs & 1) ? 1 : 0) + ((dirs & 2) ? 1 : 0);
    const int n_col = ((dirs & 4) ? 1 : 0) + ((dirs & 8) ? 1 : 0);
    const int YP = W | 1;
    // output mode: full plane in smem, else (fp32) global atomics, else bands
    for (int mode = 0; mode < 3; ++mode) {
        if (mode == 1 && !allow_yg) continue;
        for (int seg_words = 8; seg_words >= 1; seg_words >>= 1) {
            const int t_col = seg_words * 4 / es;
            if (seg_words * 4 < min_seg_bytes) break;
            if (es == 2 && (t_col % 2)) continue;
            const int pw = (seg_words % 2 == 0) ? seg_words + 1 : seg_words;
            const int slot_col = col_slot_bytes(H, pw, R);
            const int col_ring = any_col ? n_col * gspn::kStages * gspn::kTensors * slot_col : 0;
            for (int t_row = 8; t_row >= 1; t_row >>= 1) {
                const int slot_row = row_slot_bytes(t_row, W, es);
                const int row_ring = any_row ? n_row * gspn::kStages * gspn::kTensors * slot_row : 0;
                int rings = col_ring + row_ring;
                int band_rows = H, y_bytes = 0;
                if (mode == 0) {
                    y_bytes = round_up(H * YP * 4, 16);
                } else if (mode == 2) {
                    const int avail = cap - rings;
                    if (avail < YP * 4) continue;
                    band_rows = avail / (YP * 4);
                    if (band_rows >= H) band_rows = H;
                    y_bytes = round_up(band_rows * YP * 4, 16);
                }
                if (y_bytes + rings > cap) continue;
                FusedParams &p = pl.p;
                p.t_row = t_row;
                p.slot_row = slot_row;
                p.t_col = t_col;
                p.words_col = seg_words;
                p.pw_col = pw;
                p.slot_col = slot_col;
                p.y_pitch = YP;
                p.band_rows = band_rows;
                p.bands = (H + band_rows - 1) / band_rows;
                int off = y_bytes;
                for (int d = 0; d < 4; ++d) {
                    if (!(dirs & (1 << d))) { p.ring_off[d] = -1; continue; }
                    p.ring_off[d] = off;
                    off += gspn::kStages * gspn::kTensors * (d < 2 ? slot_row : slot_col);
                }
                pl.smem = off;
                pl.y_global = (mode == 1);
                pl.ok = true;
                return true;
            }
        }
    }
    return false;
}

template <typename T, int R, bool YG>
cudaError_t launch_fused_t(const FusedPlan &pl, const DeviceProps &dp, cudaStream_t stream) {
    auto kern = gspn::prop2d_fused_kernel<T, R, YG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, gspn::kFusedThreads, pl.smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(dp.sms) * per_sm;
    if (grid > pl.p.n_items) grid = pl.p.n_items;
    kern<<<static_cast<unsigned>(grid), gspn::kFusedThreads, pl.smem, stream>>>(pl.p);
    g_last.launches = 1;
    g_last.grid = static_cast<int>(grid);
    g_last.block = gspn::kFusedThreads;
    g_last.smem = pl.smem;
    g_last.path = YG ? "fused-yglobal" : (pl.p.bands > 1 ? "fused-banded" : "fused");
    return cudaGetLastError();
}

template <typename T, bool YG>
cudaError_t launch_fused_r(int R, const FusedPlan &pl, const DeviceProps &dp, cudaStream_t s) {
    switch (R) {
        case 1: return launch_fused_t<T, 1, YG>(pl, dp, s);
        case 2: return launch_fused_t<T, 2, YG>(pl, dp, s);
        case 3: return launch_fused_t<T, 3, YG>(pl, dp, s);
        case 4: return launch_fused_t<T, 4, YG>(pl, dp, s);
        case 5: return launch_fused_t<T, 5, YG>(pl, dp, s);
        case 6: return launch_fused_t<T, 6, YG>(pl, dp, s);
        case 7: return launch_fused_t<T, 7, YG>(pl, dp, s);
        case 8: return launch_fused_t<T, 8, YG>(pl, dp, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_generic(const GenericParams &gp0, const DeviceProps &dp, cudaStream_t stream,
                           bool &fits) {
    GenericParams gp = gp0;
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
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, gspn::kFusedThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(dp.sms) * per_sm;
    if (grid > gp.n_items) grid = gp.n_items;
    kern<<<static_cast<unsigned>(grid), gspn::kFusedThreads, smem, stream>>>(gp);
    g_last.launches = 1;
    g_last.grid = static_cast<int>(grid);
    g_last.block = gspn::kFusedThreads;
    g_last.smem = smem;
    g_last.path = "generic";
    return cudaGetLastError();
}

bool misaligned(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) != 0; }

}  // namespace

extern "C" const char *gspn_status_str(gspn_status s) {
    switch (s) {
        case GSPN_OK: return "GSPN_OK";
        case GSPN_ERR_NULL: return "GSPN_ERR_NULL: a required pointer is NULL";
        case GSPN_ERR_SHAPE: return "GSPN_ERR_SHAPE: unsupported or negative size";
        case GSPN_ERR_DIRS: return "GSPN_ERR_DIRS: dirs must be 1..15 and share_w 0 or 1";
        case GSPN_ERR_DTYPE: return "GSPN_ERR_DTYPE: unknown dtype";
        case GSPN_ERR_ALIGN: return "GSPN_ERR_ALIGN: device pointers must be 16-byte aligned";
        case GSPN_ERR_CUDA: return "GSPN_ERR_CUDA: CUDA runtime error";
        case GSPN_ERR_DEVICE: return "GSPN_ERR_DEVICE: the current device is not sm_100";
    }
    return "GSPN_ERR_UNKNOWN";
}

extern "C" void gspn_last_launch_info(int *launches, int *grid, int *block, int *smem_bytes,
                                      const char **path) {
    if (launches) *launches = g_last.launches;
    if (grid) *grid = g_last.grid;
    if (block) *block = g_last.block;
    if (smem_bytes) *smem_bytes = g_last.smem;
    if (path) *path = g_last.path;
}

extern "C" gspn_status gspn_prop2d_fwd(const void *x, const void *lambda, const void *wlogit,
                                       const void *u, int B, int Cc, int H, int W, int dirs,
                                       int share_w, gspn_dtype dtype, void *out,
                                       cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return GSPN_ERR_SHAPE;
    if (dirs < 1 || dirs > 15 || (share_w != 0 && share_w != 1)) return GSPN_ERR_DIRS;
    if (dtype != GSPN_F32 && dtype != GSPN_BF16) return GSPN_ERR_DTYPE;
    if (B == 0 || Cc == 0 || H == 0 || W == 0) return GSPN_OK;
    if (!x || !lambda || !wlogit || !u || !out) return GSPN_ERR_NULL;
    if (misaligned(x) || misaligned(lambda) || misaligned(wlogit) || misaligned(u) || misaligned(out))
        return GSPN_ERR_ALIGN;
    // every element offset must fit the kernels' 64-bit indexing; planes and
    // item counts must fit 32-bit ints
    const long long HW = static_cast<long long>(H) * W;
    if (HW > (1LL << 30) || static_cast<long long>(B) * Cc * H > 0x7fffffffLL)
        return GSPN_ERR_SHAPE;
    const int maxline = H > W ? H : W;
    if (maxline > kMaxGenericLine) return GSPN_ERR_SHAPE;

    DeviceProps dp;
    if (device_props(dp) != cudaSuccess) return GSPN_ERR_CUDA;
    if (dp.major != 10) return GSPN_ERR_DEVICE;

    const int es = dtype == GSPN_BF16 ? 2 : 4;
    cudaError_t err = cudaSuccess;
    const bool fused_ok = maxline <= kMaxFusedLine && (es == 4 || (W % 2 == 0));
    if (fused_ok) {
        const int R = (maxline + 31) / 32;
        FusedPlan pl;
        pl.p.x = x; pl.p.lam = lambda; pl.p.wl = wlogit; pl.p.u = u; pl.p.out = out;
        pl.p.B = B; pl.p.Cc = Cc; pl.p.H = H; pl.p.W = W; pl.p.dirs = dirs; pl.p.share_w = share_w;
        // Prefer two CTAs per SM with >= 16-byte column segments; then one CTA per SM.
        const int cap2 = dp.smem_per_sm / 2 - 1024;
        const int cap1 = dp.smem_optin;
        bool fit = plan_fused_fit(pl, cap2 < cap1 ? cap2 : cap1, H, W, dirs, es, R, es == 4, 16) ||
                   plan_fused_fit(pl, cap1, H, W, dirs, es, R, es == 4, 16) ||
                   plan_fused_fit(pl, cap1, H, W, dirs, es, R, es == 4, 4);
        if (fit) {
            pl.p.n_items = B * Cc * pl.p.bands;
            if (es == 4) {
                err = pl.y_global ? launch_fused_r<float, true>(R, pl, dp, stream)
                                  : launch_fused_r<float, false>(R, pl, dp, stream);
            } else {
                err = launch_fused_r<__nv_bfloat16, false>(R, pl, dp, stream);
            }
            return err == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
        }
    }
    GenericParams gp{};
    gp.x = x; gp.lam = lambda; gp.wl = wlogit; gp.u = u; gp.out = out;
    gp.B = B; gp.Cc = Cc; gp.H = H; gp.W = W; gp.dirs = dirs; gp.share_w = share_w;
    bool fits = false;
    err = es == 4 ? launch_generic<float>(gp, dp, stream, fits)
                  : launch_generic<__nv_bfloat16>(gp, dp, stream, fits);
    if (!fits) return GSPN_ERR_SHAPE;
    return err == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

extern "C" gspn_status gspn_prop2d_fwd_host(const void *h_x, const void *h_lambda,
                                            const void *h_wlogit, const void *h_u, void *h_out,
                                            void *d_x, void *d_lambda, void *d_wlogit, void *d_u,
                                            void *d_out, int B, int Cc, int H, int W, int dirs,
                                            int share_w, gspn_dtype dtype, cudaStream_t stream) {
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return GSPN_ERR_SHAPE;
    if (dtype != GSPN_F32 && dtype != GSPN_BF16) return GSPN_ERR_DTYPE;
    if (dirs < 1 || dirs > 15 || (share_w != 0 && share_w != 1)) return GSPN_ERR_DIRS;
    if (B == 0 || Cc == 0 || H == 0 || W == 0) return GSPN_OK;
    if (!h_x || !h_lambda || !h_wlogit || !h_u || !h_out) return GSPN_ERR_NULL;
    if (!d_x || !d_lambda || !d_wlogit || !d_u || !d_out) return GSPN_ERR_NULL;
    const size_t es = dtype == GSPN_BF16 ? 2 : 4;
    const size_t plane = static_cast<size_t>(H) * W * es;
    const size_t nx = static_cast<size_t>(B) * Cc * plane;
    const size_t ng = static_cast<size_t>(B) * 4 * Cc * plane;
    const size_t nw = static_cast<size_t>(B) * 4 * (share_w ? 1 : Cc) * 3 * plane;
    if (cudaMemcpyAsync(d_x, h_x, nx, cudaMemcpyHostToDevice, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaMemcpyAsync(d_lambda, h_lambda, ng, cudaMemcpyHostToDevice, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaMemcpyAsync(d_wlogit, h_wlogit, nw, cudaMemcpyHostToDevice, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaMemcpyAsync(d_u, h_u, ng, cudaMemcpyHostToDevice, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    gspn_status st = gspn_prop2d_fwd(d_x, d_lambda, d_wlogit, d_u, B, Cc, H, W, dirs, share_w,
                                     dtype, d_out, stream);
    if (st != GSPN_OK) return st;
    if (cudaMemcpyAsync(h_out, d_out, nx, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GSPN_ERR_CUDA;
    return GSPN_OK;
}
