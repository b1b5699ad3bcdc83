// C ABI of libgspn.so (declared in include/gspn.h): argument checks, launch
// planning and dispatch to the Prop2D kernels.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "gspn.h"
#include "launch.h"

namespace {

using gspn::DirParams;
using gspn::GenericParams;
using namespace gspn_host;

thread_local LaunchInfo g_last;

// How the gate and logit tensors are shared: direction slots of lambda and
// u (4, or 1 shared by all directions) and logit fields per (batch,
// direction) (Cc per channel; 1 the compact mode's shared field).
struct Sharing {
    int gate_dirs, w_groups;
};

constexpr int kMaxDirLine = 256;        // longest line (H or W) the direction kernel holds in registers
constexpr int kMaxGenericLine = 4096;   // longest line the general kernel accepts

}  // namespace

namespace {

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
    if ((e = cudaDeviceGetAttribute(&dp.l2_bytes, cudaDevAttrL2CacheSize, dev))) return e;
    if (dev < 64) { cache[dev] = dp; have[dev] = true; }
    return cudaSuccess;
}

}  // namespace

namespace gspn_host {

cudaError_t kernel_occupancy(const void *kernel, int threads, int smem, int &per_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    struct Entry { int dev; const void *kernel; int threads, smem, per_sm; };
    static std::mutex mu;
    static Entry cache[256];
    static int n = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i) {
        const Entry &c = cache[i];
        if (c.dev == dev && c.kernel == kernel && c.threads == threads && c.smem == smem) {
            per_sm = c.per_sm;
            return cudaSuccess;
        }
    }
    // the limit is per kernel: raise it once to the device maximum (never
    // lower it, which would fail a later launch with more shared memory)
    bool raised = false;
    for (int i = 0; i < n && !raised; ++i) raised = cache[i].dev == dev && cache[i].kernel == kernel;
    if (!raised) {
        int optin = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        if (e != cudaSuccess) return e;
    }
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (n < 256) cache[n++] = Entry{dev, kernel, threads, smem, per_sm};
    return cudaSuccess;
}

}  // namespace gspn_host

namespace {

// Shared-memory plan for output mode `mode` so that one CTA fits `cap`
// bytes.  Output modes: 0, fp32 output planes in shared memory (one for the
// row directions, one for the column directions); 1, fp32 outputs
// accumulated in global memory (L2 atomics); 2, row bands of the two planes
// in shared memory (the scans are rerun per band); 3, one fp32 plane in
// shared memory that all directions add into with shared-memory atomics.  Layout: row plane or
// band, column plane or band, the column rings of the enabled column
// directions, then the column warps' plane-pointer tables.
bool plan_dir_fit(DirPlan &pl, int cap, int H, int W, int dirs, int mode) {
    const int n_col = ((dirs >> 2) & 1) + ((dirs >> 3) & 1);
    // odd pitch above every swizzled column index (see ycol), whose last
    // column is a dummy written by row lanes past the end of a row
    const int YP = (W % 2 == 0) ? W + 1 : W + 2;
    const int stage_col = round_up(H * gspn::kColPitch, 16);
    // global accumulation (fp32 only) stages a chunk's column outputs after
    // each column ring: (H x 4 + 32) floats (rows shifted one word per lane block)
    const int col_ring = gspn::kColStages * stage_col + (mode == 1 ? round_up((H * 4 + 32) * 4, 16) : 0);
    const int rings = n_col * col_ring + gspn::kDirBarBytes;
    const int n_planes = mode == 3 ? 1 : ((dirs & 3) ? 1 : 0) + ((dirs & 12) ? 1 : 0);
    // a plane holds its rows plus one dummy row (written by the column lanes
    // past the end of a column or outside the band)
    int band_rows = H, plane_bytes = 0;
    // mode 4 (bf16 planes of pair words): W / 2 words and a dummy per row
    const int YPW = W / 2 + 1;
    if (mode == 4) {
        // the two column sweeps meet at a word boundary: each needs at least
        // one word on its side (W >= 4), or one of them would never reach
        // the midpoint barrier
        if (W < 4 || W % 2) return false;
        plane_bytes = round_up((H + 1) * YPW * 4, 16);
    } else if (mode == 0 || mode == 3) {
        plane_bytes = round_up((H + 1) * YP * 4, 16);
    } else if (mode == 2) {
        if (cap - rings < n_planes * 2 * YP * 4) return false;
        band_rows = (cap - rings) / (n_planes * YP * 4) - 1;
        if (band_rows > H) band_rows = H;
        plane_bytes = round_up((band_rows + 1) * YP * 4, 16);
    }
    const int y_bytes = n_planes * plane_bytes;
    if (y_bytes + rings > cap) return false;
    DirParams &p = pl.p;
    p.stage_col = stage_col;
    p.ycol_off = (mode != 3 && (dirs & 3)) ? plane_bytes : 0;
    int off = y_bytes;
    for (int d = 0; d < 4; ++d) {
        if (d < 2 || !((dirs >> d) & 1)) { p.ring[d] = -1; continue; }
        p.ring[d] = off;
        off += col_ring;
    }
    p.bar_off = off;
    p.y_pitch = mode == 4 ? YPW : YP;
    p.band_rows = band_rows;
    p.bands = (H + band_rows - 1) / band_rows;
    pl.smem = y_bytes + rings;
    pl.y_global = mode == 1;
    pl.y_shared = mode == 3;
    pl.y_half = mode == 4;
    return true;
}

bool misaligned(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) != 0; }

}  // namespace

extern "C" const char *gspn_status_str(gspn_status s) {
    switch (s) {
        case GSPN_OK: return "GSPN_OK";
        case GSPN_ERR_NULL: return "GSPN_ERR_NULL: a required pointer is NULL";
        case GSPN_ERR_SHAPE: return "GSPN_ERR_SHAPE: unsupported or negative size";
        case GSPN_ERR_DIRS: return "GSPN_ERR_DIRS: dirs must be 1..15 and share_w 0 or 1";
        case GSPN_ERR_WORKSPACE: return "GSPN_ERR_WORKSPACE: workspace smaller than gspn_prop2d_workspace_bytes";
        case GSPN_ERR_DTYPE: return "GSPN_ERR_DTYPE: unknown dtype";
        case GSPN_ERR_ALIGN: return "GSPN_ERR_ALIGN: device pointers must be 16-byte aligned";
        case GSPN_ERR_CUDA: return "GSPN_ERR_CUDA: CUDA runtime error";
        case GSPN_ERR_DEVICE: return "GSPN_ERR_DEVICE: the current device is not sm_100";
        case GSPN_ERR_SHARING:
            return "GSPN_ERR_SHARING: gate_dirs must be 1 or 4 and w_groups a divisor of Cc";
        case GSPN_ERR_ALGO:
            return "GSPN_ERR_ALGO: unknown algorithm, or one that cannot run these sizes";
        case GSPN_ERR_NOALLOC_LIMIT:
            return "GSPN_ERR_NOALLOC_LIMIT: these sizes need more scratch than the library's "
                   "built-in GSPN_NOALLOC_WORKSPACE_BYTES array";
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

namespace {

// Bytes of the compact mode's normalised weights: [B][4][1][3][H][W] of fp32
// (fp32 inputs) or fp16 (bf16 inputs).
size_t workspace_bytes(int B, int H, int W, int share_w, gspn_dtype dtype) {
    if (!share_w || B <= 0 || H <= 0 || W <= 0) return 0;
    const size_t es = dtype == GSPN_BF16 ? 2 : 4;
    return static_cast<size_t>(B) * 4 * 3 * H * W * es;
}

using DirLaunch = cudaError_t (*)(int, const DirPlan &, const DeviceProps &, cudaStream_t, LaunchInfo &);

// The direction kernel variant for (element size, output path, weights
// normalised ahead).
DirLaunch dir_variant(int es, const DirPlan &pl, bool pre) {
    if (es == 4) {
        // (fp32 never needs bands: global accumulation always fits)
        if (pl.y_global) return pre ? launch_dir_f32_global_pre : launch_dir_f32_global;
        if (pl.y_shared) return pre ? launch_dir_f32_shared_pre : launch_dir_f32_shared;
        return pre ? launch_dir_f32_smem_pre : launch_dir_f32_smem;
    }
    if (pl.y_half) return pre ? launch_dir_bf16_half_pre : launch_dir_bf16_half;
    if (pl.y_shared) return pre ? launch_dir_bf16_shared_pre : launch_dir_bf16_shared;
    return pre ? launch_dir_bf16_banded_pre : launch_dir_bf16_banded;
}

// Lines of up to kMaxPairLine positions run on the sweep-pair kernel, with
// RP pairs and NS single positions per lane chosen from the longer side:
// capacity 32 RP + 16 NS.
constexpr int kMaxPairLine = 128;

// Planes that leave most of the GPU idle when one CTA runs a whole plane go
// to the cluster-split kernel (one CTA per direction).
constexpr int kMaxSplitLine = 128;

// Cluster-split kernel (prop2d_split.cuh) when the shape suits it: both sides
// 2..128, plane byte sizes a multiple of 4 (4-byte tail copies), the six
// staged planes and the fp32 output plane within one CTA's shared memory.
// Without `forced`, only for fewer planes than twice the SM count (than the
// SM count for lines of up to 16, where the sweep-pair kernel is quick) whose
// CTAs (four per plane) run in at most two waves.  Measured on B200 (device time
// per call, CUDA graphs, split vs the best other kernel): 16 x 16 x 4 planes
// fp32 4.9 vs 6.9 us; 74 x 74 bf16, 64 planes 22 vs 50 us, 128 planes 42 vs
// 50 us, 256 planes (four waves) 83 vs 54 us; 37 x 37 fp32, 256 planes 21 vs
// 24 us, 512 planes (three waves) 32 vs 29 us; 16 x 16 fp32, 512 planes 15 vs
// 8 us.  `taken` tells whether it was launched.
cudaError_t try_split(const void *x, const void *lambda, const void *wlogit, const void *u, int B,
                      int Cc, int H, int W, int dirs, Sharing sh, int es, void *out,
                      const DeviceProps &dp, cudaStream_t stream, bool forced, bool &taken) {
    taken = false;
    const int mx = H > W ? H : W;
    if (H < 2 || W < 2 || mx > kMaxSplitLine) return cudaSuccess;
    const long long HW = static_cast<long long>(H) * W;
    if ((HW * es) % 4 != 0) return cudaSuccess;
    const long long planes = static_cast<long long>(B) * Cc;
    if (!forced && (planes >= 2LL * dp.sms || (planes >= dp.sms && mx <= 16))) return cudaSuccess;
    const long long slot = round_up(static_cast<int>(HW * es) + 16, 16);
    const long long y_off = gspn::kTensors * slot;
    const long long smem = y_off + round_up(static_cast<int>((HW + 1) * 4), 16);
    if (smem > dp.smem_optin) return cudaSuccess;
    const int R = (mx + 31) / 32;
    if (!forced) {
        int per_sm = 0;
        if (split_occupancy(R, es == 2, static_cast<int>(smem), per_sm) != cudaSuccess) return cudaSuccess;
        if (planes * gspn::kSplitCluster > 2LL * dp.sms * per_sm) return cudaSuccess;
    }
    if (static_cast<long long>(B) * Cc * gspn::kSplitCluster > 0x7fffffffLL) return cudaSuccess;
    gspn::SplitParams sp{};
    sp.x = x; sp.lam = lambda; sp.wl = wlogit; sp.u = u; sp.out = out;
    sp.B = B; sp.Cc = Cc; sp.H = H; sp.W = W; sp.dirs = dirs;
    sp.gate_dirs = sh.gate_dirs;
    sp.w_groups = sh.w_groups;
    sp.w_cpg = Cc / sh.w_groups;
    sp.slot = static_cast<int>(slot);
    sp.y_off = static_cast<int>(y_off);
    taken = true;
    return launch_split(R, es == 2, sp, static_cast<int>(smem), stream, g_last);
}

// Sweep-pair kernel (prop2d_pair.cuh) when the shape suits it: both sides
// 2..128, rows at least as long as the lanes' pair blocks (their words are
// read straight from global memory), bf16 rows of even width (4-byte aligned
// pair words), every tensor under 4 GiB (32-bit byte offsets), and the two
// output planes and the column rings in shared memory.  `taken` tells
// whether it was launched.
cudaError_t try_pair(const void *x, const void *lambda, const void *wlogit, const void *u, int B,
                     int Cc, int H, int W, int dirs, Sharing sh, int es, void *out,
                     const DeviceProps &dp, cudaStream_t stream, bool forced, bool &taken) {
    taken = false;
    const int mx = H > W ? H : W;
    if (H < 2 || W < 2 || mx > kMaxPairLine || (es == 2 && W % 2)) return cudaSuccess;
    // Measured on B200 against the direction kernel: the sweep-pair kernel is
    // faster for lines of up to 16 positions (16 x 16, fp32: 0.0156 vs
    // 0.0174 ms) and for the row directions alone (74 x 74, bf16: 0.229 vs
    // 0.253 ms), slower when column directions take part on longer lines
    // (74 x 74, bf16, four directions: 0.52 vs 0.33 ms; its one column warp
    // per plane runs both column sweeps).  It takes the shapes where it wins.
    if (!forced && mx > 16 && (dirs & 12) != 0) return cudaSuccess;
    const int bucket = (mx + 15) / 16 - 1;           // 0 .. 7
    const int RP = bucket / 2, NS = bucket % 2 + 1;  // capacity 32 RP + 16 NS >= mx
    if (W < 32 * RP) return cudaSuccess;
    const unsigned long long plane = static_cast<unsigned long long>(H) * W * es;
    const unsigned long long xb = static_cast<unsigned long long>(B) * Cc * plane;
    const unsigned long long gb = static_cast<unsigned long long>(sh.gate_dirs) * xb;
    const unsigned long long wb = static_cast<unsigned long long>(B) * 4 * sh.w_groups * 3 * plane;
    if (gb >= (1ULL << 32) || wb >= (1ULL << 32)) return cudaSuccess;
    // output line pitch: at least the capacity, a multiple of 4 floats with
    // an odd number of 16-byte units (conflict-free transposed reads)
    const int cap = 32 * RP + 16 * NS;
    int yp = round_up(cap, 4);
    if ((yp / 4) % 2 == 0) yp += 4;
    const int grp = RP > 0 ? 2 * RP : 1;
    const int stage = round_up(4 * (H * gspn::kPairRowWords + ((H + grp - 1) / grp) * gspn::kPairSkewWords), 16);
    // output planes of the I/O element type (bf16 partial sums for bf16 inputs)
    const int q_off = round_up(H * yp * es, 16);
    const int ring_off = q_off + round_up(W * yp * es, 16);
    const int smem = ring_off + 2 * gspn::kPairStages * stage;
    if (smem > dp.smem_optin) return cudaSuccess;
    gspn::PairParams pp{};
    pp.x = static_cast<const char *>(x);
    pp.lam = static_cast<const char *>(lambda);
    pp.u = static_cast<const char *>(u);
    pp.wl0 = static_cast<const char *>(wlogit);
    pp.wl1 = pp.wl0 + plane;
    pp.wl2 = pp.wl0 + 2 * plane;
    pp.out = out;
    pp.B = B; pp.Cc = Cc; pp.H = H; pp.W = W; pp.dirs = dirs;
    pp.gate_dirs = sh.gate_dirs;
    pp.w_groups = sh.w_groups;
    pp.w_cpg = Cc / sh.w_groups;
    pp.n_items = B * Cc;
    pp.yp = yp;
    pp.q_off = q_off;
    pp.ring_off = ring_off;
    pp.stage_bytes = stage;
    pp.x_bytes = static_cast<unsigned int>(xb);
    pp.g_bytes = static_cast<unsigned int>(gb);
    pp.w_bytes = static_cast<unsigned int>(wb);
    taken = true;
    return es == 2 ? launch_pair_bf16(RP, NS, pp, smem, dp, stream, g_last)
                   : launch_pair_f32(RP, NS, pp, smem, dp, stream, g_last);
}

// Prop2D with the callers' sharing of gates and logits, and an optional
// workspace (one logit field per (batch, direction) only: the weights are
// then normalised once into it and read by every channel).  The callers
// check `dirs` and the sharing arguments.
gspn_status prop2d_run(const void *x, const void *lambda, const void *wlogit, const void *u, int B,
                       int Cc, int H, int W, int dirs, Sharing sh, gspn_dtype dtype, void *out,
                       void *ws, cudaStream_t stream, gspn_algo algo = GSPN_ALGO_AUTO) {
    g_last = LaunchInfo{};
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return GSPN_ERR_SHAPE;
    if (dtype != GSPN_F32 && dtype != GSPN_BF16) return GSPN_ERR_DTYPE;
    if (B == 0 || Cc == 0 || H == 0 || W == 0) return GSPN_OK;
    if (!x || !lambda || !wlogit || !u || !out) return GSPN_ERR_NULL;
    if (misaligned(x) || misaligned(lambda) || misaligned(wlogit) || misaligned(u) || misaligned(out))
        return GSPN_ERR_ALIGN;
    // planes, rows and item counts must fit 32-bit ints (element offsets are 64-bit)
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
    const bool pre = sh.w_groups == 1 && ws;
    const bool any = algo == GSPN_ALGO_AUTO;
    // Routing (GSPN_ALGO_AUTO), from B200 measurements: few planes run on the
    // cluster-split kernel (see try_split); the sweep-pair kernel takes lines
    // of up to 16 and the row directions alone (see try_pair); the rest runs
    // on the direction kernel, else the general kernel.
    if (!pre && (any || algo == GSPN_ALGO_SPLIT)) {
        bool taken = false;
        err = try_split(x, lambda, wlogit, u, B, Cc, H, W, dirs, sh, es, out, dp, stream, !any, taken);
        if (taken) return err == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
        if (!any) return GSPN_ERR_ALGO;
    }
    if (!pre && (any || algo == GSPN_ALGO_SWEEP_PAIR)) {
        bool taken = false;
        err = try_pair(x, lambda, wlogit, u, B, Cc, H, W, dirs, sh, es, out, dp, stream, !any, taken);
        if (taken) return err == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
        if (!any) return GSPN_ERR_ALGO;
    }
    // bf16 rows of even width keep every row and span 4-byte aligned
    const bool dir_ok = maxline <= kMaxDirLine && H >= 2 && W >= 2 && (es == 4 || (W % 2 == 0));
    if (dir_ok && (any || algo == GSPN_ALGO_DIRECTION)) {
        const int R = (maxline + 31) / 32;
        DirPlan pl;
        pl.p.x = x; pl.p.lam = lambda; pl.p.wl = wlogit; pl.p.u = u; pl.p.out = out;
        pl.p.B = B; pl.p.Cc = Cc; pl.p.H = H; pl.p.W = W; pl.p.dirs = dirs;
        pl.p.gate_dirs = sh.gate_dirs;
        pl.p.w_groups = sh.w_groups;
        pl.p.w_cpg = Cc / sh.w_groups;
        // Output modes in order of preference (the last reruns the scans per
        // band); within a mode, the most CTAs per SM that fit.
        const int caps[4] = {dp.smem_per_sm / 4 - 1024, dp.smem_per_sm / 3 - 1024,
                             dp.smem_per_sm / 2 - 1024, dp.smem_optin};
        bool fit = false;
        // bf16: one plane with shared atomics (the four directions run
        // uncoupled until the end of an item), else bands; fp32: two planes
        // (atomic-free), one plane, else global atomics (which always fit)
        const int order_bf16[3] = {4, 3, 2}, order_f32[3] = {0, 3, 1};
        const int n_order = 3;
        for (int oi = 0; oi < n_order && !fit; ++oi) {
            const int mode = es == 2 ? order_bf16[oi] : order_f32[oi];
            for (int ci = 0; ci < 4 && !fit; ++ci) {
                const int cap = caps[ci] < dp.smem_optin ? caps[ci] : dp.smem_optin;
                fit = plan_dir_fit(pl, cap, H, W, dirs, mode);
            }
        }
        if (fit) {
            pl.p.n_items = B * Cc * pl.p.bands;
            const unsigned long long plane_bytes = static_cast<unsigned long long>(HW) * es;
            pl.p.end_x = static_cast<unsigned long long>(B) * Cc * plane_bytes;
            pl.p.end_gate = static_cast<unsigned long long>(sh.gate_dirs) * pl.p.end_x;
            pl.p.end_wl = static_cast<unsigned long long>(B) * 4 * sh.w_groups * 3 * plane_bytes;
            if (pre) {
                // the compact mode's weights, normalised once for all channels
                gspn::NormParams np{wlogit, ws, B, H, W, dirs};
                if (launch_norm(np, es == 2, dp, stream) != cudaSuccess) return GSPN_ERR_CUDA;
                pl.p.wl = ws;
            }
            err = dir_variant(es, pl, pre)(R, pl, dp, stream, g_last);
            if (pre) g_last.launches += 1;
            return err == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
        }
    }
    if (!any && algo != GSPN_ALGO_GENERIC) return GSPN_ERR_ALGO;
    GenericParams gp{};
    gp.x = x; gp.lam = lambda; gp.wl = wlogit; gp.u = u; gp.out = out;
    gp.B = B; gp.Cc = Cc; gp.H = H; gp.W = W; gp.dirs = dirs;
    gp.gate_dirs = sh.gate_dirs;
    gp.w_groups = sh.w_groups;
    gp.w_cpg = Cc / sh.w_groups;
    bool fits = false;
    err = launch_generic(gp, es == 2, dp, stream, fits, g_last);
    if (!fits) return GSPN_ERR_SHAPE;
    return err == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace

extern "C" gspn_status gspn_prop2d_fwd(const void *x, const void *lambda, const void *wlogit,
                                       const void *u, int B, int Cc, int H, int W, int dirs,
                                       int share_w, gspn_dtype dtype, void *out,
                                       cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (dirs < 1 || dirs > 15 || (share_w != 0 && share_w != 1)) return GSPN_ERR_DIRS;
    return prop2d_run(x, lambda, wlogit, u, B, Cc, H, W, dirs, Sharing{4, share_w ? 1 : Cc}, dtype,
                      out, nullptr, stream);
}

extern "C" gspn_status gspn_prop2d_fwd_ex(const void *x, const void *lambda, const void *wlogit,
                                          const void *u, int B, int Cc, int H, int W, int dirs,
                                          int gate_dirs, int w_groups, gspn_dtype dtype, void *out,
                                          cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (dirs < 1 || dirs > 15) return GSPN_ERR_DIRS;
    if ((gate_dirs != 1 && gate_dirs != 4) || w_groups < 1 || (Cc > 0 && Cc % w_groups != 0))
        return GSPN_ERR_SHARING;
    return prop2d_run(x, lambda, wlogit, u, B, Cc, H, W, dirs, Sharing{gate_dirs, w_groups}, dtype,
                      out, nullptr, stream);
}

extern "C" gspn_status gspn_prop2d_fwd_algo(const void *x, const void *lambda, const void *wlogit,
                                            const void *u, int B, int Cc, int H, int W, int dirs,
                                            int gate_dirs, int w_groups, gspn_dtype dtype,
                                            gspn_algo algo, void *out, cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (dirs < 1 || dirs > 15) return GSPN_ERR_DIRS;
    if ((gate_dirs != 1 && gate_dirs != 4) || w_groups < 1 || (Cc > 0 && Cc % w_groups != 0))
        return GSPN_ERR_SHARING;
    if (algo < GSPN_ALGO_AUTO || algo > GSPN_ALGO_GENERIC) return GSPN_ERR_ALGO;
    return prop2d_run(x, lambda, wlogit, u, B, Cc, H, W, dirs, Sharing{gate_dirs, w_groups}, dtype,
                      out, nullptr, stream, algo);
}

extern "C" size_t gspn_prop2d_workspace_bytes(int B, int Cc, int H, int W, int dirs, int share_w,
                                              gspn_dtype dtype) {
    if (Cc < 0 || dirs < 1 || dirs > 15 || (dtype != GSPN_F32 && dtype != GSPN_BF16)) return 0;
    return workspace_bytes(B, H, W, share_w, dtype);
}

extern "C" gspn_status gspn_prop2d_fwd_ws(const void *x, const void *lambda, const void *wlogit,
                                          const void *u, int B, int Cc, int H, int W, int dirs,
                                          int share_w, gspn_dtype dtype, void *out, void *workspace,
                                          size_t workspace_size, cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return GSPN_ERR_SHAPE;
    if (dirs < 1 || dirs > 15 || (share_w != 0 && share_w != 1)) return GSPN_ERR_DIRS;
    if (dtype != GSPN_F32 && dtype != GSPN_BF16) return GSPN_ERR_DTYPE;
    if (B == 0 || Cc == 0 || H == 0 || W == 0) return GSPN_OK;
    const size_t need = workspace_bytes(B, H, W, share_w, dtype);
    if (need > 0) {
        if (!workspace) return GSPN_ERR_NULL;
        if (workspace_size < need) return GSPN_ERR_WORKSPACE;
        if (misaligned(workspace)) return GSPN_ERR_ALIGN;
    }
    return prop2d_run(x, lambda, wlogit, u, B, Cc, H, W, dirs, Sharing{4, share_w ? 1 : Cc}, dtype,
                      out, need > 0 ? workspace : nullptr, stream);
}

namespace {

constexpr int kHostChunks = 4;   // batch chunks of the pipelined host entry point

// Streams and events of the host entry point's pipeline, made once per
// device: uploads, kernels and downloads of consecutive batch chunks run on
// their own streams so that they overlap.
struct HostPipe {
    std::mutex mu;            // one host call at a time per device
    bool ready = false;
    cudaStream_t up = nullptr, run = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, uploaded[kHostChunks] = {}, computed[kHostChunks] = {};
};

cudaError_t host_pipe(HostPipe *&hp) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static HostPipe pipes[64];
    static std::mutex mu;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    hp = &pipes[dev];
    std::lock_guard<std::mutex> lock(mu);
    if (hp->ready) return cudaSuccess;
    const unsigned nb = cudaStreamNonBlocking, nt = cudaEventDisableTiming;
    if ((e = cudaStreamCreateWithFlags(&hp->up, nb))) return e;
    if ((e = cudaStreamCreateWithFlags(&hp->run, nb))) return e;
    if ((e = cudaStreamCreateWithFlags(&hp->down, nb))) return e;
    if ((e = cudaEventCreateWithFlags(&hp->start, nt))) return e;
    for (int c = 0; c < kHostChunks; ++c) {
        if ((e = cudaEventCreateWithFlags(&hp->uploaded[c], nt))) return e;
        if ((e = cudaEventCreateWithFlags(&hp->computed[c], nt))) return e;
    }
    hp->ready = true;
    return cudaSuccess;
}

}  // namespace

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
    // bytes per batch element of each tensor (the batch is the outer dimension)
    const size_t bx = static_cast<size_t>(Cc) * plane;
    const size_t bg = 4 * bx;
    const size_t bw = static_cast<size_t>(4) * (share_w ? 1 : Cc) * 3 * plane;
    HostPipe *hp = nullptr;
    if (host_pipe(hp) != cudaSuccess) return GSPN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(hp->mu);
    // the pipeline starts after the work already queued on `stream`
    if (cudaEventRecord(hp->start, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaStreamWaitEvent(hp->up, hp->start, 0) != cudaSuccess) return GSPN_ERR_CUDA;
    // Chunks start at multiples of m batch elements, m the least count whose
    // bytes in every tensor are a multiple of 16, so that each chunk's device
    // pointers keep the kernels' 16-byte alignment.
    auto lcm16 = [](size_t bytes) { size_t m = 1; while ((m * bytes) % 16) ++m; return m; };
    const size_t mx_ = lcm16(bx), mw_ = lcm16(bw);
    size_t m = mx_;
    while (m % mw_) m += mx_;
    const long long units = (static_cast<long long>(B) + static_cast<long long>(m) - 1) / static_cast<long long>(m);
    const int nchunk = units < kHostChunks ? static_cast<int>(units) : kHostChunks;
    auto cb = [](const void *p, size_t off) { return static_cast<const char *>(p) + off; };
    auto mb = [](void *p, size_t off) { return static_cast<char *>(p) + off; };
    auto edge = [&](int c) {
        const long long b = static_cast<long long>(m) * (units * c / nchunk);
        return static_cast<int>(b < B ? b : B);
    };
    for (int c = 0; c < nchunk; ++c) {
        const int b0 = edge(c);
        const int b1 = edge(c + 1);
        const size_t n = static_cast<size_t>(b1 - b0);
        if (cudaMemcpyAsync(mb(d_x, b0 * bx), cb(h_x, b0 * bx), n * bx, cudaMemcpyHostToDevice, hp->up) ||
            cudaMemcpyAsync(mb(d_lambda, b0 * bg), cb(h_lambda, b0 * bg), n * bg, cudaMemcpyHostToDevice, hp->up) ||
            cudaMemcpyAsync(mb(d_wlogit, b0 * bw), cb(h_wlogit, b0 * bw), n * bw, cudaMemcpyHostToDevice, hp->up) ||
            cudaMemcpyAsync(mb(d_u, b0 * bg), cb(h_u, b0 * bg), n * bg, cudaMemcpyHostToDevice, hp->up) ||
            cudaEventRecord(hp->uploaded[c], hp->up) || cudaStreamWaitEvent(hp->run, hp->uploaded[c], 0))
            return GSPN_ERR_CUDA;
        const gspn_status st = gspn_prop2d_fwd(cb(d_x, b0 * bx), cb(d_lambda, b0 * bg),
                                               cb(d_wlogit, b0 * bw), cb(d_u, b0 * bg),
                                               b1 - b0, Cc, H, W, dirs, share_w, dtype,
                                               mb(d_out, b0 * bx), hp->run);
        if (st != GSPN_OK) return st;
        if (cudaEventRecord(hp->computed[c], hp->run) || cudaStreamWaitEvent(hp->down, hp->computed[c], 0) ||
            cudaMemcpyAsync(mb(h_out, b0 * bx), cb(d_out, b0 * bx), n * bx, cudaMemcpyDeviceToHost, hp->down))
            return GSPN_ERR_CUDA;
    }
    // the downloads wait for every kernel, which waited for every upload
    if (cudaStreamSynchronize(hp->down) != cudaSuccess) return GSPN_ERR_CUDA;
    return GSPN_OK;
}

// ---------------------------------------------------------------------------
// gspn_prop2d_fwd_noalloc: the compact mode's scratch in a library-owned
// array, for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------

// The scratch array.  Every device that loads the library holds one copy
// until the process exits.  In host code this name is only a host-side
// stand-in: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GSPN_NOALLOC_WORKSPACE_BYTES];

namespace {

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the first call on a device does it, with that device current).
cudaError_t noalloc_scratch(void **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static void *addr[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" gspn_status gspn_prop2d_fwd_noalloc(const void *x, const void *lambda,
                                               const void *wlogit, const void *u, int B, int Cc,
                                               int H, int W, int dirs, int share_w,
                                               gspn_dtype dtype, void *out, cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return GSPN_ERR_SHAPE;
    if (dirs < 1 || dirs > 15 || (share_w != 0 && share_w != 1)) return GSPN_ERR_DIRS;
    if (dtype != GSPN_F32 && dtype != GSPN_BF16) return GSPN_ERR_DTYPE;
    if (B == 0 || Cc == 0 || H == 0 || W == 0) return GSPN_OK;
    const size_t need = workspace_bytes(B, H, W, share_w, dtype);
    if (need > GSPN_NOALLOC_WORKSPACE_BYTES) return GSPN_ERR_NOALLOC_LIMIT;
    void *ws = nullptr;
    if (need > 0 && noalloc_scratch(&ws) != cudaSuccess) return GSPN_ERR_CUDA;
    return prop2d_run(x, lambda, wlogit, u, B, Cc, H, W, dirs, Sharing{4, share_w ? 1 : Cc}, dtype,
                      out, ws, stream);
}

// ---------------------------------------------------------------------------
// gspn_prop2d_bwd: gradients of Prop2D
// ---------------------------------------------------------------------------

namespace {
constexpr int kMaxBwdLine = 256;   // lines the backward kernel holds (8 positions per lane)
}  // namespace

namespace {

gspn_status prop2d_bwd_run(const void *x, const void *lambda, const void *wlogit, const void *u,
                           const void *gy, int B, int Cc, int H, int W, int dirs, Sharing sh,
                           gspn_dtype dtype, float *dx, float *dlambda, float *dwlogit, float *du,
                           cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return GSPN_ERR_SHAPE;
    if (dtype != GSPN_F32 && dtype != GSPN_BF16) return GSPN_ERR_DTYPE;
    if (B == 0 || Cc == 0 || H == 0 || W == 0) return GSPN_OK;
    if (!x || !lambda || !wlogit || !u || !gy || !dx || !dlambda || !dwlogit || !du)
        return GSPN_ERR_NULL;
    if (misaligned(x) || misaligned(lambda) || misaligned(wlogit) || misaligned(u) || misaligned(gy) ||
        misaligned(dx) || misaligned(dlambda) || misaligned(dwlogit) || misaligned(du))
        return GSPN_ERR_ALIGN;
    const int maxline = H > W ? H : W;
    if (maxline > kMaxBwdLine || static_cast<long long>(H) * W > (1LL << 30) ||
        static_cast<long long>(B) * Cc > 0x7fffffffLL)
        return GSPN_ERR_SHAPE;
    DeviceProps dp;
    if (device_props(dp) != cudaSuccess) return GSPN_ERR_CUDA;
    if (dp.major != 10) return GSPN_ERR_DEVICE;
    const size_t plane = static_cast<size_t>(H) * W * sizeof(float);
    const size_t nx = static_cast<size_t>(B) * Cc * plane;
    const size_t nw = static_cast<size_t>(B) * 4 * sh.w_groups * 3 * plane;
    if (cudaMemsetAsync(dx, 0, nx, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaMemsetAsync(dlambda, 0, sh.gate_dirs * nx, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaMemsetAsync(du, 0, sh.gate_dirs * nx, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaMemsetAsync(dwlogit, 0, nw, stream) != cudaSuccess) return GSPN_ERR_CUDA;
    gspn::BwdParams bp{};
    bp.x = x; bp.lam = lambda; bp.wl = wlogit; bp.u = u; bp.gy = gy;
    bp.dx = dx; bp.dlam = dlambda; bp.dwl = dwlogit; bp.du = du;
    bp.B = B; bp.Cc = Cc; bp.H = H; bp.W = W; bp.dirs = dirs;
    bp.gate_dirs = sh.gate_dirs;
    bp.w_groups = sh.w_groups;
    bp.w_cpg = Cc / sh.w_groups;
    bp.R = (maxline + 31) / 32;
    bp.n_ckpt = (maxline + gspn::kBwdSeg - 1) / gspn::kBwdSeg;
    bp.warp_floats = (bp.n_ckpt + gspn::kBwdSeg + 1) * 32 * bp.R;
    const int smem = 4 * bp.warp_floats * static_cast<int>(sizeof(float));
    if (smem > dp.smem_optin) return GSPN_ERR_SHAPE;
    // The column sweeps read one element per lane from 32 grid rows, and each
    // 32-byte sector is met again by the next columns' steps: when the
    // problem's inputs and gradients exceed L2, two CTAs per SM keep the
    // resident planes' sectors in L2 between those steps (B200, 74 x 74 bf16
    // x 2048 planes: 5.0 ms against 12.1 ms with six CTAs per SM, whose DRAM
    // reads were 20 x the data; 148 x 148 x 512 shared logits: 5.0 vs 6.6 ms;
    // 37 x 37 fp32 x 512 planes, whose 120 MB fit L2: 0.24 ms uncapped, 0.35
    // capped).
    const int es = dtype == GSPN_BF16 ? 2 : 4;
    const double per_plane = static_cast<double>(H) * W * (22.0 * es + 4.0 * 21.0);
    const int cap = static_cast<double>(B) * Cc * per_plane > static_cast<double>(dp.l2_bytes) ? 2 : 0;
    const cudaError_t e = launch_bwd(bp, dtype == GSPN_BF16, smem, dp, cap, stream, g_last);
    return e == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA;
}

}  // namespace

extern "C" gspn_status gspn_prop2d_bwd(const void *x, const void *lambda, const void *wlogit,
                                       const void *u, const void *gy, int B, int Cc, int H, int W,
                                       int dirs, int share_w, gspn_dtype dtype, float *dx,
                                       float *dlambda, float *dwlogit, float *du,
                                       cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (dirs < 1 || dirs > 15 || (share_w != 0 && share_w != 1)) return GSPN_ERR_DIRS;
    return prop2d_bwd_run(x, lambda, wlogit, u, gy, B, Cc, H, W, dirs,
                          Sharing{4, share_w ? 1 : (Cc > 0 ? Cc : 1)}, dtype, dx, dlambda, dwlogit,
                          du, stream);
}

extern "C" gspn_status gspn_prop2d_bwd_ex(const void *x, const void *lambda, const void *wlogit,
                                          const void *u, const void *gy, int B, int Cc, int H,
                                          int W, int dirs, int gate_dirs, int w_groups,
                                          gspn_dtype dtype, float *dx, float *dlambda,
                                          float *dwlogit, float *du, cudaStream_t stream) {
    g_last = LaunchInfo{};
    if (dirs < 1 || dirs > 15) return GSPN_ERR_DIRS;
    if ((gate_dirs != 1 && gate_dirs != 4) || w_groups < 1 || (Cc > 0 && Cc % w_groups != 0))
        return GSPN_ERR_SHARING;
    return prop2d_bwd_run(x, lambda, wlogit, u, gy, B, Cc, H, W, dirs, Sharing{gate_dirs, w_groups},
                          dtype, dx, dlambda, dwlogit, du, stream);
}
