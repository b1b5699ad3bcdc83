// Prop2D for few (batch, channel) planes: each plane is split over a
// thread-block cluster of four CTAs, one per scan direction ("Scaling
// Parallel Sequence Models to Foundation-Scale Vision Encoders", Sec. 6.1
// "L1 cache and SM utilization": small inputs leave most SMs idle when a
// plane is the unit of work, which calls for a finer decomposition).
//
// CTA d of a cluster (one warp) runs direction d of plane blockIdx.x / 4:
//   1. it copies the six planes it reads (lambda_d, u_d, the three logit
//      slots of direction d, x) whole into shared memory with 16-byte
//      cp.async (each plane's 16-byte-aligned span, plus 4-byte copies for
//      a tail that ends off a 16-byte boundary), so that every scan step
//      reads shared memory, not L2;
//   2. it scans its L lines (lane l holds positions l*R .. l*R + R - 1),
//      with the normalisation of the direction kernel (fast form, a line
//      redone in the plain form when flagged) and stores u_d * h_d of every
//      position into its own fp32 output plane in shared memory;
//   3. after a cluster barrier, CTA k sums the four planes over distributed
//      shared memory for a quarter of the positions (directions in the
//      order 0..3) and writes y; a second barrier keeps every plane alive
//      until all reads are done.
// Disabled directions copy and scan nothing and are left out of the sum.
#pragma once

#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_bf16.h>

#include "device_common.cuh"
#include "prop2d_dir.cuh"

namespace gspn {

constexpr int kSplitThreads = 32;   // one warp per CTA
constexpr int kSplitCluster = 4;    // CTAs per plane: one per direction

struct SplitParams {
    const void *x, *lam, *wl, *u;
    void *out;
    int B, Cc, H, W, dirs;
    int gate_dirs;          // direction slots of lambda and u: 4, or 1 shared by all directions
    int w_groups, w_cpg;    // logit fields per (batch, direction) and channels per field
    int slot;               // bytes per staged plane (multiple of 16)
    int y_off;              // byte offset of the fp32 output plane ([H*W] + one dummy)
};

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}

// Element offset of plane (b, c) of tensor t for direction d (tensor order
// of the direction kernel: lambda, u, logit slots 0..2, x).
__device__ __forceinline__ size_t split_plane(const SplitParams &p, int b, int c, int d, int t) {
    const size_t HW = static_cast<size_t>(p.H) * p.W;
    if (t == 5) return (static_cast<size_t>(b) * p.Cc + c) * HW;
    if (t < 2)
        return ((static_cast<size_t>(b) * p.gate_dirs + (p.gate_dirs == 4 ? d : 0)) * p.Cc + c) * HW;
    return ((((static_cast<size_t>(b) * 4 + d) * p.w_groups + c / p.w_cpg) * 3) + (t - 2)) * HW;
}

template <typename T>
__device__ __forceinline__ float split_ld(const unsigned char *p) {
    if constexpr (sizeof(T) == 2) return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const unsigned short *>(p)) << 16);
    else return *reinterpret_cast<const float *>(p);
}

template <typename T, int R>
__global__ void __cluster_dims__(kSplitCluster, 1, 1) __launch_bounds__(kSplitThreads)
prop2d_split_kernel(const SplitParams p) {
    namespace cg = cooperative_groups;
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int es = sizeof(T);
    cg::cluster_group cluster = cg::this_cluster();
    const int d = static_cast<int>(cluster.block_rank());
    const int plane = blockIdx.x / kSplitCluster;
    const int b = plane / p.Cc, c = plane - b * p.Cc;
    const int lane = threadIdx.x;
    const int HW = p.H * p.W;
    float *yp = reinterpret_cast<float *>(smem + p.y_off);

    if ((p.dirs >> d) & 1) {
        // 1. the six planes, each at (its address mod 16) within its slot
        int adj[kTensors];
#pragma unroll
        for (int t = 0; t < kTensors; ++t) {
            const void *base = t == 0 ? p.lam : t == 1 ? p.u : t == 5 ? p.x : p.wl;
            const unsigned char *src = static_cast<const unsigned char *>(base) + split_plane(p, b, c, d, t) * es;
            const uintptr_t a = reinterpret_cast<uintptr_t>(src);
            adj[t] = static_cast<int>(a & 15);
            const unsigned char *a0 = src - adj[t];
            const uintptr_t e = a + static_cast<uintptr_t>(HW) * es;
            const unsigned char *e16 = reinterpret_cast<const unsigned char *>(e & ~static_cast<uintptr_t>(15));
            const int n16 = static_cast<int>((e16 - a0) / 16);
            const uint32_t dst = smem_u32(smem + t * p.slot);
            for (int i = lane; i < n16; i += kSplitThreads) cp_async_16(dst + 16u * i, a0 + 16 * i);
            const int tail = static_cast<int>((e & 15) / 4);   // plane bytes are a multiple of 4
            if (lane < tail) cp_async_4(dst + 16u * n16 + 4u * lane, e16 + 4 * lane);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();

        // 2. the scan
        const bool rows = d < 2, fwd = (d & 1) == 0;
        const int L = rows ? p.H : p.W, M = rows ? p.W : p.H;
        const int lstride = rows ? p.W : 1;       // elements between consecutive lines
        LaneGeom<R> g;
        g.init(lane, M);
        int qo[R], yo[R];   // element offset of each position in a line (clamped), output slot base
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = min(lane * R + r, M - 1);
            qo[r] = rows ? q : q * p.W;
            yo[r] = g.valid[r] ? qo[r] : HW;      // past the end: the dummy slot
        }
        const unsigned char *sl[kTensors];
#pragma unroll
        for (int t = 0; t < kTensors; ++t) sl[t] = smem + t * p.slot + adj[t];
        auto load_line = [&](int s, float (&v)[kTensors][R]) {
            const int lo = (fwd ? s : L - 1 - s) * lstride;
#pragma unroll
            for (int t = 0; t < kTensors; ++t)
#pragma unroll
                for (int r = 0; r < R; ++r) v[t][r] = split_ld<T>(sl[t] + (qo[r] + lo) * es);
        };
        float h[R];
#pragma unroll
        for (int r = 0; r < R; ++r) h[r] = 0.0f;
        float v[kTensors][R];
        LineW<R> Wc;
        load_line(0, v);
        line_terms(v, g, Wc);
        load_line(min(1, L - 1), v);
        for (int s = 0; s < L; ++s) {
            recur(h, Wc);
            const int lo = (fwd ? s : L - 1 - s) * lstride;
#pragma unroll
            for (int r = 0; r < R; ++r) yp[g.valid[r] ? yo[r] + lo : HW] = Wc.uu[r] * h[r];
            // weights of line s+1 (past the last line: finite, never used),
            // then the values of line s+2
            const bool bad = line_weights(v, g, Wc);
            float vn[kTensors][R];
            load_line(min(s + 2, L - 1), vn);
            if (__any_sync(0xffffffffu, bad)) line_weights_plain_v<R>(v, g, Wc);
#pragma unroll
            for (int t = 0; t < kTensors; ++t)
#pragma unroll
                for (int r = 0; r < R; ++r) v[t][r] = vn[t][r];
        }
        __syncwarp();
    }

    // 3. the sum of the directions' planes over distributed shared memory
    cluster.sync();
    const float *pl[kSplitCluster];
#pragma unroll
    for (int k = 0; k < kSplitCluster; ++k) pl[k] = cluster.map_shared_rank(yp, k);
    const int per = (HW + kSplitCluster - 1) / kSplitCluster;
    const int lo = d * per, hi = min(HW, lo + per);
    T *o = static_cast<T *>(p.out) + static_cast<size_t>(plane) * HW;
    for (int i = lo + lane; i < hi; i += kSplitThreads) {
        float s = 0.0f;
#pragma unroll
        for (int k = 0; k < kSplitCluster; ++k)
            if ((p.dirs >> k) & 1) s += pl[k][i];
        o[i] = from_f<T>(s);
    }
    cluster.sync();
}

}  // namespace gspn
