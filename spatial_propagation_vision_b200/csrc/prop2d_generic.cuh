// General Prop2D forward for shapes the direction and sweep-pair kernels do
// not take (lines longer than 256 positions, lines of one position, or bf16
// rows of odd width, whose rows are not 4-byte aligned).  A CTA of four warps owns a
// plane band, warp d runs direction d; each warp keeps its
// previous and current hidden line in shared memory, lanes stride over the
// positions of a line, and inputs are read straight from global memory.
// Correct for every size; not tuned.
#pragma once

#include "device_common.cuh"

namespace gspn {

constexpr int kGenericThreads = 128;   // 4 warps: one per direction

struct GenericParams {
    const void *x, *lam, *wl, *u;
    void *out;
    int B, Cc, H, W, dirs;
    int gate_dirs;          // direction slots of lambda and u: 4, or 1 shared by all directions
    int w_groups, w_cpg;    // logit fields per (batch, direction) and channels per field
    int n_items, bands, band_rows;
    int hline;      // floats reserved per hidden line (>= max(H, W))
    int y_pitch;
};

template <typename T>
__global__ void __launch_bounds__(kGenericThreads)
prop2d_generic_kernel(const GenericParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = warp;
    const bool active = (p.dirs >> d) & 1;
    const bool rowdir = d < 2, fwd = (d & 1) == 0;
    const int H = p.H, W = p.W;
    const int L = rowdir ? H : W, M = rowdir ? W : H;
    const size_t HW = static_cast<size_t>(H) * W;
    const int YP = p.y_pitch;
    float *ys = reinterpret_cast<float *>(smem);
    float *hbuf = ys + static_cast<size_t>(p.band_rows) * YP + static_cast<size_t>(warp) * 2 * p.hline;
    const T *X = static_cast<const T *>(p.x);
    const T *LA = static_cast<const T *>(p.lam);
    const T *U = static_cast<const T *>(p.u);
    const T *WL = static_cast<const T *>(p.wl);

    for (int e = threadIdx.x; e < p.band_rows * YP; e += kGenericThreads) ys[e] = 0.0f;
    __syncthreads();

    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
        const int plane = item / p.bands, band = item - plane * p.bands;
        const int band_lo = band * p.band_rows, band_hi = min(H, band_lo + p.band_rows);
        const int b = plane / p.Cc, c = plane - b * p.Cc;
        if (active) {
            const size_t xo = (static_cast<size_t>(b) * p.Cc + c) * HW;
            const size_t go =
                ((static_cast<size_t>(b) * p.gate_dirs + (p.gate_dirs == 4 ? d : 0)) * p.Cc + c) * HW;
            const size_t wo = (((static_cast<size_t>(b) * 4 + d) * p.w_groups + c / p.w_cpg) * 3) * HW;
            float *hprev = hbuf, *hcur = hbuf + p.hline;
            for (int q = lane; q < M; q += 32) hprev[q] = 0.0f;
            __syncwarp();
            for (int step = 0; step < L; ++step) {
                const int line = fwd ? step : L - 1 - step;
                for (int q = lane; q < M; q += 32) {
                    const int i = rowdir ? line : q, j = rowdir ? q : line;
                    const size_t e = static_cast<size_t>(i) * W + j;
                    const float z0 = q > 0 ? to_f(WL[wo + e]) : 0.0f;
                    const float z1 = to_f(WL[wo + HW + e]);
                    const float z2 = q + 1 < M ? to_f(WL[wo + 2 * HW + e]) : 0.0f;
                    const W3 w = normalise_plain(z0, z1, z2, q > 0, q + 1 < M);
                    float acc = to_f(LA[go + e]) * to_f(X[xo + e]);
                    if (q > 0) acc = fmaf(w.w0, hprev[q - 1], acc);
                    acc = fmaf(w.w1, hprev[q], acc);
                    if (q + 1 < M) acc = fmaf(w.w2, hprev[q + 1], acc);
                    hcur[q] = acc;
                    if (i >= band_lo && i < band_hi)
                        atomicAdd(ys + (i - band_lo) * YP + j, to_f(U[go + e]) * acc);
                }
                __syncwarp();
                float *t = hprev; hprev = hcur; hcur = t;
            }
        }
        __syncthreads();
        T *outp = static_cast<T *>(p.out) + (static_cast<size_t>(b) * p.Cc + c) * HW +
                  static_cast<size_t>(band_lo) * W;
        const int n = (band_hi - band_lo) * W;
        for (int e = threadIdx.x; e < n; e += kGenericThreads) {
            const int i = e / W, j = e - i * W;
            outp[e] = from_f<T>(ys[i * YP + j]);
            ys[i * YP + j] = 0.0f;
        }
        __syncthreads();
    }
}

}  // namespace gspn
