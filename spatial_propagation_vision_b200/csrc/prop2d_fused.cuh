// Fused Prop2D forward: normalisation + four directional line scans + gated
// direction sum in one launch.
//
// Work unit ("item"): one (batch, channel) plane, or one band of its rows
// when the plane's fp32 output does not fit in shared memory.  A CTA of four
// warps owns an item; warp d runs direction d (0 top->bottom, 1 bottom->top,
// 2 left->right, 3 right->left) over the whole plane.  CTAs are persistent
// and stride over the items.
//
// Per warp, lane l holds the R consecutive positions q = l*R + r of the
// current line in registers (the hidden line never leaves the register
// file); the q-1 / q+1 neighbours at lane edges come from warp shuffles.
// Input lines are streamed into a private 3-stage shared-memory ring with
// cp.async, several lines per stage:
//   * row directions stage whole rows: the rows of a chunk are one
//     contiguous span per tensor, moved in 16-byte pieces;
//   * column directions stage a strip of columns for every row (row
//     segments moved in 4-byte words), so each column line is read from
//     shared memory without a transpose pass in global memory.  The strip
//     pitch is an odd number of words so that lanes reading one column from
//     consecutive rows hit distinct banks.
// The six tensors of a line (lambda, u, three logits, x) share one stage.
// The normalised weights are computed in registers from the logits
// ("Fused CUDA normalization") and never stored.  The gated outputs of all
// four directions are summed into one fp32 plane in shared memory (or, for
// fp32 planes too large for it, straight into the fp32 output with L2
// atomics) and written once.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace gspn {

constexpr int kFusedThreads = 128;   // 4 warps: one per direction
constexpr int kStages = 3;           // cp.async ring depth per warp
constexpr int kTensors = 6;          // lambda, u, logit0, logit1, logit2, x

struct FusedParams {
    const void *x, *lam, *wl, *u;
    void *out;
    int B, Cc, H, W, dirs, share_w;
    int n_items, bands, band_rows;
    int t_row, slot_row;             // lines per chunk and bytes per tensor slot, row directions
    int t_col, words_col, pw_col, slot_col;  // col directions: lines per chunk, words per row
                                             // segment, row pitch in words, bytes per slot
    int ring_off[4];                 // byte offset of each warp's ring (-1: direction off)
    int y_pitch;                     // floats per staged output row (odd)
};

// Element offsets of the start of the (H x W) plane of each tensor for
// plane index (b, c) and direction d.
struct PlaneOffsets {
    size_t x, gate, wl;   // wl: offset of logit slot 0; slots 1, 2 follow at +HW, +2HW
};

__device__ __forceinline__ PlaneOffsets plane_offsets(const FusedParams &p, int b, int c, int d) {
    const size_t HW = static_cast<size_t>(p.H) * p.W;
    const int Cw = p.share_w ? 1 : p.Cc;
    const int cw = p.share_w ? 0 : c;
    PlaneOffsets o;
    o.x = (static_cast<size_t>(b) * p.Cc + c) * HW;
    o.gate = ((static_cast<size_t>(b) * 4 + d) * p.Cc + c) * HW;
    o.wl = (((static_cast<size_t>(b) * 4 + d) * Cw + cw) * 3) * HW;
    return o;
}

template <typename T>
__device__ __forceinline__ const char *tensor_plane(const FusedParams &p, const PlaneOffsets &o,
                                                    int t) {
    const size_t HW = static_cast<size_t>(p.H) * p.W;
    switch (t) {
        case 0: return reinterpret_cast<const char *>(static_cast<const T *>(p.lam) + o.gate);
        case 1: return reinterpret_cast<const char *>(static_cast<const T *>(p.u) + o.gate);
        case 2: return reinterpret_cast<const char *>(static_cast<const T *>(p.wl) + o.wl);
        case 3: return reinterpret_cast<const char *>(static_cast<const T *>(p.wl) + o.wl + HW);
        case 4: return reinterpret_cast<const char *>(static_cast<const T *>(p.wl) + o.wl + 2 * HW);
        default: return reinterpret_cast<const char *>(static_cast<const T *>(p.x) + o.x);
    }
}

// Range of grid lines (rows for row directions, columns for column
// directions) covered by chunk c of a direction: [lo, hi).
__device__ __forceinline__ void chunk_range(int c, int T_, int L, bool fwd, int &lo, int &hi) {
    if (fwd) {
        lo = c * T_;
        hi = min(L, lo + T_);
    } else {
        hi = L - c * T_;
        lo = max(0, hi - T_);
    }
}

template <typename T, int R, bool YG>
__global__ void __launch_bounds__(kFusedThreads)
prop2d_fused_kernel(const FusedParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    constexpr int es = sizeof(T);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int d = warp;
    const bool active = (p.dirs >> d) & 1;
    const bool rowdir = d < 2;
    const bool fwd = (d & 1) == 0;
    const int H = p.H, W = p.W;
    const int L = rowdir ? H : W;   // lines swept
    const int M = rowdir ? W : H;   // positions per line
    const int T_ = rowdir ? p.t_row : p.t_col;
    const int slot = rowdir ? p.slot_row : p.slot_col;
    const int ring_off = d == 0 ? p.ring_off[0] : d == 1 ? p.ring_off[1]
                       : d == 2 ? p.ring_off[2] : p.ring_off[3];
    unsigned char *ring = smem + (active ? ring_off : 0);
    float *ys = reinterpret_cast<float *>(smem);   // output band (fp32), when !YG
    const int YP = p.y_pitch;

    // zero the output band once; later items re-zero it after writing it out
    if (!YG) {
        for (int e = threadIdx.x; e < p.band_rows * YP; e += kFusedThreads) ys[e] = 0.0f;
    }
    __syncthreads();

    const int n_my = blockIdx.x < p.n_items
                         ? (p.n_items - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int nch = (L + T_ - 1) / T_;
    const int total = active ? n_my * nch : 0;

    // Issue the copies of global chunk g (item g / nch, chunk g % nch) into stage g % kStages.
    auto issue = [&](int g) {
        const int k = g / nch, c = g - k * nch;
        const int item = blockIdx.x + k * gridDim.x;
        const int plane = item / p.bands;
        const int b = plane / p.Cc, ch = plane - b * p.Cc;
        const PlaneOffsets o = plane_offsets(p, b, ch, d);
        int lo, hi;
        chunk_range(c, T_, L, fwd, lo, hi);
        unsigned char *st = ring + (g % kStages) * kTensors * slot;
        if (rowdir) {
            const int nbytes = (hi - lo) * W * es;
            for (int t = 0; t < kTensors; ++t) {
                const char *src = tensor_plane<T>(p, o, t) + static_cast<size_t>(lo) * W * es;
                const uint32_t dst = smem_u32(st + t * slot) +
                                     static_cast<uint32_t>(reinterpret_cast<uintptr_t>(src) & 15);
                warp_copy_words(dst, src, nbytes, lane);
            }
        } else {
            const int nw = ((hi - lo) * es) >> 2;           // words in this chunk's row segments
            const int wpr = p.words_col;                     // power of two, >= nw
            const int w = lane & (wpr - 1);
            const int i0 = lane / wpr, istep = 32 / wpr;
            if (w < nw) {
                for (int t = 0; t < kTensors; ++t) {
                    const char *base = tensor_plane<T>(p, o, t) + static_cast<size_t>(lo) * es;
                    const uint32_t sbase = smem_u32(st + t * slot);
                    for (int i = i0; i < H; i += istep) {
                        const int rw = i * p.pw_col + ((R % 2 == 0) ? (i >> 5) : 0);
                        cp_async_4(sbase + 4u * (rw + w),
                                   base + static_cast<size_t>(i) * W * es + 4 * w);
                    }
                }
            }
        }
    };

    for (int s = 0; s < kStages - 1; ++s) {
        if (s < total) issue(s);
        cp_async_commit();
    }

    int g = 0;
    for (int k = 0; k < n_my; ++k) {
        const int item = blockIdx.x + k * gridDim.x;
        const int plane = item / p.bands;
        const int band = item - plane * p.bands;
        const int band_lo = band * p.band_rows;
        const int band_hi = min(H, band_lo + p.band_rows);
        const int b = plane / p.Cc, ch = plane - b * p.Cc;
        float *yg = nullptr;
        if (YG) {
            // accumulate straight into the fp32 output plane: zero it first
            yg = reinterpret_cast<float *>(p.out) + (static_cast<size_t>(b) * p.Cc + ch) * H * W;
            for (int e = threadIdx.x; e < H * W; e += kFusedThreads) yg[e] = 0.0f;
            __syncthreads();
        }

        if (active) {
            float h[R];
#pragma unroll
            for (int r = 0; r < R; ++r) h[r] = 0.0f;
            const PlaneOffsets o = plane_offsets(p, b, ch, d);

            for (int c = 0; c < nch; ++c, ++g) {
                cp_async_wait<kStages - 2>();
                __syncwarp();
                if (g + kStages - 1 < total) issue(g + kStages - 1);
                cp_async_commit();

                int lo, hi;
                chunk_range(c, T_, L, fwd, lo, hi);
                const unsigned char *st = ring + (g % kStages) * kTensors * slot;
                // where each tensor's data starts in its slot
                const unsigned char *tp[kTensors];
#pragma unroll
                for (int t = 0; t < kTensors; ++t) {
                    if (rowdir) {
                        const char *src = tensor_plane<T>(p, o, t) + static_cast<size_t>(lo) * W * es;
                        tp[t] = st + t * slot + (reinterpret_cast<uintptr_t>(src) & 15);
                    } else {
                        tp[t] = st + t * slot;
                    }
                }
                const int nl = hi - lo;
                for (int tt = 0; tt < nl; ++tt) {
                    const int line = fwd ? lo + tt : hi - 1 - tt;   // grid row / column
                    const int li = line - lo;                         // line within the chunk
                    float z0[R], z1[R], z2[R], la[R], uu[R], xx[R];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const int q = lane * R + r;
                        if (q < M) {
                            int off;   // element offset within the staged tensor
                            if (rowdir) {
                                off = li * W + q;
                            } else {
                                const int rw = q * p.pw_col + ((R % 2 == 0) ? (q >> 5) : 0);
                                off = rw * (4 / es) + li;
                            }
                            la[r] = to_f(reinterpret_cast<const T *>(tp[0])[off]);
                            uu[r] = to_f(reinterpret_cast<const T *>(tp[1])[off]);
                            z0[r] = to_f(reinterpret_cast<const T *>(tp[2])[off]);
                            z1[r] = to_f(reinterpret_cast<const T *>(tp[3])[off]);
                            z2[r] = to_f(reinterpret_cast<const T *>(tp[4])[off]);
                            xx[r] = to_f(reinterpret_cast<const T *>(tp[5])[off]);
                        } else {
                            la[r] = uu[r] = z0[r] = z1[r] = z2[r] = xx[r] = 0.0f;
                        }
                    }
                    W3 w[R];
                    bool ok = true;
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const int q = lane * R + r;
                        const bool f = normalise_fast(z0[r], z1[r], z2[r], q > 0, q + 1 < M, w[r]);
                        ok = ok && (f || q >= M);
                    }
                    if (!__all_sync(0xffffffffu, ok)) {
#pragma unroll
                        for (int r = 0; r < R; ++r) {
                            const int q = lane * R + r;
                            if (q < M)
                                w[r] = normalise_plain(z0[r], z1[r], z2[r], q > 0, q + 1 < M);
                        }
                    }
                    float hl = __shfl_up_sync(0xffffffffu, h[R - 1], 1);
                    float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
                    if (lane == 0) hl = 0.0f;
                    if (lane == 31) hr = 0.0f;
                    float hn[R];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const int q = lane * R + r;
                        const float left = r > 0 ? h[r - 1] : hl;
                        const float right = r < R - 1 ? h[r + 1] : hr;
                        float acc = la[r] * xx[r];
                        acc = fmaf(w[r].w0, left, acc);
                        acc = fmaf(w[r].w1, h[r], acc);
                        acc = fmaf(w[r].w2, right, acc);
                        hn[r] = q < M ? acc : 0.0f;
                    }
#pragma unroll
                    for (int r = 0; r < R; ++r) h[r] = hn[r];
                    // gate and accumulate y += u * h
                    if (rowdir) {
                        if (YG) {
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                const int q = lane * R + r;
                                if (q < M) atomicAdd(yg + static_cast<size_t>(line) * W + q, uu[r] * hn[r]);
                            }
                        } else if (line >= band_lo && line < band_hi) {
                            float *yrow = ys + (line - band_lo) * YP;
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                const int q = lane * R + r;
                                if (q < M) atomicAdd(yrow + q, uu[r] * hn[r]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int r = 0; r < R; ++r) {
                            const int q = lane * R + r;
                            if (YG) {
                                if (q < M) atomicAdd(yg + static_cast<size_t>(q) * W + line, uu[r] * hn[r]);
                            } else if (q >= band_lo && q < band_hi) {
                                atomicAdd(ys + (q - band_lo) * YP + line, uu[r] * hn[r]);
                            }
                        }
                    }
                }
            }
        }
        __syncthreads();
        if (!YG) {
            T *outp = static_cast<T *>(p.out) + (static_cast<size_t>(b) * p.Cc + ch) * H * W +
                      static_cast<size_t>(band_lo) * W;
            const int n = (band_hi - band_lo) * W;
            for (int e = threadIdx.x; e < n; e += kFusedThreads) {
                const int i = e / W, j = e - i * W;
                outp[e] = from_f<T>(ys[i * YP + j]);
                ys[i * YP + j] = 0.0f;
            }
            __syncthreads();
        }
    }
    cp_async_wait<0>();
}

}  // namespace gspn
