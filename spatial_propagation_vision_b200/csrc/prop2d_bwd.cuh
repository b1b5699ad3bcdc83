// Backward of Prop2D: the vector-Jacobian product of the forward recurrence
// and normalisation ("Scaling Parallel Sequence Models to Foundation-Scale
// Vision Encoders", Sec. 6.1 "Scaling with input size, batch, and channels",
// Fig. 8 reports the backward kernel's timings; the backward itself is the
// chain rule of Sec. 3 "Line-scan recurrence" and Sec. 5.1 "Fused CUDA
// normalization").
//
// Given gy = dL/dy, for every (batch, channel, enabled direction):
//
//     g_l       = u_l gy_l + W_{l+1}^T g_{l+1}          (adjoint, reverse scan order)
//     du_l      = gy_l h_l
//     dlambda_l = g_l x_l,      dx_l += g_l lambda_l
//     dw_l(q,k) = g_l(q) h_{l-1}(q+k-1)
//     dz_j      = ds_j s_j (1 - s_j),   ds_j = (dw_j - sum_k dw_k w_k) / S
//                 (S = sum of the on-grid sigmoids; dw_j / eps when the clamp
//                 holds the denominator at eps)
//
// One CTA of four warps owns one (batch, channel) plane; warp d runs
// direction d.  Lane l holds positions l*R .. l*R + R - 1 of a line.  The
// forward lines are recomputed: a first sweep keeps h at every kSeg-th line
// (checkpoints) in shared memory; the reverse sweep then replays each
// segment of kSeg lines from its checkpoint into a segment buffer and walks
// it backwards.  Shared memory per warp: (L / kSeg + kSeg + 1) lines.
// Weights are recomputed in the plain form (sigmoid, local sum, clamp,
// divide) in fp32 in both sweeps.  Every sweep loads the next line's inputs
// one step ahead, into registers, so that a step does not wait for its own
// loads (two lines ahead measured slower).  Gradients are fp32: dlambda, du and (per
// channel) dwlogit are stored once; dx adds the four directions with global
// fp32 atomics, and shared inputs add over their uses likewise (lambda and u
// shared by the four directions: their gradients add over the directions;
// a logit field shared by a group of channels: over the channels)
// likewise, into buffers the host zeroed.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace gspn {

constexpr int kBwdThreads = 128;   // warp d runs direction d
constexpr int kBwdSeg = 16;        // lines per recomputed segment

struct BwdParams {
    const void *x, *lam, *wl, *u, *gy;
    float *dx, *dlam, *dwl, *du;
    int B, Cc, H, W, dirs;
    int gate_dirs;          // direction slots of lambda and u: 4, or 1 shared by all directions
    int w_groups, w_cpg;    // logit fields per (batch, direction) and channels per field
    int R;            // positions per lane (line capacity 32 R >= max(H, W))
    int n_ckpt;       // checkpoint lines per warp (ceil(maxL / kBwdSeg))
    int warp_floats;  // shared-memory floats per warp
};

template <typename T> __device__ __forceinline__ float bwd_in(const T *p, size_t i);
template <> __device__ __forceinline__ float bwd_in<float>(const float *p, size_t i) { return __ldg(p + i); }
template <> __device__ __forceinline__ float bwd_in<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

// sigmoid in fp32 (hardware 2^x and reciprocal), saturating to 0 or 1
__device__ __forceinline__ float bwd_sigmoid(float z) {
    return rcp(1.0f + ex2(z * -1.4426950408889634f));
}

// Inputs of a lane's R positions of one line: the three logit slots,
// lambda, x, and (reverse sweep) u and the output gradient.
template <int R>
struct BwdIn {
    float z[3][R], lam[R], x[R], u[R], gy[R];
};

template <typename T, int R>
struct BwdLine {
    const BwdParams &p;
    const int lane, d;
    const bool fwd, rows;
    const int L, M;
    const int lstride;                 // elements between consecutive lines: W (rows) or 1 (columns)
    const bool gate_shared, w_shared;  // lambda/u shared by the directions; logits by channels
    int qo_[R];           // element offset of position lane R + r within a line (clamped to M - 1)
    bool valid_[R];       // lane R + r < M
    bool on0_[R], on2_[R];    // the slot k = 0 / k = 2 neighbour is on the line (valid positions)
    const T *x, *lam, *u, *gy, *wl0, *wl1, *wl2;   // this plane's tensors (direction d)
    float *dx, *dlam, *du, *dwl0, *dwl1, *dwl2;

    __device__ BwdLine(const BwdParams &p_, int lane_, int d_, int b, int c)
        : p(p_), lane(lane_), d(d_), fwd((d_ & 1) == 0), rows(d_ < 2),
          L(d_ < 2 ? p_.H : p_.W), M(d_ < 2 ? p_.W : p_.H), lstride(d_ < 2 ? p_.W : 1),
          gate_shared(p_.gate_dirs == 1), w_shared(p_.w_cpg > 1) {
        const size_t HW = static_cast<size_t>(p.H) * p.W;
        const size_t xo = (static_cast<size_t>(b) * p.Cc + c) * HW;
        const size_t go = ((static_cast<size_t>(b) * p.gate_dirs + (p.gate_dirs == 4 ? d : 0)) * p.Cc + c) * HW;
        const size_t wo = (((static_cast<size_t>(b) * 4 + d) * p.w_groups + c / p.w_cpg) * 3) * HW;
        x = static_cast<const T *>(p.x) + xo;
        gy = static_cast<const T *>(p.gy) + xo;
        lam = static_cast<const T *>(p.lam) + go;
        u = static_cast<const T *>(p.u) + go;
        wl0 = static_cast<const T *>(p.wl) + wo;
        wl1 = wl0 + HW;
        wl2 = wl1 + HW;
        dx = p.dx + xo;
        dlam = p.dlam + go;
        du = p.du + go;
        dwl0 = p.dwl + wo;
        dwl1 = dwl0 + HW;
        dwl2 = dwl1 + HW;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = lane * R + r;
            const int qc = min(q, M - 1);
            qo_[r] = rows ? qc : qc * p.W;
            valid_[r] = q < M;
            on0_[r] = q < M && q > 0;
            on2_[r] = q + 1 < M;
        }
    }
    __device__ __forceinline__ int qo(int r) const { return qo_[r]; }
    __device__ __forceinline__ bool valid(int r) const { return valid_[r]; }
    __device__ __forceinline__ bool on0(int r) const { return on0_[r]; }
    __device__ __forceinline__ bool on2(int r) const { return on2_[r]; }

    // element offset of scan line s's first position within the plane
    // (plane offsets fit 32 bits: H W <= 2^30)
    __device__ __forceinline__ int loff(int s) const { return (fwd ? s : L - 1 - s) * lstride; }

    // Inputs of line s (positions past the line's end read position M-1:
    // finite, never used; off-grid logit slots are read but never used).
    template <bool REV>
    __device__ __forceinline__ void load_in(int s, BwdIn<R> &in) const {
        const int lo = loff(s);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int e = lo + qo(r);
            in.z[0][r] = bwd_in(wl0, e);
            in.z[1][r] = bwd_in(wl1, e);
            in.z[2][r] = bwd_in(wl2, e);
            in.lam[r] = bwd_in(lam, e);
            in.x[r] = bwd_in(x, e);
            if (REV) {
                in.u[r] = bwd_in(u, e);
                in.gy[r] = bwd_in(gy, e);
            }
        }
    }

    // normalised weights (w), sigmoids (s), local sum (S) and the
    // reciprocal of the clamped sum (rs = 1 / max(S, eps), hardware
    // reciprocal) of the lane's position r; off-grid slots are selected away
    __device__ __forceinline__ void weights(const BwdIn<R> &in, int r, float (&s)[3], float (&w)[3],
                                            float &S, float &rs) const {
        s[0] = on0(r) ? bwd_sigmoid(in.z[0][r]) : 0.f;
        s[1] = valid(r) ? bwd_sigmoid(in.z[1][r]) : 0.f;
        s[2] = on2(r) ? bwd_sigmoid(in.z[2][r]) : 0.f;
        S = (s[0] + s[1]) + s[2];
        rs = rcp(fmaxf(S, 1e-6f));
#pragma unroll
        for (int k = 0; k < 3; ++k) w[k] = s[k] * rs;
    }

    // one forward step: h <- W h + lambda x (positions past the end stay 0)
    __device__ __forceinline__ void fwd_step(const BwdIn<R> &in, float (&h)[R]) const {
        const float hl = __shfl_up_sync(0xffffffffu, h[R - 1], 1);
        const float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
        float hn[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float sg[3], w[3], S, rs;
            weights(in, r, sg, w, S, rs);
            const float left = r > 0 ? h[r > 0 ? r - 1 : 0] : (lane > 0 ? hl : 0.f);
            const float right = r + 1 < R ? h[r + 1 < R ? r + 1 : r] : hr;
            const float v = w[0] * left + w[1] * h[r] + w[2] * right + in.lam[r] * in.x[r];
            hn[r] = valid(r) ? v : 0.f;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) h[r] = hn[r];
    }

    // steps [s0, s1) forwards from h, storing h after step s into
    // out(s); the next line's inputs load one step ahead
    template <typename Out>
    __device__ __forceinline__ void sweep(int s0, int s1, float (&h)[R], Out out) const {
        BwdIn<R> a, b;
        load_in<false>(s0, a);
        for (int s = s0; s < s1; s += 2) {
            if (s + 1 < s1) load_in<false>(s + 1, b);
            fwd_step(a, h);
            out(s, h);
            if (s + 1 >= s1) break;
            if (s + 2 < s1) load_in<false>(s + 2, a);
            fwd_step(b, h);
            out(s + 1, h);
        }
    }

    __device__ __forceinline__ void store_line(float *buf, const float (&h)[R]) const {
#pragma unroll
        for (int r = 0; r < R; ++r) buf[lane * R + r] = h[r];
    }
    __device__ __forceinline__ void load_line(const float *buf, float (&h)[R]) const {
#pragma unroll
        for (int r = 0; r < R; ++r) h[r] = buf[lane * R + r];
    }

    // The reverse step s (adjoint of line s): gradients of line s's inputs,
    // the carry into line s-1.  hcur / hprv: h after steps s and s-1.
    __device__ __forceinline__ void rev_step(int s, const BwdIn<R> &in, const float *hcur, const float *hprv,
                                             float (&carry)[R]) const {
        const int lo = loff(s);
        float cl = 0.f, cr = 0.f, cmid[R];
#pragma unroll
        for (int r = 0; r < R; ++r) cmid[r] = 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = lane * R + r;
            const int e = lo + qo(r);
            const float gyv = in.gy[r];
            // positions past the line's end take no adjoint: they pass nothing on
            const float a = valid(r) ? in.u[r] * gyv + carry[r] : 0.f;
            if (valid(r)) {
                if (gate_shared) {
                    atomicAdd(du + e, gyv * hcur[q]);
                    atomicAdd(dlam + e, a * in.x[r]);
                } else {
                    du[e] = gyv * hcur[q];
                    dlam[e] = a * in.x[r];
                }
                atomicAdd(dx + e, a * in.lam[r]);
            }
            float sgm[3], w[3], S, rs;
            weights(in, r, sgm, w, S, rs);
            // dw_k = a h_{s-1}(q + k - 1) for on-grid slots (line 0 has no predecessor)
            float hp[3] = {0.f, 0.f, 0.f};
            if (s > 0) {
                if (on0(r)) hp[0] = hprv[q - 1 >= 0 ? q - 1 : 0];
                if (valid(r)) hp[1] = hprv[q];
                if (on2(r)) hp[2] = hprv[q + 1];
            }
            float dw[3], dot = 0.f;
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                dw[k] = a * hp[k];
                dot += dw[k] * w[k];
            }
            const bool on[3] = {on0(r), valid(r), on2(r)};
            float *const dwk[3] = {dwl0, dwl1, dwl2};
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                // (dw_j - sum_k dw_k w_k) / S, or dw_j / eps where the clamp holds
                const float ds = (S > 1e-6f ? dw[k] - dot : dw[k]) * rs;
                const float dz = ds * sgm[k] * (1.f - sgm[k]);
                if (on[k]) {
                    if (w_shared) atomicAdd(dwk[k] + e, dz);
                    else dwk[k][e] = dz;
                }
            }
            // transposed stencil: position q passes w_k a to q + k - 1
            const float c0 = w[0] * a, c1 = w[1] * a, c2 = w[2] * a;
            cmid[r] += c1;
            if (r > 0) cmid[r - 1 > 0 ? r - 1 : 0] += c0;
            else cl = c0;
            if (r + 1 < R) cmid[r + 1 < R ? r + 1 : r] += c2;
            else cr = c2;
        }
        // contributions that cross lanes
        const float from_right = __shfl_down_sync(0xffffffffu, cl, 1);   // lane+1's position 0 -> my last
        const float from_left = __shfl_up_sync(0xffffffffu, cr, 1);      // lane-1's last -> my first
#pragma unroll
        for (int r = 0; r < R; ++r) carry[r] = cmid[r];
        if (lane < 31) carry[R - 1] += from_right;
        if (lane > 0) carry[0] += from_left;
    }

    // The whole backward of this direction.  `ck`: checkpoint lines
    // (line i holds h after step i * kSeg + kSeg - 1), `seg`: kSeg + 1 lines
    // (line 0: h before the segment, line 1 + t: after its step t).
    __device__ void run(float *ck, float *seg) const {
        const int line_f = 32 * R;
        float h[R];
#pragma unroll
        for (int r = 0; r < R; ++r) h[r] = 0.f;
        // forward sweep: checkpoints at the end of every segment
        sweep(0, L, h, [&](int s, const float (&hh)[R]) {
            if (s % kBwdSeg == kBwdSeg - 1) store_line(ck + (s / kBwdSeg) * line_f, hh);
        });
        __syncwarp();
        float carry[R];
#pragma unroll
        for (int r = 0; r < R; ++r) carry[r] = 0.f;
        const int nseg = (L + kBwdSeg - 1) / kBwdSeg;
        for (int sg = nseg - 1; sg >= 0; --sg) {
            const int s0 = sg * kBwdSeg, s1 = min(L, s0 + kBwdSeg);
            // replay the segment: seg[0] = h before step s0, seg[1 + t] after step s0 + t
            if (sg == 0) {
#pragma unroll
                for (int r = 0; r < R; ++r) h[r] = 0.f;
            } else {
                load_line(ck + (sg - 1) * line_f, h);
            }
            store_line(seg, h);
            sweep(s0, s1, h, [&](int s, const float (&hh)[R]) { store_line(seg + (s - s0 + 1) * line_f, hh); });
            __syncwarp();
            // reverse steps of the segment, the inputs of line s-1 loaded
            // while line s is processed
            BwdIn<R> a, b;
            load_in<true>(s1 - 1, a);
            for (int s = s1 - 1; s >= s0; s -= 2) {
                if (s - 1 >= s0) load_in<true>(s - 1, b);
                rev_step(s, a, seg + (s - s0 + 1) * line_f, seg + (s - s0) * line_f, carry);
                if (s - 1 < s0) break;
                if (s - 2 >= s0) load_in<true>(s - 2, a);
                rev_step(s - 1, b, seg + (s - s0) * line_f, seg + (s - 1 - s0) * line_f, carry);
            }
            __syncwarp();
        }
    }
};

template <typename T, int R>
__global__ void __launch_bounds__(kBwdThreads) prop2d_bwd_kernel(const BwdParams p) {
    extern __shared__ __align__(16) float bsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (!((p.dirs >> warp) & 1)) return;
    float *ck = bsm + warp * p.warp_floats;
    float *seg = ck + p.n_ckpt * 32 * R;
    for (int plane = blockIdx.x; plane < p.B * p.Cc; plane += gridDim.x) {
        const int b = plane / p.Cc, c = plane - b * p.Cc;
        BwdLine<T, R> ln(p, lane, warp, b, c);
        ln.run(ck, seg);
        __syncwarp();
    }
}

}  // namespace gspn
