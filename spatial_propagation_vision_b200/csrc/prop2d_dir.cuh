// Fused Prop2D forward, one warp per direction.
//
// One CTA of four warps owns one (batch, channel) plane (or one band of its
// output rows when the fp32 output plane does not fit in shared memory);
// warp d runs direction d: 0 top->bottom, 1 bottom->top (row lines),
// 2 left->right, 3 right->left (column lines).  Lane l holds the R
// consecutive positions q = l*R + r of the current line in registers; the
// neighbours across lanes come from shuffles.  Four independent warps per
// plane give the scheduler enough warps to hide the latency of the
// dependent arithmetic (the kernel is bound by instruction issue, not by
// memory), and pairs of positions share packed f32x2 instructions.
//
// Normalisation (Sec. 5.1 "Fused CUDA normalization": sigmoid, local sum,
// clamp, divide), folded into the update.  With a_k = 1 + exp(-z_k),
// sigmoid(z_k) = 1 / a_k and, for P_k = product of a_j over the other
// on-grid slots j != k and D = sum_k P_k,
//     h = sum_k w_k h_prev(q+k-1) + lambda x = (sum_k P_k h_prev(q+k-1)) / D + lambda x,
// which takes three exponentials and one reciprocal per position.  An
// off-grid slot takes a_k = 1, P_k = 0.  Whenever the clamp of the
// denominator could bind, or a product overflows, D exceeds a threshold
// (1e11 with three on-grid slots, 1e5 with two) or is not finite, and the
// line is recomputed in the plain form.  The weights of line s+1 do not
// depend on the hidden line; they are computed in the same straight block
// as line s's recurrence so the two chains interleave.
//
// Input lines are staged in shared memory, several lines per chunk, in a
// two-stage ring per warp:
//   * row lines: the rows of a chunk are one contiguous span per tensor;
//     lane t < 6 moves tensor t's span with one bulk copy (TMA engine) into a
//     16-byte aligned slot and arrives on the stage's mbarrier;
//   * column lines: a strip of 16 bytes of every row (8 bf16 / 4 fp32
//     columns) moved by the lanes with 4-byte cp.async; a strip row takes 4
//     words, XOR-swizzled by row so that the lanes reading one column hit
//     distinct banks (odd R), or 5 words plus one word per lane (even R).
// The gated outputs u * h of the four directions are summed into one fp32
// plane in shared memory with shared-memory atomics and written once.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace gspn {

constexpr int kDirThreads = 128;   // warp d runs direction d
constexpr int kDirStages = 2;      // ring depth per warp
constexpr int kColWords = 4;       // 16 bytes of each row per column chunk
constexpr int kTensors = 6;        // lambda, u, logit0, logit1, logit2, x

// Output modes.
constexpr int kYSmem = 0;     // whole fp32 output plane in shared memory
constexpr int kYBanded = 1;   // a band of output rows in shared memory, scans rerun per band
constexpr int kYGlobal = 2;   // fp32 output accumulated in global memory (L2 atomics)

struct DirParams {
    const void *x, *lam, *wl, *u;
    void *out;
    int B, Cc, H, W, dirs, share_w;
    int n_items, bands, band_rows;
    int t_row;                  // rows per row-line chunk
    int slot_row, slot_col;     // bytes per tensor slot of a row / column ring stage
    int ring[4];                // byte offset of direction d's ring (-1: direction off)
    int bar_off;                // byte offset of the mbarriers and shift tables (256 bytes)
    int y_pitch;                // floats per staged output row (odd)
    unsigned long long end_x, end_gate, end_wl;   // byte sizes of x, lambda/u, logits
};

// Column-strip geometry: word address (relative to its slot) of word w of
// strip row q.
template <int R>
struct ColLayout {
    static constexpr bool kSwizzle = (R % 2) == 1;
    static __device__ __forceinline__ int word(int q, int w) {
        if (kSwizzle) return q * 4 + (w ^ ((q / (8 * R)) & 3));
        return q * 5 + q / R + w;
    }
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T> __device__ __forceinline__ float sload(const unsigned char *p);
template <> __device__ __forceinline__ float sload<float>(const unsigned char *p) {
    return *reinterpret_cast<const float *>(p);
}
template <> __device__ __forceinline__ float sload<__nv_bfloat16>(const unsigned char *p) {
    return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const unsigned short *>(p)) << 16);
}

// Element offset of plane (b, c) of tensor t for direction d.
__device__ __forceinline__ size_t dir_plane(const DirParams &p, int b, int c, int d, int t) {
    const size_t HW = static_cast<size_t>(p.H) * p.W;
    if (t == 5) return (static_cast<size_t>(b) * p.Cc + c) * HW;
    if (t < 2) return ((static_cast<size_t>(b) * 4 + d) * p.Cc + c) * HW;
    const int Cw = p.share_w ? 1 : p.Cc;
    return ((((static_cast<size_t>(b) * 4 + d) * Cw + (p.share_w ? 0 : c)) * 3) + (t - 2)) * HW;
}

__device__ __forceinline__ const char *dir_tensor(const DirParams &p, int t) {
    const void *base = t == 0 ? p.lam : t == 1 ? p.u : t == 5 ? p.x : p.wl;
    return static_cast<const char *>(base);
}

__device__ __forceinline__ unsigned long long dir_tensor_bytes(const DirParams &p, int t) {
    return t == 5 ? p.end_x : t < 2 ? p.end_gate : p.end_wl;
}

// Per-line normalisation terms and gates of the lane's R positions.
template <int R>
struct LineW {
    float P0[R], P1[R], P2[R], rD[R], bx[R], uu[R];
    bool bad;   // some position needs the plain form
};

template <typename T, int R, bool ROW, int MODE>
struct DirWarp {
    static constexpr int es = sizeof(T);
    static constexpr int NS = kDirStages;
    static constexpr int kColRows = (32 * R + 32 / kColWords - 1) / (32 / kColWords);  // strip rows per lane

    const DirParams &p;
    const int lane;
    const int D;                    // direction slot (0..3)
    const bool fwd;                 // sweeps forward (top->bottom / left->right)
    unsigned char *const ring;
    const uint32_t bars;            // this warp's NS mbarriers (row lines)
    unsigned char *const shifts;    // this warp's [stage][tensor] span shifts (row lines)
    const int slot;
    const int L, M, T_, nch;
    // source planes of the item whose chunks are being issued
    int issue_item;
    const char *my_gp;              // row lines: lane t < 6 keeps tensor t's plane
    const char *gtab[kTensors];     // column lines: every lane copies every tensor
    int col_off[kColRows];          // strip-row word offsets of this lane's rows (column lines)

    __device__ DirWarp(const DirParams &p_, unsigned char *smem_, int lane_, int d_)
        : p(p_), lane(lane_), D(d_), fwd((d_ % 2) == 0),
          ring(smem_ + (d_ == 0 ? p_.ring[0] : d_ == 1 ? p_.ring[1] : d_ == 2 ? p_.ring[2] : p_.ring[3])),
          bars(smem_u32(smem_ + p_.bar_off) + 8 * NS * D),
          shifts(smem_ + p_.bar_off + 64 + 16 * D),
          slot(ROW ? p_.slot_row : p_.slot_col),
          L(ROW ? p_.H : p_.W), M(ROW ? p_.W : p_.H),
          T_(ROW ? p_.t_row : kColWords * 4 / es),
          nch(((ROW ? p_.H : p_.W) + (ROW ? p_.t_row : kColWords * 4 / es) - 1) /
              (ROW ? p_.t_row : kColWords * 4 / es)),
          issue_item(-1), my_gp(nullptr) {
        if (!ROW) {
            const int w = lane & (kColWords - 1), i0 = lane / kColWords;
#pragma unroll
            for (int k = 0; k < kColRows; ++k) col_off[k] = 4 * ColLayout<R>::word(i0 + k * (32 / kColWords), w);
        }
    }

    // Lines [lo, hi) of chunk c in grid coordinates.
    __device__ __forceinline__ void chunk(int c, int &lo, int &hi) const {
        if (fwd) {
            lo = c * T_;
            hi = min(L, lo + T_);
        } else {
            hi = L - c * T_;
            lo = max(0, hi - T_);
        }
    }

    __device__ __forceinline__ unsigned char *slot_ptr(int stage, int t) const {
        return ring + (stage * kTensors + t) * slot;
    }

    __device__ __forceinline__ void set_issue_item(int item) {
        if (item == issue_item) return;
        issue_item = item;
        const int plane = item / p.bands;
        const int b = plane / p.Cc, ch = plane - b * p.Cc;
        if (ROW) {
            if (lane < kTensors) my_gp = dir_tensor(p, lane) + dir_plane(p, b, ch, D, lane) * es;
        } else {
#pragma unroll
            for (int t = 0; t < kTensors; ++t) gtab[t] = dir_tensor(p, t) + dir_plane(p, b, ch, D, t) * es;
        }
    }

    // Issue the copies of chunk c of `item` into ring stage `stage`.  Every
    // read of that stage has completed: its values were consumed by
    // instructions issued before this point.
    __device__ __forceinline__ void issue(int item, int c, int stage) {
        set_issue_item(item);
        int lo, hi;
        chunk(c, lo, hi);
        if (ROW) {
            if (lane < kTensors) {
                const int t = lane;
                const char *s = my_gp + static_cast<size_t>(lo) * p.W * es;
                const uint32_t sh = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(s) & 15);
                const char *a = s - sh;
                uint32_t n = (sh + static_cast<uint32_t>((hi - lo) * p.W * es) + 15u) & ~15u;
                int tl = 0;
                // never read past the end of the tensor: the last partial 16 bytes
                // are then copied by hand
                const unsigned long long end = dir_tensor_bytes(p, t);
                const unsigned long long off = static_cast<unsigned long long>(a - dir_tensor(p, t));
                if (off + n > end) {
                    tl = static_cast<int>(end - (off + n - 16));
                    n -= 16;
                }
                unsigned char *dst = slot_ptr(stage, t);
                shifts[stage * 8 + t] = static_cast<unsigned char>(sh);
                for (int e = 0; e < tl; e += 2)   // rare: end of the tensor
                    *reinterpret_cast<unsigned short *>(dst + n + e) =
                        *reinterpret_cast<const unsigned short *>(a + n + e);
                const uint32_t bar = bars + 8 * stage;
                mbar_arrive_expect_tx(bar, n);
                if (n) bulk_copy_g2s(smem_u32(dst), a, n, bar);
            }
        } else {
            const int w = lane & (kColWords - 1), i0 = lane / kColWords;
            const int nw = ((hi - lo) * es) >> 2;   // words per row segment, <= kColWords
            if (w < nw) {
                const size_t gstep = static_cast<size_t>(32 / kColWords) * p.W * es;
                const size_t lane_off = (static_cast<size_t>(i0) * p.W + lo) * es + 4 * w;
#pragma unroll
                for (int t = 0; t < kTensors; ++t) {
                    const char *s = gtab[t] + lane_off;
                    const uint32_t sb = smem_u32(slot_ptr(stage, t));
#pragma unroll
                    for (int k = 0; k < kColRows; ++k) {
                        if (i0 + k * (32 / kColWords) < p.H) cp_async_4(sb + col_off[k], s);
                        s += gstep;
                    }
                }
            }
            cp_async_commit();
        }
    }

    // Wait until the g-th chunk of this warp (in `stage`) has landed.
    __device__ __forceinline__ void wait_chunk(int g, int stage) const {
        if (ROW) {
            mbar_wait_bounded(bars + 8 * stage, static_cast<uint32_t>((g / NS) & 1));
        } else {
            cp_async_wait<NS - 2>();
            __syncwarp();
        }
    }

    // Shared-memory address of line li's element at position lane*R + r.
    __device__ __forceinline__ const unsigned char *elem(const unsigned char *slotp, int shift,
                                                         int li, int r) const {
        if (ROW) return slotp + shift + (li * p.W + lane * R + r) * es;
        const int q = lane * R + r;
        return slotp + 4 * ColLayout<R>::word(q, (li * es) >> 2) + ((li * es) & 3);
    }

    // Raw inputs of line li of the current chunk -> normalisation terms.
    __device__ __forceinline__ void weights(const unsigned char *const (&sp)[kTensors],
                                            const int (&shift)[kTensors], int li,
                                            const float (&m0)[R], const float (&m2)[R],
                                            const float (&ithr)[R], const bool (&valid)[R],
                                            LineW<R> &W) const {
        float v[kTensors][R];
#pragma unroll
        for (int t = 0; t < kTensors; ++t)
#pragma unroll
            for (int r = 0; r < R; ++r) v[t][r] = sload<T>(elem(sp[t], shift[t], li, r));
        constexpr float nl2e = -1.4426950408889634f;
        bool bad = false;
        // positions (r, r+1) as one f32x2 pair; a last odd position alone
#pragma unroll
        for (int r = 0; r + 1 < R; r += 2) {
            const float2 n2 = make_float2(nl2e, nl2e);
            const float2 one2 = make_float2(1.0f, 1.0f);
            const float2 t0 = __fmul2_rn(make_float2(v[2][r], v[2][r + 1]), n2);
            const float2 t1 = __fmul2_rn(make_float2(v[3][r], v[3][r + 1]), n2);
            const float2 t2 = __fmul2_rn(make_float2(v[4][r], v[4][r + 1]), n2);
            const float2 a0 = __ffma2_rn(make_float2(ex2(t0.x), ex2(t0.y)), make_float2(m0[r], m0[r + 1]), one2);
            const float2 a1 = __fadd2_rn(make_float2(ex2(t1.x), ex2(t1.y)), one2);
            const float2 a2 = __ffma2_rn(make_float2(ex2(t2.x), ex2(t2.y)), make_float2(m2[r], m2[r + 1]), one2);
            const float2 P0 = __fmul2_rn(__fmul2_rn(a1, a2), make_float2(m0[r], m0[r + 1]));
            const float2 P1 = __fmul2_rn(a0, a2);
            const float2 P2 = __fmul2_rn(__fmul2_rn(a0, a1), make_float2(m2[r], m2[r + 1]));
            const float2 Dn = __fadd2_rn(__fadd2_rn(P0, P1), P2);
            const float2 k = __fmul2_rn(Dn, make_float2(ithr[r], ithr[r + 1]));
            // over the threshold, or NaN (an off-grid slot whose exponential overflowed)
            bad = bad || (valid[r] && !(k.x <= 1.0f)) || (valid[r + 1] && !(k.y <= 1.0f));
            const float2 bx = __fmul2_rn(make_float2(v[0][r], v[0][r + 1]), make_float2(v[5][r], v[5][r + 1]));
            W.P0[r] = P0.x; W.P0[r + 1] = P0.y;
            W.P1[r] = P1.x; W.P1[r + 1] = P1.y;
            W.P2[r] = P2.x; W.P2[r + 1] = P2.y;
            W.rD[r] = rcp(Dn.x); W.rD[r + 1] = rcp(Dn.y);
            W.bx[r] = bx.x; W.bx[r + 1] = bx.y;
            W.uu[r] = v[1][r]; W.uu[r + 1] = v[1][r + 1];
        }
        if (R % 2) {
            const int r = R - 1;
            const float a0 = fmaf(ex2(v[2][r] * nl2e), m0[r], 1.0f);
            const float a1 = ex2(v[3][r] * nl2e) + 1.0f;
            const float a2 = fmaf(ex2(v[4][r] * nl2e), m2[r], 1.0f);
            const float P0 = a1 * a2 * m0[r];
            const float P1 = a0 * a2;
            const float P2 = a0 * a1 * m2[r];
            const float Dn = (P0 + P1) + P2;
            bad = bad || (valid[r] && !(Dn * ithr[r] <= 1.0f));
            W.P0[r] = P0;
            W.P1[r] = P1;
            W.P2[r] = P2;
            W.rD[r] = rcp(Dn);
            W.bx[r] = v[0][r] * v[5][r];
            W.uu[r] = v[1][r];
        }
        W.bad = bad;
    }

    // Plain-form update of line li for every position (rare path).
    __device__ __forceinline__ void plain_line(const unsigned char *const (&sp)[kTensors],
                                               const int (&shift)[kTensors], int li,
                                               const float (&h)[R], float hl, float hr,
                                               float (&hn)[R]) const {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = lane * R + r;
            const float left = r > 0 ? h[r - 1] : hl;
            const float right = r < R - 1 ? h[r + 1] : hr;
            float v[kTensors];
#pragma unroll
            for (int t = 0; t < kTensors; ++t) v[t] = sload<T>(elem(sp[t], shift[t], li, r));
            const W3 w = normalise_plain(v[2], v[3], v[4], q > 0, q + 1 < M);
            float acc = v[0] * v[5];
            if (q > 0) acc = fmaf(w.w0, left, acc);
            acc = fmaf(w.w1, h[r], acc);
            if (q + 1 < M) acc = fmaf(w.w2, right, acc);
            hn[r] = acc;
        }
    }

    // Run every line of `item`.  `g` counts this warp's chunks in the launch
    // (ring position); `total` is the number of chunks it runs in the launch.
    __device__ void run_item(int item, int &g, int total, float *ys, float *yg, int band_lo,
                             int band_hi) {
        float m0[R], m2[R], ithr[R];
        bool valid[R], inband[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = lane * R + r;
            valid[r] = q < M;
            m0[r] = q > 0 ? 1.0f : 0.0f;
            m2[r] = q + 1 < M ? 1.0f : 0.0f;
            ithr[r] = (q > 0 && q + 1 < M) ? 1e-11f : 1e-5f;
            inband[r] = valid[r] && (ROW || MODE != kYBanded || (q >= band_lo && q < band_hi));
        }
        const uint32_t ysa = smem_u32(ys);
        float hs[R];
#pragma unroll
        for (int r = 0; r < R; ++r) hs[r] = 0.0f;

        const unsigned char *sp[kTensors];
        int shift[kTensors];
        int lo = 0, nl = 0;
        auto enter_chunk = [&](int c) {
            const int stage = g % NS;
            wait_chunk(g, stage);
            if (g + NS - 1 < total) {
                const int gn = g + NS - 1;
                const int kk = gn / nch;
                issue(blockIdx.x + kk * gridDim.x, gn - kk * nch, gn % NS);
            } else if (!ROW) {
                cp_async_commit();
            }
            int hi;
            chunk(c, lo, hi);
            nl = hi - lo;
#pragma unroll
            for (int t = 0; t < kTensors; ++t) {
                sp[t] = slot_ptr(stage, t);
                shift[t] = ROW ? shifts[stage * 8 + t] : 0;
            }
        };

        // Iteration s (from -1) finishes line s and prepares line s+1: the
        // rare plain form of line s, the chunk change, then one straight block
        // with the weights of line s+1 and the recurrence of line s, then the
        // outputs of line s.  tt is the scan-order index of line s in its chunk.
        int c = 0, tt = -1;
        enter_chunk(0);
        LineW<R> Wc;
        Wc.bad = false;
        int cur = 0;
#pragma unroll 1
        for (int s = -1; s < L; ++s) {
            float hl = __shfl_up_sync(0xffffffffu, hs[R - 1], 1);
            float hr = __shfl_down_sync(0xffffffffu, hs[0], 1);
            float hp[R];
            const bool plain = s >= 0 && __any_sync(0xffffffffu, Wc.bad);
            if (plain) plain_line(sp, shift, fwd ? tt : nl - 1 - tt, hs, hl, hr, hp);
            int tt1 = tt + 1;
            if (s + 1 < L && tt1 == nl) {
                ++g;
                ++c;
                tt1 = 0;
                enter_chunk(c);
            }
            LineW<R> Wn;
            weights(sp, shift, fwd ? tt1 : nl - 1 - tt1, m0, m2, ithr, valid, Wn);
            float hn[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float left = r > 0 ? hs[r - 1] : hl;
                const float right = r < R - 1 ? hs[r + 1] : hr;
                float N = Wc.P0[r] * left;
                N = fmaf(Wc.P1[r], hs[r], N);
                N = fmaf(Wc.P2[r], right, N);
                hn[r] = fmaf(N, Wc.rD[r], Wc.bx[r]);
                if (plain) hn[r] = hp[r];
            }
            float uu[R];
#pragma unroll
            for (int r = 0; r < R; ++r) uu[r] = Wc.uu[r];
            const int line = cur;   // grid line of step s
            Wc = Wn;
            tt = tt1;
            cur = fwd ? lo + tt : lo + nl - 1 - tt;
            if (s < 0) continue;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                hs[r] = valid[r] ? hn[r] : 0.0f;
                const float cy = uu[r] * hs[r];
                const int q = lane * R + r;
                if (MODE == kYGlobal) {
                    if (valid[r]) {
                        if (ROW) atomicAdd(yg + static_cast<size_t>(line) * p.W + q, cy);
                        else atomicAdd(yg + static_cast<size_t>(q) * p.W + line, cy);
                    }
                } else if (ROW) {
                    const bool in = MODE != kYBanded || (line >= band_lo && line < band_hi);
                    red_add_shared_if(ysa + 4u * ((line - band_lo) * p.y_pitch + q), cy, valid[r] && in);
                } else {
                    red_add_shared_if(ysa + 4u * ((q - band_lo) * p.y_pitch + line), cy, inband[r]);
                }
            }
        }
        ++g;   // the last chunk of the item is done
    }
};

// Barrier of the CTA's four warps.  The warps run different code paths (one
// per direction), so the barrier is a named PTX barrier with an explicit
// thread count rather than __syncthreads.
__device__ __forceinline__ void dir_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(kDirThreads) : "memory");
}

// The whole kernel seen from the warp that runs direction D (row lines when
// ROW); only that orientation's state is live in its registers, and the two
// directions of an orientation share one code path.
template <typename T, int R, bool ROW, int MODE>
__device__ __forceinline__ void dir_role(const DirParams &p, unsigned char *smem, int warp, int lane, int D) {
    float *ys = reinterpret_cast<float *>(smem);   // output plane or band, fp32 [rows][y_pitch]
    const int YP = p.y_pitch;
    const bool active = (p.dirs >> D) & 1;
    const int n_my = blockIdx.x < p.n_items ? (p.n_items - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    DirWarp<T, R, ROW, MODE> w(p, smem, lane, D);
    constexpr int NS = kDirStages;
    const int total = active ? n_my * w.nch : 0;
    for (int s = 0; s < NS - 1; ++s) {
        if (s < total) w.issue(blockIdx.x, s, s);
        else if (!ROW) cp_async_commit();
    }

    int g = 0;
    for (int k = 0; k < n_my; ++k) {
        const int item = blockIdx.x + k * gridDim.x;
        const int plane = item / p.bands;
        const int band = item - plane * p.bands;
        const int band_lo = band * p.band_rows;
        const int band_hi = min(p.H, band_lo + p.band_rows);
        float *yg = nullptr;
        if (MODE == kYGlobal) {
            yg = reinterpret_cast<float *>(p.out) + static_cast<size_t>(plane) * p.H * p.W;
            for (int e = threadIdx.x; e < p.H * p.W; e += kDirThreads) yg[e] = 0.0f;
            dir_barrier();
        }
        if (active) w.run_item(item, g, total, ys, yg, band_lo, band_hi);
        dir_barrier();
        if (MODE != kYGlobal) {
            // write the band out once (converted) and clear it for the next item
            T *outp = static_cast<T *>(p.out) + static_cast<size_t>(plane) * p.H * p.W +
                      static_cast<size_t>(band_lo) * p.W;
            for (int i = warp; i < band_hi - band_lo; i += 4) {
                float *yrow = ys + i * YP;
                T *orow = outp + static_cast<size_t>(i) * p.W;
                for (int j = lane; j < p.W; j += 32) {
                    orow[j] = from_f<T>(yrow[j]);
                    yrow[j] = 0.0f;
                }
            }
            dir_barrier();
        }
    }
    cp_async_wait<0>();
}

template <typename T, int R, int MODE>
__global__ void __launch_bounds__(kDirThreads)
prop2d_dir_kernel(const DirParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *ys = reinterpret_cast<float *>(smem);
    if (MODE != kYGlobal)
        for (int e = threadIdx.x; e < p.band_rows * p.y_pitch; e += kDirThreads) ys[e] = 0.0f;
    if (threadIdx.x == 0) {
        // one arrival per tensor span of a row chunk
        for (int i = 0; i < 2 * kDirStages; ++i) mbar_init(smem_u32(smem + p.bar_off) + 8 * i, kTensors);
        mbar_init_fence();
    }
    __syncthreads();
    if (warp < 2) dir_role<T, R, true, MODE>(p, smem, warp, lane, warp);
    else dir_role<T, R, false, MODE>(p, smem, warp, lane, warp);
}

}  // namespace gspn
