// Fused Prop2D forward, paired-direction kernel.
//
// One CTA of two warps owns one (batch, channel) plane (or one band of its
// output rows when the fp32 output plane does not fit in shared memory):
//   warp 0 sweeps row lines: top->bottom and bottom->top at the same time,
//   warp 1 sweeps column lines: left->right and right->left at the same time.
// The two opposite directions of a warp advance in lock step (step s handles
// line s of the forward sweep and line L-1-s of the backward sweep) and are
// held as the two halves of packed fp32x2 values, so every multiply-add of
// the normalisation and of the recurrence is one f32x2 instruction for both
// directions.  Lane l holds the R consecutive positions q = l*R + r of its
// lines in registers; neighbours across lanes come from shuffles.
//
// Normalisation (Sec. 5.1 "Fused CUDA normalization": sigmoid, local sum,
// clamp, divide), folded into the update.  With a_k = 1 + exp(-z_k),
// sigmoid(z_k) = 1 / a_k and, for P_k = product of a_j over the other
// on-grid slots j != k and D = sum_k P_k,
//     h = sum_k w_k h_prev(q+k-1) + lambda x = (sum_k P_k h_prev(q+k-1)) / D + lambda x,
// which takes three exponentials and one reciprocal per position and
// direction.  An off-grid slot takes a_k = 1, P_k = 0.  Whenever the clamp
// of the denominator could bind, or a product overflows, D exceeds a
// threshold (1e11 with three on-grid slots, 1e5 with two) or is not finite,
// and the positions of that step are recomputed in the plain form.
// The weights of step s+1 do not depend on the hidden line, so they are
// computed while step s's recurrence runs (software pipelining).
//
// Input lines are staged in shared memory, several lines per chunk, in a
// per-warp ring:
//   * row lines: the rows of a chunk are one contiguous span per tensor; one
//     lane moves each span with a single bulk copy (TMA engine) into a
//     16-byte aligned slot, completion tracked by one mbarrier per stage;
//   * column lines: a strip of 16 bytes of every row (8 bf16 / 4 fp32
//     columns) moved by the lanes with 4-byte cp.async; a strip row takes 4
//     words and the word index is XOR-swizzled by row so that the lanes
//     reading one column hit distinct banks (odd R), or rows are padded to 5
//     words plus one word per lane (even R).
// The gated outputs u * h of the four directions are summed into one fp32
// plane in shared memory with shared-memory atomics and written once.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace gspn {

constexpr int kPairThreads = 64;   // warp 0: row lines, warp 1: column lines
constexpr int kRowStages = 3;
constexpr int kColStages = 2;
constexpr int kColWords = 4;       // 16 bytes of each row per column chunk
constexpr int kPairTensors = 6;    // lambda, u, logit0, logit1, logit2, x

// Output modes.
constexpr int kYSmem = 0;     // whole fp32 output plane in shared memory
constexpr int kYBanded = 1;   // a band of output rows in shared memory, scans rerun per band
constexpr int kYGlobal = 2;   // fp32 output accumulated in global memory (L2 atomics)

struct PairParams {
    const void *x, *lam, *wl, *u;
    void *out;
    int B, Cc, H, W, dirs, share_w;
    int n_items, bands, band_rows;
    int t_row;                 // rows per row-warp chunk
    int slot_row, slot_col;    // bytes per (half, tensor) slot of each ring
    int ring_row, ring_col;    // byte offsets of the two rings in shared memory
    int bar_off;               // byte offset of the row ring's mbarriers and shift table
    int y_pitch;               // floats per staged output row (odd)
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
__device__ __forceinline__ size_t pair_plane(const PairParams &p, int b, int c, int d, int t) {
    const size_t HW = static_cast<size_t>(p.H) * p.W;
    if (t == 5) return (static_cast<size_t>(b) * p.Cc + c) * HW;
    if (t < 2) return ((static_cast<size_t>(b) * 4 + d) * p.Cc + c) * HW;
    const int Cw = p.share_w ? 1 : p.Cc;
    return ((((static_cast<size_t>(b) * 4 + d) * Cw + (p.share_w ? 0 : c)) * 3) + (t - 2)) * HW;
}

__device__ __forceinline__ const char *pair_tensor(const PairParams &p, int t) {
    const void *base = t == 0 ? p.lam : t == 1 ? p.u : t == 5 ? p.x : p.wl;
    return static_cast<const char *>(base);
}

__device__ __forceinline__ unsigned long long pair_tensor_bytes(const PairParams &p, int t) {
    return t == 5 ? p.end_x : t < 2 ? p.end_gate : p.end_wl;
}

// Lines [lo, hi) of chunk c for the forward (h = 0) or backward (h = 1) sweep.
__device__ __forceinline__ void pair_chunk(int c, int T_, int L, int h, int &lo, int &hi) {
    if (h == 0) {
        lo = c * T_;
        hi = min(L, lo + T_);
    } else {
        hi = L - c * T_;
        lo = max(0, hi - T_);
    }
}

// Per-step precomputed normalisation and gates of the lane's R positions.
template <int R>
struct StepW {
    float2 P0[R], P1[R], P2[R], rD[R], bx[R], uu[R];
    bool bad;      // some position needs the plain form (D over its threshold, or NaN)
};

template <typename T, int R, bool ROW, int MODE>
struct PairWarp {
    static constexpr int es = sizeof(T);
    static constexpr int NS = ROW ? kRowStages : kColStages;
    static constexpr int kColRows = (32 * R + 32 / kColWords - 1) / (32 / kColWords);  // strip rows per lane

    const PairParams &p;
    const int lane;
    unsigned char *const ring;
    const uint32_t bars;      // shared address of the row ring's mbarriers (ROW only)
    unsigned char *const shifts;   // [stage][half][tensor] byte shift of each staged span (ROW only)
    const int slot;
    const int L, M, T_, nch;
    const bool on_f, on_b;
    const int d_f, d_b;
    // Plane base pointers of the item whose chunks are being issued.  ROW:
    // lane (h * 6 + t) < 12 keeps the pointer of the (half, tensor) span it
    // copies.  COL: every lane copies every (half, tensor), so the 12
    // pointers live in a shared table.
    int issue_item;
    const char *my_gp;
    const char **gtab;
    int col_off[kColRows];    // strip-row word offsets of this lane's rows (COL only)

    __device__ PairWarp(const PairParams &p_, unsigned char *smem_, int lane_)
        : p(p_), lane(lane_),
          ring(smem_ + (ROW ? p_.ring_row : p_.ring_col)),
          bars(smem_u32(smem_ + p_.bar_off)),
          shifts(smem_ + p_.bar_off + 64),
          slot(ROW ? p_.slot_row : p_.slot_col),
          L(ROW ? p_.H : p_.W), M(ROW ? p_.W : p_.H),
          T_(ROW ? p_.t_row : kColWords * 4 / es),
          nch(((ROW ? p_.H : p_.W) + (ROW ? p_.t_row : kColWords * 4 / es) - 1) /
              (ROW ? p_.t_row : kColWords * 4 / es)),
          on_f((p_.dirs >> (ROW ? 0 : 2)) & 1), on_b((p_.dirs >> (ROW ? 1 : 3)) & 1),
          d_f(ROW ? 0 : 2), d_b(ROW ? 1 : 3), issue_item(-1), my_gp(nullptr),
          gtab(reinterpret_cast<const char **>(smem_ + p_.bar_off + 128)) {
        if (!ROW) {
            const int w = lane & (kColWords - 1), i0 = lane / kColWords;
#pragma unroll
            for (int k = 0; k < kColRows; ++k) col_off[k] = 4 * ColLayout<R>::word(i0 + k * (32 / kColWords), w);
        }
    }

    __device__ __forceinline__ unsigned char *slot_ptr(int stage, int h, int t) const {
        return ring + ((stage * 2 + h) * kPairTensors + t) * slot;
    }

    __device__ __forceinline__ void set_issue_item(int item) {
        if (item == issue_item) return;
        issue_item = item;
        const int plane = item / p.bands;
        const int b = plane / p.Cc, ch = plane - b * p.Cc;
        if (!ROW) __syncwarp();   // every lane is done with the previous item's table
        if (lane < 2 * kPairTensors) {
            const int h = lane / kPairTensors, t = lane - h * kPairTensors;
            my_gp = pair_tensor(p, t) + pair_plane(p, b, ch, h == 0 ? d_f : d_b, t) * es;
            if (!ROW) gtab[lane] = my_gp;
        }
        if (!ROW) __syncwarp();   // the new table is visible to every lane
    }

    // Issue the copies of chunk c of item `item` into ring stage `stage`.
    // ROW: lane h*6+t < 12 copies the span of (half h, tensor t) with one bulk
    // copy and arrives on the stage's mbarrier (initialised for 12 arrivals)
    // with its byte count.  COL: every lane issues 4-byte cp.async for its
    // strip rows of every (half, tensor), then commits.
    __device__ __forceinline__ void issue(int item, int c, int stage) {
        set_issue_item(item);
        if (ROW) {
            __syncwarp();   // every lane is done reading the stage being refilled
            if (lane < 2 * kPairTensors) {
                const int h = lane / kPairTensors, t = lane - h * kPairTensors;
                fence_proxy_async_smem();
                int lo, hi;
                pair_chunk(c, T_, L, h, lo, hi);
                const char *s = my_gp + static_cast<size_t>(lo) * p.W * es;
                const uint32_t sh = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(s) & 15);
                const char *a = s - sh;
                uint32_t n = (sh + static_cast<uint32_t>((hi - lo) * p.W * es) + 15u) & ~15u;
                int tl = 0;
                // never read past the end of the tensor: the last partial 16 bytes
                // are then copied by hand
                const unsigned long long end = pair_tensor_bytes(p, t);
                const unsigned long long off = static_cast<unsigned long long>(a - pair_tensor(p, t));
                if (off + n > end) {
                    tl = static_cast<int>(end - (off + n - 16));
                    n -= 16;
                }
                if (!(h == 0 ? on_f : on_b)) { n = 0; tl = 0; }
                unsigned char *dst = slot_ptr(stage, h, t);
                shifts[(stage * 2 + h) * kPairTensors + t] = static_cast<unsigned char>(sh);
                for (int e = 0; e < tl; e += 2)   // rare: end of the tensor
                    *reinterpret_cast<unsigned short *>(dst + n + e) =
                        *reinterpret_cast<const unsigned short *>(a + n + e);
                const uint32_t bar = bars + 8 * stage;
                mbar_arrive_expect_tx(bar, n);
                if (n) bulk_copy_g2s(smem_u32(dst), a, n, bar);
            }
        } else {
            const int w = lane & (kColWords - 1), i0 = lane / kColWords;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (!(h == 0 ? on_f : on_b)) continue;
                int lo, hi;
                pair_chunk(c, T_, L, h, lo, hi);
                const int nw = ((hi - lo) * es) >> 2;   // words per row segment, <= kColWords
                if (w >= nw) continue;
                const size_t gstep = static_cast<size_t>(32 / kColWords) * p.W * es;
#pragma unroll
                for (int t = 0; t < kPairTensors; ++t) {
                    const char *s = gtab[h * kPairTensors + t] + (static_cast<size_t>(i0) * p.W + lo) * es + 4 * w;
                    const uint32_t sb = smem_u32(slot_ptr(stage, h, t));
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

    // Wait until the chunk in `stage` (the g-th chunk of this warp) has landed.
    __device__ __forceinline__ void wait_chunk(int g, int stage) const {
        if (ROW) {
            mbar_wait_bounded(bars + 8 * stage, static_cast<uint32_t>((g / NS) & 1));
        } else {
            cp_async_wait<0>();
            __syncwarp();
        }
    }

    __device__ __forceinline__ const unsigned char *elem(const unsigned char *slotp, int shift,
                                                         int li, int r) const {
        if (ROW) return slotp + shift + (li * p.W + lane * R + r) * es;
        const int q = lane * R + r;
        return slotp + 4 * ColLayout<R>::word(q, (li * es) >> 2) + ((li * es) & 3);
    }

    // Raw inputs of one line (both halves) -> normalisation terms.
    __device__ __forceinline__ void weights(const unsigned char *const (&sp)[2][kPairTensors],
                                            const int (&shift)[2][kPairTensors], int li_f, int li_b,
                                            const float (&m0)[R], const float (&m2)[R],
                                            const float (&ithr)[R], const bool (&valid)[R],
                                            StepW<R> &W) const {
        const float2 one2 = make_float2(1.0f, 1.0f);
        const float2 nl2e = make_float2(-1.4426950408889634f, -1.4426950408889634f);
        bool bad = false;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float v[2][kPairTensors];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int t = 0; t < kPairTensors; ++t)
                    v[h][t] = sload<T>(elem(sp[h][t], shift[h][t], h == 0 ? li_f : li_b, r));
            const float2 t0 = __fmul2_rn(make_float2(v[0][2], v[1][2]), nl2e);
            const float2 t1 = __fmul2_rn(make_float2(v[0][3], v[1][3]), nl2e);
            const float2 t2 = __fmul2_rn(make_float2(v[0][4], v[1][4]), nl2e);
            const float2 e0 = make_float2(ex2(t0.x), ex2(t0.y));
            const float2 e1 = make_float2(ex2(t1.x), ex2(t1.y));
            const float2 e2 = make_float2(ex2(t2.x), ex2(t2.y));
            const float2 a0 = r == 0 ? __ffma2_rn(e0, make_float2(m0[r], m0[r]), one2) : __fadd2_rn(e0, one2);
            const float2 a1 = __fadd2_rn(e1, one2);
            const float2 a2 = __ffma2_rn(e2, make_float2(m2[r], m2[r]), one2);
            float2 P0 = __fmul2_rn(a1, a2);
            if (r == 0) P0 = __fmul2_rn(P0, make_float2(m0[r], m0[r]));
            const float2 P1 = __fmul2_rn(a0, a2);
            const float2 P2 = __fmul2_rn(__fmul2_rn(a0, a1), make_float2(m2[r], m2[r]));
            const float2 D = __fadd2_rn(__fadd2_rn(P0, P1), P2);
            // over the threshold, or NaN (an off-grid slot whose exponential overflowed)
            const float2 k = __fmul2_rn(D, make_float2(ithr[r], ithr[r]));
            bad = bad || (valid[r] && !(k.x <= 1.0f && k.y <= 1.0f));
            W.P0[r] = P0;
            W.P1[r] = P1;
            W.P2[r] = P2;
            W.rD[r] = make_float2(rcp(D.x), rcp(D.y));
            W.bx[r] = __fmul2_rn(make_float2(v[0][0], v[1][0]), make_float2(v[0][5], v[1][5]));
            W.uu[r] = make_float2(v[0][1], v[1][1]);
        }
        W.bad = bad;
    }

    // Plain-form update of the step for every position (rare path).
    __device__ __forceinline__ void plain_step(const unsigned char *const (&sp)[2][kPairTensors],
                                               const int (&shift)[2][kPairTensors], int li_f, int li_b,
                                               const float2 (&h)[R], float2 hl, float2 hr,
                                               float2 (&hn)[R]) const {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = lane * R + r;
            const float2 left = r > 0 ? h[r - 1] : hl;
            const float2 right = r < R - 1 ? h[r + 1] : hr;
            float out[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int li = hh == 0 ? li_f : li_b;
                float v[kPairTensors];
#pragma unroll
                for (int t = 0; t < kPairTensors; ++t) v[t] = sload<T>(elem(sp[hh][t], shift[hh][t], li, r));
                const W3 w = normalise_plain(v[2], v[3], v[4], q > 0, q + 1 < M);
                const float hl_ = hh == 0 ? left.x : left.y, hc = hh == 0 ? h[r].x : h[r].y,
                            hr_ = hh == 0 ? right.x : right.y;
                float acc = v[0] * v[5];
                if (q > 0) acc = fmaf(w.w0, hl_, acc);
                acc = fmaf(w.w1, hc, acc);
                if (q + 1 < M) acc = fmaf(w.w2, hr_, acc);
                out[hh] = acc;
            }
            hn[r] = make_float2(out[0], out[1]);
        }
    }

    // Run every line of `item`.  `g` counts this warp's chunks in the launch
    // (ring position); `total` is the number of chunks it runs in the launch.
    // Lines are processed in one software-pipelined sequence: the weights of
    // line s+1 (which may sit in the next chunk) are computed during line s.
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
        float2 hs[R];
#pragma unroll
        for (int r = 0; r < R; ++r) hs[r] = make_float2(0.0f, 0.0f);

        // chunk state: current chunk c, its stage pointers and line ranges
        const unsigned char *sp[2][kPairTensors];
        int shift[2][kPairTensors];
        int lo_f = 0, hi_b = 0, nl = 0;
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
            int hi_f, lo_b;
            pair_chunk(c, T_, L, 0, lo_f, hi_f);
            pair_chunk(c, T_, L, 1, lo_b, hi_b);
            nl = hi_f - lo_f;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int t = 0; t < kPairTensors; ++t) {
                    sp[h][t] = slot_ptr(stage, h, t);
                    shift[h][t] = ROW ? shifts[(stage * 2 + h) * kPairTensors + t] : 0;
                }
        };

        // Iteration s runs the recurrence of line s-1 (weights already in Wc),
        // then computes the weights of line s, then accumulates line s-1's
        // outputs; the weights and the recurrence each appear once in the code.
        int c = 0, tt = -1;
        enter_chunk(0);
        StepW<R> Wc;
        int cur_f = 0, cur_b = 0;
        for (int s = 0; s <= L; ++s) {
            float2 hn[R], uu[R];
            if (s > 0) {
                float2 hl, hr;
                hl.x = __shfl_up_sync(0xffffffffu, hs[R - 1].x, 1);
                hl.y = __shfl_up_sync(0xffffffffu, hs[R - 1].y, 1);
                hr.x = __shfl_down_sync(0xffffffffu, hs[0].x, 1);
                hr.y = __shfl_down_sync(0xffffffffu, hs[0].y, 1);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float2 left = r > 0 ? hs[r - 1] : hl;
                    const float2 right = r < R - 1 ? hs[r + 1] : hr;
                    float2 N = __fmul2_rn(Wc.P0[r], left);
                    N = __ffma2_rn(Wc.P1[r], hs[r], N);
                    N = __ffma2_rn(Wc.P2[r], right, N);
                    hn[r] = __ffma2_rn(N, Wc.rD[r], Wc.bx[r]);
                }
                if (__any_sync(0xffffffffu, Wc.bad))
                    plain_step(sp, shift, tt, nl - 1 - tt, hs, hl, hr, hn);
#pragma unroll
                for (int r = 0; r < R; ++r) uu[r] = Wc.uu[r];
            }
            const int pl_f = cur_f, pl_b = cur_b;   // lines of step s-1
            if (s < L) {
                // next line, possibly in the next chunk
                if (++tt == nl) {
                    ++g;
                    ++c;
                    tt = 0;
                    enter_chunk(c);
                }
                cur_f = lo_f + tt;
                cur_b = hi_b - 1 - tt;
                weights(sp, shift, tt, nl - 1 - tt, m0, m2, ithr, valid, Wc);
            }
            if (s == 0) continue;
            const int line_f = pl_f, line_b = pl_b;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                hs[r] = valid[r] ? hn[r] : make_float2(0.0f, 0.0f);
                const float2 cy = __fmul2_rn(uu[r], hs[r]);
                const int q = lane * R + r;
                if (MODE == kYGlobal) {
                    if (valid[r]) {
                        if (ROW) {
                            atomicAdd(yg + static_cast<size_t>(line_f) * p.W + q, cy.x);
                            atomicAdd(yg + static_cast<size_t>(line_b) * p.W + q, cy.y);
                        } else {
                            atomicAdd(yg + static_cast<size_t>(q) * p.W + line_f, cy.x);
                            atomicAdd(yg + static_cast<size_t>(q) * p.W + line_b, cy.y);
                        }
                    }
                } else if (ROW) {
                    const bool inf_ = MODE != kYBanded || (line_f >= band_lo && line_f < band_hi);
                    const bool inb_ = MODE != kYBanded || (line_b >= band_lo && line_b < band_hi);
                    red_add_shared_if(ysa + 4u * ((line_f - band_lo) * p.y_pitch + q), cy.x, valid[r] && inf_);
                    red_add_shared_if(ysa + 4u * ((line_b - band_lo) * p.y_pitch + q), cy.y, valid[r] && inb_);
                } else {
                    const uint32_t yrow = ysa + 4u * ((q - band_lo) * p.y_pitch);
                    red_add_shared_if(yrow + 4u * line_f, cy.x, inband[r]);
                    red_add_shared_if(yrow + 4u * line_b, cy.y, inband[r]);
                }
            }
        }
        ++g;   // the last chunk of the item is done
    }
};

// Barrier of the CTA's two warps.  The two warps run different code paths
// (one per role), so the barrier is a named PTX barrier with an explicit
// thread count rather than __syncthreads.
__device__ __forceinline__ void pair_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(kPairThreads) : "memory");
}

// The whole kernel seen from one warp of role ROW (row lines) or !ROW
// (column lines); only that role's state is live in its registers.
template <typename T, int R, bool ROW, int MODE>
__device__ __forceinline__ void pair_role(const PairParams &p, unsigned char *smem, int warp, int lane) {
    float *ys = reinterpret_cast<float *>(smem);   // output plane or band, fp32 [rows][y_pitch]
    const int YP = p.y_pitch;
    const bool active = ROW ? (p.dirs & 3) != 0 : (p.dirs & 12) != 0;
    const int n_my = blockIdx.x < p.n_items ? (p.n_items - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    PairWarp<T, R, ROW, MODE> w(p, smem, lane);
    constexpr int NS = ROW ? kRowStages : kColStages;
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
            for (int e = threadIdx.x; e < p.H * p.W; e += kPairThreads) yg[e] = 0.0f;
            pair_barrier();
        }
        if (active) w.run_item(item, g, total, ys, yg, band_lo, band_hi);
        pair_barrier();
        if (MODE != kYGlobal) {
            // write the band out once (converted) and clear it for the next item
            T *outp = static_cast<T *>(p.out) + static_cast<size_t>(plane) * p.H * p.W +
                      static_cast<size_t>(band_lo) * p.W;
            for (int i = warp; i < band_hi - band_lo; i += 2) {
                float *yrow = ys + i * YP;
                T *orow = outp + static_cast<size_t>(i) * p.W;
                for (int j = lane; j < p.W; j += 32) {
                    orow[j] = from_f<T>(yrow[j]);
                    yrow[j] = 0.0f;
                }
            }
            pair_barrier();
        }
    }
    cp_async_wait<0>();
}

template <typename T, int R, int MODE>
__global__ void __launch_bounds__(kPairThreads)
prop2d_pair_kernel(const PairParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *ys = reinterpret_cast<float *>(smem);
    const int YP = p.y_pitch;
    const bool row_on = p.dirs & 3, col_on = p.dirs & 12;

    // zero the output band and the staging slots of disabled directions
    // (a disabled half of an enabled warp then reads zeros: no contribution)
    if (MODE != kYGlobal)
        for (int e = threadIdx.x; e < p.band_rows * YP; e += kPairThreads) ys[e] = 0.0f;
    if (row_on && ((p.dirs & 3) != 3)) {
        const int h = (p.dirs & 1) ? 1 : 0;
        for (int s = 0; s < kRowStages; ++s) {
            float *z = reinterpret_cast<float *>(smem + p.ring_row + ((s * 2 + h) * kPairTensors) * p.slot_row);
            for (int e = threadIdx.x; e < kPairTensors * p.slot_row / 4; e += kPairThreads) z[e] = 0.0f;
        }
    }
    if (col_on && ((p.dirs & 12) != 12)) {
        const int h = (p.dirs & 4) ? 1 : 0;
        for (int s = 0; s < kColStages; ++s) {
            float *z = reinterpret_cast<float *>(smem + p.ring_col + ((s * 2 + h) * kPairTensors) * p.slot_col);
            for (int e = threadIdx.x; e < kPairTensors * p.slot_col / 4; e += kPairThreads) z[e] = 0.0f;
        }
    }
    if (threadIdx.x == 0) {
        // one arrival per (half, tensor) span of a row chunk
        for (int s = 0; s < kRowStages; ++s) mbar_init(smem_u32(smem + p.bar_off) + 8 * s, 2 * kPairTensors);
        mbar_init_fence();
    }
    __syncthreads();
    if (warp == 0) pair_role<T, R, true, MODE>(p, smem, warp, lane);
    else pair_role<T, R, false, MODE>(p, smem, warp, lane);
}

}  // namespace gspn
