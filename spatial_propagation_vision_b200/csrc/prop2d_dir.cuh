// Fused Prop2D forward, one warp per direction.
//
// One CTA of four warps owns one (batch, channel) plane (or one band of its
// output rows when the fp32 output plane does not fit in shared memory);
// warp d runs direction d: 0 top->bottom, 1 bottom->top (row lines),
// 2 left->right, 3 right->left (column lines).  The two sweeps of an
// orientation share one code path with a runtime sweep sign, which halves
// the instruction footprint.  Lane l holds R positions of the current line
// in registers: for row lines positions 2l and 2l+1 of every 64-position
// block (one 32-bit word of bf16) plus 64*(R/2) + l when R is odd; for
// column lines the R consecutive positions q = l*R + r.  Neighbours held by
// another lane come from shuffles.
//
// Normalisation (Sec. 5.1 "Fused CUDA normalization": sigmoid, local sum,
// clamp, divide), folded into the update.  With a_k = 1 + exp(-z_k),
// sigmoid(z_k) = 1 / a_k and, for P_k = product of a_j over the other
// on-grid slots j != k and D = sum_k P_k, w_k = P_k / D: three exponentials
// and one reciprocal per position.  An off-grid slot takes a_k = 1, P_k = 0.
// Whenever the clamp of the denominator could bind, or a product overflows,
// D exceeds a threshold (1e11 with three on-grid slots, 1e5 with two) or is
// not finite; the weights of that line are then recomputed in the plain
// form.  The weights of line s+1 do not depend on the hidden state; they are
// computed in the same block as line s's update, alternating between two
// register sets.  In the compact mode with a workspace (PRE), the weights
// were normalised ahead once for all channels (prop2d_norm.cuh) and are read.
//
// Input staging:
//   * row lines: each lane loads its words of a line straight from global
//     memory (read-only path), three or four lines ahead into registers; one
//     lane per tensor issues a bulk L2 prefetch (TMA engine) of the lines
//     about to be read, eight lines ahead, continuing into the warp's next
//     plane;
//   * column lines: a chunk is a strip of 16 bytes of every grid row (8 bf16
//     or 4 fp32 columns), copied by the warp with 4-byte cp.async (four lanes
//     per grid row) into a two-stage ring.  The strip rows of the six tensors
//     are interleaved (104-byte pitch), and right-to-left sweeps store the
//     words of a strip row in reverse order, so both sweeps meet their
//     columns in scan order.  A four-step body reads its columns with one
//     8-byte read per tensor and position (bf16; two for fp32).
// Outputs u * h are accumulated in shared memory and written once,
// converted, at the end of the plane (modes below): two planes (rows,
// columns) written without atomics, each shared by a sweep pair that splits
// at the midpoint (fp32 planes, or for bf16 inputs bf16 planes of pair words
// whose column midpoint is word-aligned); one fp32 plane that all directions
// add into with shared-memory atomics; global atomics and row bands cover
// planes too large for shared memory.
//
// Positions past the end of a line (q >= M) compute finite garbage that
// never reaches a valid position: their right-hand neighbour term of
// position M-1 has P_2 = 0.  For that they read finite values only: the
// rings are zeroed at launch and afterwards hold copies of the inputs
// (column lanes past the end read grid row 0's strip; row lanes read a
// clamped in-plane word).
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_common.cuh"

namespace gspn {

constexpr int kDirThreads = 128;   // warp d runs direction d
constexpr int kColStages = 2;      // column ring depth
constexpr int kTensors = 6;        // lambda, u, logit0, logit1, logit2, x
constexpr int kColStrip = 16;      // bytes of each grid row per column chunk
constexpr int kColPitch = 104;     // bytes per grid row of a column stage: 6 x 16 + 8
constexpr int kDirBarBytes = 256;  // plane-pointer tables of the column warps

// Output modes.
constexpr int kYSmem = 0;     // whole fp32 output plane in shared memory
constexpr int kYBanded = 1;   // a band of output rows in shared memory, scans rerun per band
constexpr int kYGlobal = 2;   // fp32 output accumulated in global memory (L2 atomics)
constexpr int kYShared = 3;   // one fp32 plane in shared memory for all four directions
                              // (shared-memory atomics; the warps never wait for one
                              // another before the end of a plane)
constexpr int kYHalf = 4;     // bf16 only: two bf16 planes (rows, columns) of pair words
                              // (columns 2j, 2j+1 in word j), written without atomics:
                              // each sweep pair splits at a word-aligned midpoint

struct DirParams {
    const void *x, *lam, *wl, *u;
    void *out;
    int B, Cc, H, W, dirs;
    int gate_dirs;              // direction slots of lambda and u: 4, or 1 shared by all directions
    int w_groups, w_cpg;        // logit fields per (batch, direction) and channels per field
    int n_items, bands, band_rows;
    int stage_col;              // bytes per column ring stage
    int ring[4];                // byte offset of column direction d's ring (-1: none)
    int bar_off;                // byte offset of the column warps' plane-pointer tables
    int ycol_off;               // byte offset of the column directions' output plane
    int y_pitch;                // floats per staged output row (odd, > every ycol(j), j < W);
                                // kYHalf: 32-bit words per row (>= W/2 + 1, the last a dummy)
    unsigned long long end_x, end_gate, end_wl;   // byte sizes of x, lambda/u, logits
};


// Element offset of plane (b, c) of tensor t for direction d.
__device__ __forceinline__ size_t dir_plane(const DirParams &p, int b, int c, int d, int t) {
    const size_t HW = static_cast<size_t>(p.H) * p.W;
    if (t == 5) return (static_cast<size_t>(b) * p.Cc + c) * HW;
    if (t < 2)
        return ((static_cast<size_t>(b) * p.gate_dirs + (p.gate_dirs == 4 ? d : 0)) * p.Cc + c) * HW;
    return ((((static_cast<size_t>(b) * 4 + d) * p.w_groups + c / p.w_cpg) * 3) + (t - 2)) * HW;
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
    float w0[R], w1[R], w2[R], bx[R], uu[R];   // w_k: normalised weight of slot k
};

// Per-lane constants of a line of M positions.
template <int R>
struct LaneGeom {
    float m0[R], m2[R];   // 1 where the slot k = 0 / k = 2 neighbour is on the grid
    int thr[R];           // bit pattern of the fast-form threshold on D
    bool valid[R];        // q < M
    __device__ __forceinline__ void init(int lane, int M) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = lane * R + r;
            valid[r] = q < M;
            m0[r] = q > 0 ? 1.0f : 0.0f;
            m2[r] = q + 1 < M ? 1.0f : 0.0f;
            thr[r] = __float_as_int((q > 0 && q + 1 < M) ? 1e11f : 1e5f);
        }
    }
};

// Raw inputs of one line -> normalisation terms.  Returns true when some
// position is outside the fast form's range: D above its threshold, or not
// finite (as bit patterns, +inf and the hardware's NaN compare above every
// threshold).  Positions past the end of the line take part; a flagged line
// is simply recomputed in the plain form.
template <int R>
__device__ __forceinline__ bool line_weights(const float (&v)[kTensors][R], const LaneGeom<R> &g,
                                             LineW<R> &W) {
    constexpr float nl2e = -1.4426950408889634f;
    bool bad = false;
#pragma unroll
    for (int r = 0; r + 1 < R; r += 2) {
        const float2 n2 = make_float2(nl2e, nl2e);
        const float2 one2 = make_float2(1.0f, 1.0f);
        const float2 mm0 = make_float2(g.m0[r], g.m0[r + 1]);
        const float2 mm2 = make_float2(g.m2[r], g.m2[r + 1]);
        const float2 t0 = __fmul2_rn(make_float2(v[2][r], v[2][r + 1]), n2);
        const float2 t1 = __fmul2_rn(make_float2(v[3][r], v[3][r + 1]), n2);
        const float2 t2 = __fmul2_rn(make_float2(v[4][r], v[4][r + 1]), n2);
        const float2 a0 = __ffma2_rn(make_float2(ex2(t0.x), ex2(t0.y)), mm0, one2);
        const float2 a1 = __fadd2_rn(make_float2(ex2(t1.x), ex2(t1.y)), one2);
        const float2 a2 = __ffma2_rn(make_float2(ex2(t2.x), ex2(t2.y)), mm2, one2);
        const float2 P0 = __fmul2_rn(__fmul2_rn(a1, a2), mm0);
        const float2 P1 = __fmul2_rn(a0, a2);
        const float2 P2 = __fmul2_rn(__fmul2_rn(a0, a1), mm2);
        const float2 Dn = __fadd2_rn(__fadd2_rn(P0, P1), P2);
        bad |= (__float_as_int(Dn.x) > g.thr[r]) | (__float_as_int(Dn.y) > g.thr[r + 1]);
        const float2 rD = make_float2(rcp(Dn.x), rcp(Dn.y));
        const float2 w0 = __fmul2_rn(P0, rD), w1 = __fmul2_rn(P1, rD), w2 = __fmul2_rn(P2, rD);
        const float2 bx = __fmul2_rn(make_float2(v[0][r], v[0][r + 1]), make_float2(v[5][r], v[5][r + 1]));
        W.w0[r] = w0.x; W.w0[r + 1] = w0.y;
        W.w1[r] = w1.x; W.w1[r + 1] = w1.y;
        W.w2[r] = w2.x; W.w2[r + 1] = w2.y;
        W.bx[r] = bx.x; W.bx[r + 1] = bx.y;
        W.uu[r] = v[1][r]; W.uu[r + 1] = v[1][r + 1];
    }
    if (R % 2) {
        const int r = R - 1;
        const float a0 = fmaf(ex2(v[2][r] * nl2e), g.m0[r], 1.0f);
        const float a1 = ex2(v[3][r] * nl2e) + 1.0f;
        const float a2 = fmaf(ex2(v[4][r] * nl2e), g.m2[r], 1.0f);
        const float P0 = a1 * a2 * g.m0[r];
        const float P1 = a0 * a2;
        const float P2 = a0 * a1 * g.m2[r];
        const float Dn = (P0 + P1) + P2;
        bad |= __float_as_int(Dn) > g.thr[r];
        const float rD = rcp(Dn);
        W.w0[r] = P0 * rD;
        W.w1[r] = P1 * rD;
        W.w2[r] = P2 * rD;
        W.bx[r] = v[0][r] * v[5][r];
        W.uu[r] = v[1][r];
    }
    return bad;
}

// Plain-form terms of one line (rare path): the normalised weights go in
// w0..w2 like the fast form's.  Same
// arithmetic as the fast form's exponentials and reciprocals, without
// products: sigmoid(z) = 1 / (1 + 2^(-z log2 e)) saturates to 0 or 1 instead
// of overflowing, and the clamp of the local sum is explicit.
template <int R>
__device__ __forceinline__ void line_weights_plain_v(const float (&v)[kTensors][R], const LaneGeom<R> &g,
                                                     LineW<R> &W) {
    constexpr float nl2e = -1.4426950408889634f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        // off-grid slots are selected away (their logits may be anything,
        // NaN included, and must not reach the weights)
        // (positions past the line's end read another position's inputs,
        // off-grid slots included, and take no weight at all)
        const bool on = g.valid[r];
        const float s0 = on && g.m0[r] != 0.0f ? rcp(1.0f + ex2(v[2][r] * nl2e)) : 0.0f;
        const float s1 = on ? rcp(1.0f + ex2(v[3][r] * nl2e)) : 0.0f;
        const float s2 = on && g.m2[r] != 0.0f ? rcp(1.0f + ex2(v[4][r] * nl2e)) : 0.0f;
        const float iS = rcp(fmaxf((s0 + s1) + s2, 1e-6f));
        W.w0[r] = s0 * iS;
        W.w1[r] = s1 * iS;
        W.w2[r] = s2 * iS;
        W.bx[r] = v[0][r] * v[5][r];
        W.uu[r] = v[1][r];
    }
}

// Terms of one line from its raw inputs: the fast form, or the plain form
// for the whole line (every lane) when some position is out of the fast
// form's range.
template <int R>
__device__ __forceinline__ void line_terms(const float (&v)[kTensors][R], const LaneGeom<R> &g, LineW<R> &W) {
    const bool bad = line_weights(v, g, W);
    if (__any_sync(0xffffffffu, bad)) line_weights_plain_v<R>(v, g, W);
}
// The same check as a separate call, so that a step can place it (a branch,
// which ends a straight-line block) after the rest of its work.
template <int R>
__device__ __forceinline__ void line_terms_fix(bool bad, const float (&v)[kTensors][R], const LaneGeom<R> &g,
                                               LineW<R> &W) {
    if (__any_sync(0xffffffffu, bad)) line_weights_plain_v<R>(v, g, W);
}

// Terms of one line whose weights were normalised ahead of the scan (the
// compact mode's weights, shared by every channel): slots 2, 3 and 4 hold w0,
// the sum of the three weights and w2, so w1 is their difference and the
// weights of a position sum exactly to that sum (1 unless the clamp bound).
template <int R>
__device__ __forceinline__ void line_pre(const float (&v)[kTensors][R], LineW<R> &W) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
        W.w0[r] = v[2][r];
        W.w2[r] = v[4][r];
        W.w1[r] = (v[3][r] - v[2][r]) - v[4][r];
        W.bx[r] = v[0][r] * v[5][r];
        W.uu[r] = v[1][r];
    }
}

// Weights of the next line from its unpacked inputs: computed from the
// logits (fast form, flagged lines redone in the plain form by
// line_terms_fix), or read when they were normalised ahead (PRE).
template <bool PRE, int R>
__device__ __forceinline__ bool next_weights(const float (&v)[kTensors][R], const LaneGeom<R> &g, LineW<R> &W) {
    if constexpr (PRE) {
        line_pre(v, W);
        return false;
    } else {
        return line_weights(v, g, W);
    }
}
template <bool PRE, int R>
__device__ __forceinline__ void first_weights(const float (&v)[kTensors][R], const LaneGeom<R> &g, LineW<R> &W) {
    if constexpr (PRE) line_pre(v, W);
    else line_terms(v, g, W);
}

// 16-bit half `hi` of a word as an fp32 value: bf16 bits, or (a weight
// normalised ahead, for bf16 inputs) fp16.
template <bool F16>
__device__ __forceinline__ float half_word(uint32_t w, bool hi) {
    if constexpr (F16) return __half2float(__ushort_as_half(static_cast<unsigned short>(hi ? (w >> 16) : w)));
    else return __uint_as_float(hi ? (w & 0xffff0000u) : (w << 16));
}

// Column of output position j in a staged output row: bit 0 of j is flipped
// in every other 32-column block, so that the row lanes' atomics on the
// even (odd) positions 2l (2l+1) of a 64-position block hit 32 banks.
__device__ __forceinline__ int ycol(int j) { return j ^ ((j >> 5) & 1); }

// The two sweeps of an orientation (top-down and bottom-up rows; left-right
// and right-left columns) add into one fp32 output plane of their own
// without atomics: before the midpoint each writes only the half of the
// plane it reaches first (rows / columns below ceil(L/2) for the forward
// sweep, the rest for the backward one) and stores; after a barrier of the
// two warps each adds to the half the other stored.  `split` is the first
// step after the midpoint; with one sweep of the orientation active it
// stores everywhere (split = L + 1: no barrier).
__device__ __forceinline__ int sweep_split(bool pair, bool fwd, int L) {
    return pair ? (fwd ? (L + 1) / 2 : L / 2) : L + 1;
}
__device__ __forceinline__ void pair_barrier(int id) {
    asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}
// Branch-free: positions past the end of a line write a dummy column /
// row of the plane, `first` is warp-uniform.
__device__ __forceinline__ void put_y(float *a, float v, bool first) {
    const float o = *a;
    *a = (first ? 0.0f : o) + v;
}

// One step of the recurrence: h <- (sum_k P_k h(q+k-1)) / D + lambda x.  The
// terms that need a neighbour lane's value (from the shuffles) come last.
template <int R>
__device__ __forceinline__ void recur(float (&h)[R], const LineW<R> &W) {
    const float hl = __shfl_up_sync(0xffffffffu, h[R - 1], 1);
    const float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
    float hn[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float N = fmaf(W.w1[r], h[r], W.bx[r]);
        if (r > 0) N = fmaf(W.w0[r], h[r - 1], N);
        if (r < R - 1) N = fmaf(W.w2[r], h[r + 1], N);
        if (r == 0) N = fmaf(W.w0[r], hl, N);
        if (r == R - 1) N = fmaf(W.w2[r], hr, N);
        hn[r] = N;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) h[r] = hn[r];
}

// ---------------------------------------------------------------------------
// Row lines (directions 0 and 1).
// ---------------------------------------------------------------------------
template <typename T, int R, int MODE, bool PRE>
struct RowScan {
    static constexpr int es = sizeof(T);
    static constexpr int NP = R / 2;            // blocks of position pairs
    static constexpr bool kSingle = (R % 2) != 0;
    // raw words of one line per tensor: bf16 pairs share a 32-bit word
    static constexpr int kWords = es == 2 ? NP + (kSingle ? 1 : 0) : R;
    using Raw = uint32_t[kTensors][kWords];
    // Raw words of the next kDepth lines are in flight in registers; the loop
    // body is kUnroll steps so that both the two weight sets and the kDepth
    // raw buffers are indexed statically.  Three lines while a line's words
    // fit 18 registers, fewer for longer lines so that the lookahead stays
    // within about 54 registers (beyond that the kernel spills).
    static constexpr int kDepth = kTensors * kWords <= 18 ? (es == 2 && kTensors * kWords <= 12 ? 4 : 3)
                                  : kTensors * kWords <= 24 ? 2 : 1;
    static constexpr int kUnroll = kDepth % 2 == 0 ? kDepth : 2 * kDepth;
    static constexpr int kPrefetchAhead = 8;    // lines between an L2 prefetch and its use
    static constexpr int kPrefetchLines = kUnroll;   // lines per prefetch (one per loop body)

    const DirParams &p;
    const int lane, D;
    const int L, nch;
    int total_chunks;
    LaneGeom<R> g;
    int eo[kWords];     // element offset (in a row) of each raw word, clamped into the row
    int cs[R];          // output column of each position in the staged output plane
    const char *gp[kTensors];   // the current item's planes
    // lane t < 6: byte offsets of tensor t's planes of the current and the
    // next item (-1: none), for the L2 prefetches
    long long pf_cur, pf_next;
    const bool fwd;             // top-down (else bottom-up)
    const int split;            // first step after the midpoint (see sweep_split)
    int hw[NP > 0 ? NP : 1];    // kYHalf: word of each position pair in a plane row
    int hs;                     // kYHalf: byte of the single position in a plane row

    __device__ static int pos(int lane, int r) {
        return r < 2 * NP ? 64 * (r / 2) + 2 * lane + (r & 1) : 64 * NP + lane;
    }

    __device__ RowScan(const DirParams &p_, unsigned char *, int lane_, int d)
        : p(p_), lane(lane_), D(d), L(p_.H), nch(1), total_chunks(0), pf_cur(-1), pf_next(-1),
          fwd(d == 0), split(sweep_split((p_.dirs & 3) == 3, d == 0, p_.H)) {
        const int W = p_.W;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = pos(lane_, r);
            g.valid[r] = q < W;
            g.m0[r] = q > 0 ? 1.0f : 0.0f;
            g.m2[r] = q + 1 < W ? 1.0f : 0.0f;
            g.thr[r] = __float_as_int((q > 0 && q + 1 < W) ? 1e11f : 1e5f);
            // positions past the row end write the plane's last (dummy) column
            cs[r] = q < W ? q ^ ((q >> 5) & 1) : p_.y_pitch - 1;
        }
        if (MODE == kYHalf) {
            // pairs past the row end write the dummy word; a single past the
            // end writes the dummy word's half of the lane's parity
#pragma unroll
            for (int k = 0; k < (NP > 0 ? NP : 1); ++k) hw[k] = 64 * k + 2 * lane_ < W ? 32 * k + lane_ : p_.y_pitch - 1;
            hs = 64 * NP + lane_ < W ? 4 * (32 * NP) + 2 * lane_ : 4 * (p_.y_pitch - 1) + 2 * (lane_ & 1);
        }
#pragma unroll
        for (int k = 0; k < kWords; ++k) {
            if (es == 2) {
                // a pair word covers positions (q, q+1), q even; W is even
                const int q = k < NP ? 64 * k + 2 * lane : 64 * NP + lane;
                eo[k] = k < NP ? min(q, W - 2) : min(q, W - 1);
            } else {
                eo[k] = min(pos(lane_, k), W - 1);
            }
        }
    }

    // Byte offset of tensor t's plane of the CTA's k-th item (-1: none).
    __device__ __forceinline__ long long plane_off(int k, int t) const {
        const int item = blockIdx.x + k * gridDim.x;
        if (item >= p.n_items) return -1;
        const int plane = item / p.bands;
        const int b = plane / p.Cc, ch = plane - b * p.Cc;
        return static_cast<long long>(dir_plane(p, b, ch, D, t) * es);
    }

    __device__ __forceinline__ void set_item(int k) {
#pragma unroll
        for (int t = 0; t < kTensors; ++t) gp[t] = dir_tensor(p, t) + plane_off(k, t);
        if (lane < kTensors) {
            pf_cur = plane_off(k, lane);
            pf_next = plane_off(k + 1, lane);
        }
    }

    __device__ __forceinline__ int row_of(int s) const { return fwd ? s : L - 1 - s; }

    // Raw words of scan line s (global loads, L2-resident after the prefetch).
    __device__ __forceinline__ void load(int s, Raw &w) const {
        const int base = row_of(s) * p.W;
#pragma unroll
        for (int k = 0; k < kWords; ++k) {
            const int idx = base + eo[k];
#pragma unroll
            for (int t = 0; t < kTensors; ++t) {
                if (es == 2 && k < NP) w[t][k] = __ldg(reinterpret_cast<const unsigned int *>(gp[t]) + (idx >> 1));
                else if (es == 2) w[t][k] = __ldg(reinterpret_cast<const unsigned short *>(gp[t]) + idx);
                else w[t][k] = __ldg(reinterpret_cast<const unsigned int *>(gp[t]) + idx);
            }
        }
    }

    // (weights normalised ahead are fp16 when the inputs are bf16)
    __device__ __forceinline__ static void unpack(const Raw &w, float (&v)[kTensors][R]) {
#pragma unroll
        for (int t = 0; t < kTensors; ++t)
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if constexpr (es == 4) {
                    v[t][r] = __uint_as_float(w[t][r]);
                } else {
                    const uint32_t word = r < 2 * NP ? w[t][r / 2] : w[t][NP];
                    const bool hi = r < 2 * NP && (r & 1);
                    v[t][r] = (PRE && t >= 2 && t <= 4) ? half_word<true>(word, hi) : half_word<false>(word, hi);
                }
            }
    }

    // L2 prefetch (bulk prefetch, TMA engine) of lines [s0, s0 + kPrefetchLines)
    // of the warp's line stream, which continues into its next item.
    __device__ __forceinline__ void prefetch(int s0) const {
        if (lane >= kTensors) return;
        const long long po = s0 < L ? pf_cur : pf_next;
        const int s = s0 < L ? s0 : s0 - L;
        if (po < 0 || s >= L) return;
        const int n = min(kPrefetchLines, L - s);
        const int r0 = fwd ? s : L - s - n;
        const unsigned long long end = dir_tensor_bytes(p, lane);
        unsigned long long a = static_cast<unsigned long long>(po) + static_cast<unsigned long long>(r0) * p.W * es;
        unsigned long long e = a + static_cast<unsigned long long>(n) * p.W * es;
        a &= ~15ull;
        e = (e + 15) & ~15ull;
        if (e > end) e = end & ~15ull;
        if (e > a) prefetch_l2(dir_tensor(p, lane) + a, static_cast<uint32_t>(e - a));
    }

    // Gated output of the step's row into the row plane / band / global.
    __device__ __forceinline__ void emit(const float (&h)[R], const LineW<R> &W, int row, float *ys,
                                         float *yg, int band_lo, int band_hi, bool first) const {
        const bool in = MODE != kYBanded || (row >= band_lo && row < band_hi);
        float *yl = ys + (row - band_lo) * p.y_pitch;
        if constexpr (MODE == kYHalf) {
            uint32_t *wl = reinterpret_cast<uint32_t *>(yl);
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                float2 v = make_float2(W.uu[2 * k] * h[2 * k], W.uu[2 * k + 1] * h[2 * k + 1]);
                if (!first) {
                    const uint32_t o = wl[hw[k]];
                    v.x += __uint_as_float(o << 16);
                    v.y += __uint_as_float(o & 0xffff0000u);
                }
                wl[hw[k]] = pack_bf16x2(v);
            }
            if (kSingle) {
                unsigned short *a = reinterpret_cast<unsigned short *>(reinterpret_cast<unsigned char *>(yl) + hs);
                float v = W.uu[R - 1] * h[R - 1];
                if (!first) v += __uint_as_float(static_cast<uint32_t>(*a) << 16);
                *a = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            }
        } else {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float cy = W.uu[r] * h[r];
                if (MODE == kYGlobal) {
                    if (g.valid[r]) atomicAdd(yg + static_cast<size_t>(row) * p.W + pos(lane, r), cy);
                } else if (MODE == kYShared) {
                    if (g.valid[r] && in) atomicAdd(yl + cs[r], cy);
                } else {
                    if (in) put_y(yl + cs[r], cy, first);
                }
            }
        }
    }

    // One step of the recurrence with this lane layout: positions 2l, 2l+1
    // of each 64-position block and 64 NP + l; the neighbours across lanes
    // (and across blocks, between lanes 31 and 0) come from shuffles.
    __device__ __forceinline__ void recur_rows(float (&h)[R], const LineW<R> &W) const {
        float left[R], right[R];
#pragma unroll
        for (int p2 = 0; p2 < NP; ++p2) {
            const int a = 2 * p2, b = 2 * p2 + 1;
            // left of the even position: lane-1's odd one; lane 0 takes the
            // previous block's last position from lane 31
            const float sendl = (p2 > 0 && lane == 31) ? h[a - 1] : h[b];
            left[a] = __shfl_sync(0xffffffffu, sendl, (lane + 31) & 31);
            left[b] = h[a];
            // right of the odd position: lane+1's even one; lane 31 takes
            // the next block's first position from lane 0
            const int nxt = b + 1 < R ? b + 1 : b;
            const float sendr = (b + 1 < R && lane == 0) ? h[nxt] : h[a];
            right[b] = __shfl_sync(0xffffffffu, sendr, (lane + 1) & 31);
            right[a] = h[b];
        }
        if (kSingle) {
            const int s1 = R - 1;
            const float sendl = (NP > 0 && lane == 31) ? h[s1 > 0 ? s1 - 1 : 0] : h[s1];
            left[s1] = __shfl_sync(0xffffffffu, sendl, (lane + 31) & 31);
            right[s1] = __shfl_down_sync(0xffffffffu, h[s1], 1);
        }
        float hn[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float N = fmaf(W.w1[r], h[r], W.bx[r]);
            N = fmaf(W.w0[r], left[r], N);
            hn[r] = fmaf(W.w2[r], right[r], N);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) h[r] = hn[r];
    }

    // Step s (J = s mod 2): the plain form if line s was flagged, the update
    // of line s, the weights of line s+1 (its raw words arrived two steps
    // ago), the loads of line s+3 into the freed buffer, the outputs.
    template <int J>
    __device__ __forceinline__ void step(int s, float (&h)[R], LineW<R> (&Wb)[2],
                                         Raw (&rb)[kDepth], float *ys, float *yg, int band_lo, int band_hi) {
        constexpr int cur = J & 1, nxt = (J + 1) & 1, buf = (J + 1) % kDepth;
        LineW<R> &Wc = Wb[cur];
        recur_rows(h, Wc);
        // weights of line s+1 (past the last line: stale but finite words,
        // never used) and the loads of line s+1+kDepth into the freed buffer
        // (clamped into the plane)
        float v[kTensors][R];
        unpack(rb[buf], v);
        const bool bad = next_weights<PRE>(v, g, Wb[nxt]);
        load(min(s + 1 + kDepth, L - 1), rb[buf]);
        emit(h, Wc, row_of(s), ys, yg, band_lo, band_hi, s < split);
        if (!PRE) line_terms_fix(bad, v, g, Wb[nxt]);
        if (MODE != kYGlobal && MODE != kYShared && s + 1 == split) pair_barrier(2);
    }

    template <int J>
    __device__ __forceinline__ void steps(int s, float (&h)[R], LineW<R> (&Wb)[2], Raw (&rb)[kDepth],
                                          float *ys, float *yg, int band_lo, int band_hi) {
        if constexpr (J < kUnroll) {
            if (J == 0 || s + J < L) {
                step<J>(s + J, h, Wb, rb, ys, yg, band_lo, band_hi);
                steps<J + 1>(s, h, Wb, rb, ys, yg, band_lo, band_hi);
            }
        }
    }

    // Run every line of the CTA's k-th item.
    __device__ void run_item(int k, float *ys, float *yg, int band_lo, int band_hi) {
        set_item(k);
        if (k == 0) {
            for (int s0 = 0; s0 < kPrefetchAhead; s0 += kPrefetchLines) prefetch(s0);
        }
        float h[R];
#pragma unroll
        for (int r = 0; r < R; ++r) h[r] = 0.0f;
        LineW<R> Wb[2];
        Raw rb[kDepth];
#pragma unroll
        for (int m = 0; m < kDepth; ++m) load(min(m, L - 1), rb[m]);
        {
            float v[kTensors][R];
            unpack(rb[0], v);
            first_weights<PRE>(v, g, Wb[0]);
        }
        load(min(kDepth, L - 1), rb[0]);
#pragma unroll 1
        for (int s = 0; s < L; s += kUnroll) {
            prefetch(s + kPrefetchAhead);
            steps<0>(s, h, Wb, rb, ys, yg, band_lo, band_hi);
        }
    }
};

// ---------------------------------------------------------------------------
// Column lines (directions 2 and 3).
// ---------------------------------------------------------------------------
template <typename T, int R, int MODE, bool PRE>
struct ColScan {
    static constexpr int es = sizeof(T);
    static constexpr int NS = kColStages;
    static constexpr int CH = kColStrip / es;   // columns (steps) per chunk: 8 bf16, 4 fp32
    static constexpr int NB = CH / 4;           // 4-step bodies per chunk: 2 bf16, 1 fp32
    // Two consecutive columns of a strip row are one 32-bit (bf16) or 64-bit
    // (fp32) word; a body's two word sets cover its four columns.
    using Pair = typename std::conditional<es == 2, uint32_t, uint2>::type;
    using PairSet = Pair[kTensors][R];
    static constexpr int kCopyRows = 32 / 4;    // grid rows per copy instruction (4 lanes per row)

    const DirParams &p;
    const int lane, D;
    unsigned char *const ring;
    const int L, nch;
    int total_chunks;
    LaneGeom<R> g;
    int rowq[R];        // byte offset of strip row q_r in a stage (row 0 when q_r >= H)
    bool inb[R];        // q_r is an output row of the current item
    int yoff[R];        // offset (floats; kYHalf: words) of its output row in the column plane
    float held[R];      // kYHalf: outputs of the first column of a word pair
    int issue_item;
    const char **gtab;  // [kTensors] planes of the item being issued (shared memory)
    const bool fwd;     // left-right (else right-left)
    const int split;    // first step after the midpoint (see sweep_split)
    const uint32_t selA, selB;   // byte permutations of a bf16 word's columns

    __device__ ColScan(const DirParams &p_, unsigned char *smem, int lane_, int d)
        : p(p_), lane(lane_), D(d),
          ring(smem + (d == 2 ? p_.ring[2] : p_.ring[3])),
          L(p_.W), nch((p_.W + kColStrip / static_cast<int>(sizeof(T)) - 1) /
                       (kColStrip / static_cast<int>(sizeof(T)))),
          total_chunks(0), issue_item(-1),
          gtab(reinterpret_cast<const char **>(smem + p_.bar_off + 128 + 64 * (d - 2))),
          fwd(d == 2),
          split(MODE == kYHalf && (p_.dirs & 12) == 12
                    ? (d == 2 ? 2 * ((p_.W / 2 + 1) / 2) : 2 * ((p_.W / 2) / 2))
                    : sweep_split((p_.dirs & 12) == 12, d == 2, p_.W)),
          // bf16 word -> float of its first / second column in scan order:
          // the low half (bits << 16) or the high half (bits & 0xffff0000)
          selA(d == 2 ? 0x1044u : 0x3244u), selB(d == 2 ? 0x3244u : 0x1044u) {
        g.init(lane_, p_.H);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = lane_ * R + r < p_.H ? lane_ * R + r : 0;
            rowq[r] = q * kColPitch;
        }
    }

    // bf16 strips are read 64 bits per lane (a body's four columns of a
    // tensor): lanes l < 16 read rows 3l + r, whose 104-byte pitches put
    // each half-warp's 8-byte reads on distinct bank pairs; fp32 strips are
    // read 64 bits per lane too (two columns).

    // Lowest column of chunk c (chunks are numbered in scan order).
    __device__ __forceinline__ int chunk_lo(int c) const { return fwd ? c * CH : L - CH - c * CH; }

    __device__ __forceinline__ unsigned char *stage_ptr(int gi) const {
        return ring + (gi % NS) * p.stage_col;
    }

    // The warp copies the strip: lane (i0, w) = (lane / 4, lane % 4) moves
    // word w of grid rows i0, i0 + 8, ... of every tensor (4 lanes cover
    // one row's 16 bytes, so a copy instruction reads 8 rows).
    template <bool FULL>
    __device__ __forceinline__ void copy_strip(uint32_t sb, int lo) const {
        const char *gt[kTensors];
#pragma unroll
        for (int t = 0; t < kTensors; ++t) gt[t] = gtab[t];
        const int w = lane & 3, i0 = lane >> 2;
        if (!FULL) {
            const int col = lo + w * (4 / es);
            if (col < 0 || col + 4 / es > L) return;
        }
        // right-to-left scans store the words of a strip row reversed
        const int dw = fwd ? w : 3 - w;
        const int rowstep = kCopyRows * p.W * es;
        int src_off = (i0 * p.W + lo) * es + 4 * w;
        uint32_t drow = sb + static_cast<uint32_t>(i0 * kColPitch);
#pragma unroll 1
        for (int row = i0; row < p.H; row += kCopyRows) {
            const uint32_t dst = drow + 4u * static_cast<uint32_t>(dw);
#pragma unroll
            for (int t = 0; t < kTensors; ++t) cp_async_4(dst + 16 * t, gt[t] + src_off);
            src_off += rowstep;
            drow += kCopyRows * kColPitch;
        }
    }

    // Issue (and commit as one group) the warp's copies of chunk gi.  Every
    // read of the stage it overwrites (chunk gi-2) is complete: the values
    // were consumed before this point.
    __device__ __forceinline__ void issue(int gi) {
        __syncwarp();
        if (gi < total_chunks) {
            const int kk = gi / nch;
            const int c = gi - kk * nch;
            const int item = blockIdx.x + kk * gridDim.x;
            if (item != issue_item) {
                issue_item = item;
                const int plane = item / p.bands;
                const int b = plane / p.Cc, ch = plane - b * p.Cc;
                if (lane < kTensors) gtab[lane] = dir_tensor(p, lane) + dir_plane(p, b, ch, D, lane) * es;
                __syncwarp();
            }
            const int lo = chunk_lo(c);
            const uint32_t sb = smem_u32(stage_ptr(gi));
            if (lo >= 0 && lo + CH <= L) copy_strip<true>(sb, lo);
            else copy_strip<false>(sb, lo);
        }
        cp_async_commit();
    }

    // Wait until at most N of the warp's copy groups are in flight; rows are
    // copied by other lanes than the ones that read them.
    template <int N>
    __device__ __forceinline__ void wait() const {
        cp_async_wait<N>();
        __syncwarp();
    }

    // fp32: word set of the column pair `pidx` (0..3 in scan order within a
    // strip row) of a stage, 8 bytes per tensor and position.
    __device__ __forceinline__ void load_pair(const unsigned char *sp, int pidx, PairSet &w) const {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int off = rowq[r] + 8 * pidx;
#pragma unroll
            for (int t = 0; t < kTensors; ++t)
                w[t][r] = *reinterpret_cast<const Pair *>(sp + off + 16 * t);
        }
    }

    // fp32 lines of more than 160 positions read one column per step
    // straight from the stage: two two-column word sets of six or more
    // positions per lane would hold 144+ registers and spill.
    static constexpr bool kDirect = es == 4 && R >= 6;

    // fp32: column kk (0..3 in scan order within a strip row) of a stage.
    __device__ __forceinline__ void load_col(const unsigned char *sp, int kk, float (&v)[kTensors][R]) const {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int off = rowq[r] + 4 * kk;
#pragma unroll
            for (int t = 0; t < kTensors; ++t) v[t][r] = *reinterpret_cast<const float *>(sp + off + 16 * t);
        }
    }

    // bf16: both word sets of body b (columns 4b..4b+3 in scan order) of a
    // stage, one 8-byte read per tensor and position.
    __device__ __forceinline__ void load_quad(const unsigned char *sp, int b, PairSet &A, PairSet &B) const {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int off = rowq[r] + 8 * b;
#pragma unroll
            for (int t = 0; t < kTensors; ++t) {
                const uint2 q = *reinterpret_cast<const uint2 *>(sp + off + 16 * t);
                if constexpr (es == 2) {
                    A[t][r] = q.x;
                    B[t][r] = q.y;
                }
            }
        }
    }

    // Column K (0 or 1, scan order) of a word set as floats.
    template <int K>
    __device__ __forceinline__ void unpack(const PairSet &w, float (&v)[kTensors][R]) const {
#pragma unroll
        for (int t = 0; t < kTensors; ++t)
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if constexpr (es == 4) {
                    v[t][r] = __uint_as_float(K == 0 ? w[t][r].x : w[t][r].y);
                } else if (PRE && t >= 2 && t <= 4) {
                    // fp16 weight normalised ahead: the half met K-th in scan order
                    v[t][r] = half_word<true>(w[t][r], (K == 0) != fwd);
                } else {
                    // a word holds columns (2m, 2m+1); reversed sweeps meet the odd one first
                    v[t][r] = __uint_as_float(prmt0(w[t][r], K == 0 ? selA : selB));
                }
            }
    }

    // kYHalf: the first column of a word pair (scan order) is held, the
    // second stores the pair (LR: columns 2j, 2j+1; RL: 2j+1, 2j).
    template <int J>
    __device__ __forceinline__ void emit_half(const float (&h)[R], const LineW<R> &W, int col, float *ys,
                                              bool first) {
        if constexpr ((J & 1) == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r) held[r] = W.uu[r] * h[r];
        } else {
            uint32_t *yw = reinterpret_cast<uint32_t *>(ys) + (col >> 1);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float cur = W.uu[r] * h[r];
                float2 v = fwd ? make_float2(held[r], cur) : make_float2(cur, held[r]);
                if (!first) {
                    const uint32_t o = yw[yoff[r]];
                    v.x += __uint_as_float(o << 16);
                    v.y += __uint_as_float(o & 0xffff0000u);
                }
                yw[yoff[r]] = pack_bf16x2(v);
            }
        }
    }

    // kYGlobal: the outputs of a chunk's CH columns are staged in shared
    // memory, [grid row][CH] fp32 in column order after the column ring,
    // row q at q CH + q / R (one word more per lane block, so that the
    // lanes' stores of a step fall on distinct banks), and added to the
    // output once per chunk: a row's CH columns in one 16-byte vector atomic
    // instead of CH scattered 4-byte ones.
    __device__ __forceinline__ float *ystage() const { return reinterpret_cast<float *>(ring + NS * p.stage_col); }

    // column j (column order within the chunk) of the step's outputs
    __device__ __forceinline__ void emit_stage(const float (&h)[R], const LineW<R> &W, int j) const {
        float *st = ystage();
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int q = lane * R + r;
            if (g.valid[r]) st[q * CH + j + lane] = W.uu[r] * h[r];
        }
    }

    // add the staged outputs of chunk c (n columns scanned) to the output
    __device__ __forceinline__ void flush_stage(int c, int n, float *yg) const {
        __syncwarp();
        const float *st = ystage();
        const int lo = chunk_lo(c);
        // a full chunk on a 16-byte boundary: one vector atomic per row
        const bool vec = CH == 4 && n == CH && lo >= 0 && lo % 4 == 0 && p.W % 4 == 0;
        const int j0 = fwd ? 0 : CH - n;   // the chunk's scanned columns: j0 .. j0 + n - 1
        for (int i = lane; i < p.H; i += 32) {
            const float *sr = st + i * CH + i / R;
            float *o = yg + static_cast<size_t>(i) * p.W + lo;
            if (vec) {
                atomicAdd(reinterpret_cast<float4 *>(o), make_float4(sr[0], sr[1], sr[2], sr[3]));
            } else {
                for (int j = j0; j < j0 + n; ++j) atomicAdd(o + j, sr[j]);
            }
        }
        __syncwarp();
    }

    __device__ __forceinline__ void emit(const float (&h)[R], const LineW<R> &W, int col, float *ys,
                                         float *yg, bool first) const {
        const int yc = ycol(col);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float cy = W.uu[r] * h[r];
            if (MODE == kYGlobal) {
                if (g.valid[r]) atomicAdd(yg + static_cast<size_t>(lane * R + r) * p.W + col, cy);
            } else if (MODE == kYShared) {
                if (inb[r]) atomicAdd(ys + yoff[r] + yc, cy);
            } else {
                put_y(ys + yoff[r] + yc, cy, first);
            }
        }
    }

    // Step J of body b of chunk c (launch chunk number gi; n of its CH steps
    // exist, n < CH only in the item's last chunk): steps 0-1 read word set
    // A, steps 2-3 word set B.  bf16: step 2 reads both sets of the next body
    // (from the next chunk, waited for here, when b is the chunk's last
    // body); fp32: B is read by step 0, the next body's A by step 2.  `last`
    // when chunk c ends the item.
    template <int J>
    __device__ __forceinline__ void bstep(int gi, int c, int b, bool last, int n, float (&h)[R],
                                          LineW<R> (&Wb)[2], PairSet &A, PairSet &B,
                                          float *ys, float *yg) {
        LineW<R> &Wc = Wb[J & 1];
        const int k = 4 * b + J;   // step within the chunk
        if (k >= n) return;
        const int st = c * CH + k;  // step within the item
        recur(h, Wc);
        const bool more = b + 1 < NB || !last;   // a step follows this body's last
        // weights of the next step (when none follows: stale but finite
        // words, never used)
        float v[kTensors][R];
        if constexpr (kDirect) {
            // the next step's column, read from the stage now
            if (J < 3) {
                load_col(stage_ptr(gi), J + 1, v);
            } else if (more) {
                wait<0>();               // chunk gi+1 (issued when chunk gi was entered)
                load_col(stage_ptr(gi + 1), 0, v);
            } else {
                load_col(stage_ptr(gi), 3, v);
            }
        } else if (J == 0) {
            unpack<1>(A, v);
        } else if (J == 1) {
            unpack<0>(B, v);
        } else if (J == 2) {
            unpack<1>(B, v);
        } else {
            unpack<0>(A, v);
        }
        // word sets of the steps ahead, read after the step's last use of
        // the set they replace
        if constexpr (kDirect) {
        } else if constexpr (es == 2) {
            if (J == 2 && more) {
                if (b + 1 < NB) {
                    load_quad(stage_ptr(gi), b + 1, A, B);
                } else {
                    wait<0>();           // chunk gi+1 (issued when chunk gi was entered)
                    load_quad(stage_ptr(gi + 1), 0, A, B);
                }
            }
        } else {
            if (J == 0) load_pair(stage_ptr(gi), 2 * b + 1, B);
            if (J == 2 && more) {
                if (b + 1 < NB) {
                    load_pair(stage_ptr(gi), 2 * b + 2, A);
                } else {
                    wait<0>();           // chunk gi+1 (issued when chunk gi was entered)
                    load_pair(stage_ptr(gi + 1), 0, A);
                }
            }
        }
        const bool bad = next_weights<PRE>(v, g, Wb[(J + 1) & 1]);
        if constexpr (MODE == kYHalf) emit_half<J>(h, Wc, fwd ? st : L - 1 - st, ys, st < split);
        else if constexpr (MODE == kYGlobal) emit_stage(h, Wc, fwd ? k : CH - 1 - k);
        else emit(h, Wc, fwd ? st : L - 1 - st, ys, yg, st < split);
        if (!PRE) line_terms_fix(bad, v, g, Wb[(J + 1) & 1]);
        if (MODE != kYGlobal && MODE != kYShared && st + 1 == split) pair_barrier(3);
    }

    // Run every column of the item whose first chunk is g0.
    __device__ void run_item(int g0, float *ys, float *yg, int band_lo, int band_hi) {
        float h[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            h[r] = 0.0f;
            const int q = lane * R + r;
            inb[r] = g.valid[r] && (MODE != kYBanded || (q >= band_lo && q < band_hi));
            // rows outside the band (or past the end) write the plane's dummy row
            yoff[r] = (inb[r] ? q - band_lo : p.band_rows) * p.y_pitch;
        }
        LineW<R> Wb[2];
        PairSet A, B;
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
            const int gi = g0 + c;
            // entering chunk gi: the stage of chunk gi-1 is free for gi+1
            issue(gi + 1);
            if (c == 0) {
                // the item's first chunk: wait for it, weights of step 0
                wait<1>();
                float v[kTensors][R];
                if constexpr (kDirect) {
                    load_col(stage_ptr(gi), 0, v);
                } else {
                    if constexpr (es == 2) load_quad(stage_ptr(gi), 0, A, B);
                    else load_pair(stage_ptr(gi), 0, A);
                    unpack<0>(A, v);
                }
                first_weights<PRE>(v, g, Wb[0]);
            }
            const bool last = c + 1 == nch;
            const int n = min(CH, L - c * CH);
#pragma unroll 1
            for (int b = 0; b < NB; ++b) {
                bstep<0>(gi, c, b, last, n, h, Wb, A, B, ys, yg);
                bstep<1>(gi, c, b, last, n, h, Wb, A, B, ys, yg);
                bstep<2>(gi, c, b, last, n, h, Wb, A, B, ys, yg);
                bstep<3>(gi, c, b, last, n, h, Wb, A, B, ys, yg);
            }
            if constexpr (MODE == kYGlobal) flush_stage(c, n, yg);
        }
    }
};

// Barrier of the CTA's four warps.  The warps run different code paths (one
// per direction), so the barrier is a named PTX barrier with an explicit
// thread count rather than __syncthreads.
__device__ __forceinline__ void dir_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(kDirThreads) : "memory");
}

// The whole kernel seen from the warp that runs direction D.
template <typename T, int R, bool ROW, int MODE, bool PRE>
__device__ __forceinline__ void dir_role(const DirParams &p, unsigned char *smem, int warp, int lane, int D) {
    // output planes (or bands), fp32 [rows][y_pitch]: rows, then columns
    float *ysr = reinterpret_cast<float *>(smem);
    float *ysc = reinterpret_cast<float *>(smem + p.ycol_off);
    const bool has_row = (p.dirs & 3) != 0, has_col = (p.dirs & 12) != 0;
    const int YP = p.y_pitch;
    const bool active = (p.dirs >> D) & 1;
    const int n_my = blockIdx.x < p.n_items ? (p.n_items - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    using Scan = typename std::conditional<ROW, RowScan<T, R, MODE, PRE>, ColScan<T, R, MODE, PRE>>::type;
    Scan sc(p, smem, lane, D);
    const int total = active ? n_my * sc.nch : 0;
    sc.total_chunks = total;
    // column lines: the first chunk; each chunk entered later issues the next
    if constexpr (!ROW) {
        if (active) sc.issue(0);
    }

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
        if (active) sc.run_item(ROW ? k : k * sc.nch, (ROW || MODE == kYShared) ? ysr : ysc, yg, band_lo, band_hi);
        dir_barrier();
        if (MODE != kYGlobal) {
            // the sum of the two planes, written out once (converted); every
            // position of a plane is stored again by the next item
            T *outp = static_cast<T *>(p.out) + static_cast<size_t>(plane) * p.H * p.W +
                      static_cast<size_t>(band_lo) * p.W;
            if constexpr (MODE == kYHalf) {
                // word j of a plane row holds columns 2j, 2j+1 (W is even)
                const uint32_t *wr = reinterpret_cast<const uint32_t *>(ysr);
                const uint32_t *wc = reinterpret_cast<const uint32_t *>(ysc);
                uint32_t *ow = reinterpret_cast<uint32_t *>(outp);
                const int nw = p.W / 2;
                for (int i = warp; i < p.H; i += 4) {
                    for (int j = lane; j < nw; j += 32) {
                        float2 v = make_float2(0.0f, 0.0f);
                        if (has_row) {
                            const uint32_t o = wr[i * YP + j];
                            v.x += __uint_as_float(o << 16);
                            v.y += __uint_as_float(o & 0xffff0000u);
                        }
                        if (has_col) {
                            const uint32_t o = wc[i * YP + j];
                            v.x += __uint_as_float(o << 16);
                            v.y += __uint_as_float(o & 0xffff0000u);
                        }
                        ow[static_cast<size_t>(i) * nw + j] = pack_bf16x2(v);
                    }
                }
            } else {
                for (int i = warp; i < band_hi - band_lo; i += 4) {
                    float *yr = ysr + i * YP;
                    const float *yc = ysc + i * YP;
                    T *orow = outp + static_cast<size_t>(i) * p.W;
                    for (int j = lane; j < p.W; j += 32) {
                        const int c = ycol(j);
                        if (MODE == kYShared) {
                            // the single plane is accumulated into: clear it
                            orow[j] = from_f<T>(yr[c]);
                            yr[c] = 0.0f;
                        } else {
                            const float v = (has_row ? yr[c] : 0.0f) + (has_col ? yc[c] : 0.0f);
                            orow[j] = from_f<T>(v);
                        }
                    }
                }
            }
            dir_barrier();
        }
    }
    if (!ROW) cp_async_wait<0>();
}

// Lines of up to 64 positions run four CTAs (16 warps) per SM, a budget of
// 128 registers per thread (a few spill for fp32; measured 28 % faster on
// 37x37 planes than three CTAs); lines of up to 96 keep three (168
// registers: capping them at 128 was slower); longer lines two.
template <typename T, int R, int MODE, bool PRE>
__global__ void __launch_bounds__(kDirThreads, R <= 2 ? 4 : R <= 3 ? 3 : 2)
prop2d_dir_kernel(const DirParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Zero the output plane and the rings: staged slots then never hold
    // non-finite values, also where positions past a line's end read them.
    {
        uint4 *z = reinterpret_cast<uint4 *>(smem);
        for (int e = threadIdx.x; e < p.bar_off / 16; e += kDirThreads) z[e] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    // the two sweeps of an orientation share one code path (the sweep sign
    // is a runtime value), which halves the instruction footprint
    if (warp < 2) dir_role<T, R, true, MODE, PRE>(p, smem, warp, lane, warp);
    else dir_role<T, R, false, MODE, PRE>(p, smem, warp, lane, warp);
}

}  // namespace gspn
