// Fused Prop2D forward with the two sweeps of an orientation in one warp.
//
// One CTA of two warps owns one (batch, channel) plane at a time (persistent
// CTAs stride over the planes).  Warp 0 runs the row lines: its lanes 0-15
// sweep top->bottom (direction slot 0) and lanes 16-31 bottom->top (slot 1).
// Warp 1 runs the column lines: lanes 0-15 left->right (slot 2), lanes 16-31
// right->left (slot 3).  Every position of a line is updated from three
// neighbours of the previous line ("Scaling Parallel Sequence Models to
// Foundation-Scale Vision Encoders", Sec. 3 "Line-scan recurrence"; the
// papernotes.org summary's operator and normalisation formula):
//
//     h_l(q) = sum_k w_l(q,k) h_{l-1}(q+k-1) + lambda_l(q) x_l(q),   y += u_l(q) h_l(q)
//
// Lane layout (both orientations).  Lane hl of a half-warp holds the 2*RP
// consecutive positions 2*RP*hl .. 2*RP*hl + 2*RP - 1 (RP pairs) and NS
// single positions 32*RP + 16*i + hl.  A pair is two neighbouring positions,
// so a bf16 pair of a row line is one aligned 32-bit word and every pair is
// one packed f32x2 operand.  Neighbours held by other lanes of the half-warp
// come from four shuffles per step.
//
// Output.  The two sweeps of an orientation add into one fp32 plane of
// their own: at step s the forward sweep reaches line s and the backward
// sweep line L-1-s, so the sweep that reaches a line first stores and the
// other adds.  Both are lanes of one warp, so program order (with a warp
// barrier) orders the store before the add: no atomics, no barrier between
// warps.  The column plane is kept transposed ([column][row]) so that both
// orientations store pair blocks the same way.  After both warps finished a
// plane they meet at a CTA barrier, add the two planes, convert and write
// the output once.
//
// Normalisation (Sec. 5.1 "Fused CUDA normalization": sigmoid, local sum,
// clamp, divide), folded into the update.  With a_k = 1 + exp(-z_k),
// sigmoid(z_k) = 1 / a_k, P_k = product of the other two a_j and
// D = sum over on-grid k of P_k, the normalised weights are P_k / D, and
//
//     h = (P0 h(q-1) + P1 h(q) + P2 h(q+1)) * (1 / D) + lambda x
//
// An off-grid slot (q = 0 for k = 0, q = M-1 for k = 2) is left out of D and
// meets a zero neighbour; its a_k is a common factor of the other two P
// and cancels.  Three exponentials and one reciprocal per position.  The
// clamp of the local sum at 1e-6 can only bind when D > 1e5, and a product
// that overflows (or a non-finite logit) gives an infinite or NaN D; a step
// with any such D in the warp is recomputed in the plain form
// (sigmoid, explicit clamp, divide).  The weights of line s+1 are computed
// during step s.
//
// Inputs.  Row lines are read straight from global memory (one 32-bit word
// per bf16 pair, lookahead of D_ROW lines in registers, L2 bulk prefetch
// ahead of that).  Column lines go through a ring of strips in shared
// memory: a strip holds 16 bytes of every grid row of each of the six
// tensors (8 bf16 or 4 fp32 columns), copied with 4-byte cp.async so that
// every grid row lands at a fixed pitch; right->left sweeps store the words
// of a strip row in reverse, so both sweeps meet their columns in scan
// order.  A four-step body (bf16) reads each position's columns with one
// 8-byte shared load per tensor.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace gspn {

constexpr int kPairThreads = 64;     // warp 0: row lines, warp 1: column lines
constexpr int kTensorsP = 6;         // lambda, u, logits k = 0..2, x
constexpr int kPairStages = 2;       // column ring depth, in strips
constexpr int kPairRowWords = 24;    // 32-bit words per grid row of a strip stage (6 tensors x 16 B)
constexpr int kPairSkewWords = 2;    // extra words after each group of 2*RP grid rows (bank skew)

struct PairParams {
    // tensor bases; wl0/wl1/wl2 are the logit slots k = 0, 1, 2 of plane 0
    const char *x, *lam, *u, *wl0, *wl1, *wl2;
    void *out;
    int B, Cc, H, W, dirs;
    int gate_dirs;          // direction slots of lambda and u: 4, or 1 shared by all directions
    int w_groups, w_cpg;    // logit fields per (batch, direction) and channels per field
    int n_items;
    int yp;                 // floats per line of an output plane
    int q_off;              // byte offset of the column plane
    int ring_off;           // byte offset of the column rings (one per sweep)
    int stage_bytes;        // bytes of one ring stage of one sweep
    unsigned int x_bytes, g_bytes, w_bytes;   // byte sizes of x, lambda (= u) and the logits
};

// ---------------------------------------------------------------------------
// packed f32x2 arithmetic
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 splat2(float a) { return make_float2(a, a); }
// bf16 pair word -> (low half, high half) as fp32
__device__ __forceinline__ float2 bf16x2_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// ---------------------------------------------------------------------------
// One step's inputs and terms for the lane's positions
// ---------------------------------------------------------------------------
template <int RP, int NS>
struct PairVals {
    static constexpr int RA = RP > 0 ? RP : 1;
    float2 v[kTensorsP][RA];   // tensors: 0 lambda, 1 u, 2..4 logits k = 0..2, 5 x
    float s[kTensorsP][NS];
};

template <int RP, int NS>
struct PairTerms {
    static constexpr int RA = RP > 0 ? RP : 1;
    float2 P0[RA], P1[RA], P2[RA], r[RA], bx[RA], u[RA];
    float P0s[NS], P1s[NS], P2s[NS], rs[NS], bxs[NS], us[NS];
};

// Per-lane constants of a line of M positions.
template <int RP, int NS>
struct PairGeom {
    static constexpr int RA = RP > 0 ? RP : 1;
    static constexpr int NP = 2 * RP;
    float2 m0[RA], m2[RA];   // 1 where neighbour slot 0 / 2 is on the grid
    float m0s[NS], m2s[NS];
    bool vs[NS];             // single i is a position of the line
    uint32_t vp_bits;        // bit j: pair-block position j is a position of the line
    bool left_edge;          // hl == 0: position 0 has no left neighbour
    __device__ __forceinline__ void init(int hl, int M) {
        vp_bits = 0;
#pragma unroll
        for (int p = 0; p < RP; ++p) {
            const int q0 = NP * hl + 2 * p, q1 = q0 + 1;
            m0[p] = make_float2(q0 > 0 ? 1.f : 0.f, 1.f);
            m2[p] = make_float2(q1 < M ? 1.f : 0.f, q1 + 1 < M ? 1.f : 0.f);
            vp_bits |= (q0 < M ? 1u : 0u) << (2 * p);
            vp_bits |= (q1 < M ? 1u : 0u) << (2 * p + 1);
        }
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int q = 32 * RP + 16 * i + hl;
            m0s[i] = q > 0 ? 1.f : 0.f;
            m2s[i] = q + 1 < M ? 1.f : 0.f;
            vs[i] = q < M;
        }
        left_edge = hl == 0;
    }
};

// Fast form of one step's terms; returns true when some D is outside the
// form's range (above 1e5, infinite or NaN: compared as integer bit patterns,
// where the hardware's NaN is above every finite value).
template <int RP, int NS>
__device__ __forceinline__ bool pair_terms(const PairVals<RP, NS> &V, const PairGeom<RP, NS> &g,
                                           PairTerms<RP, NS> &T) {
    constexpr float nl2e = -1.4426950408889634f;
    int dmax = 0;
#pragma unroll
    for (int p = 0; p < RP; ++p) {
        const float2 t0 = mul2(V.v[2][p], splat2(nl2e));
        const float2 t1 = mul2(V.v[3][p], splat2(nl2e));
        const float2 t2 = mul2(V.v[4][p], splat2(nl2e));
        const float2 a0 = add2(make_float2(ex2(t0.x), ex2(t0.y)), splat2(1.f));
        const float2 a1 = add2(make_float2(ex2(t1.x), ex2(t1.y)), splat2(1.f));
        const float2 a2 = add2(make_float2(ex2(t2.x), ex2(t2.y)), splat2(1.f));
        const float2 P0 = mul2(a1, a2), P1 = mul2(a0, a2), P2 = mul2(a0, a1);
        const float2 D = fma2(g.m2[p], P2, fma2(g.m0[p], P0, P1));
        dmax = max(dmax, max(__float_as_int(D.x), __float_as_int(D.y)));
        T.P0[p] = P0;
        T.P1[p] = P1;
        T.P2[p] = P2;
        T.r[p] = make_float2(rcp(D.x), rcp(D.y));
        T.bx[p] = mul2(V.v[0][p], V.v[5][p]);
        T.u[p] = V.v[1][p];
    }
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const float a0 = ex2(V.s[2][i] * nl2e) + 1.f;
        const float a1 = ex2(V.s[3][i] * nl2e) + 1.f;
        const float a2 = ex2(V.s[4][i] * nl2e) + 1.f;
        const float P0 = a1 * a2, P1 = a0 * a2, P2 = a0 * a1;
        const float D = fmaf(g.m2s[i], P2, fmaf(g.m0s[i], P0, P1));
        dmax = max(dmax, __float_as_int(D));
        T.P0s[i] = P0;
        T.P1s[i] = P1;
        T.P2s[i] = P2;
        T.rs[i] = rcp(D);
        T.bxs[i] = V.s[0][i] * V.s[5][i];
        T.us[i] = V.s[1][i];
    }
    return dmax > 0x47C35000;   // bits of 1e5f
}

// Plain form of one position (rare path): off-grid slots weigh 0, sigmoids
// saturate instead of overflowing, and the clamp of the local sum is explicit.
__device__ __forceinline__ void plain_pos(float z0, float z1, float z2, float m0, float m2,
                                          float &P0, float &P1, float &P2, float &r) {
    constexpr float nl2e = -1.4426950408889634f;
    const float s0 = m0 != 0.f ? rcp(1.f + ex2(z0 * nl2e)) : 0.f;
    const float s1 = rcp(1.f + ex2(z1 * nl2e));
    const float s2 = m2 != 0.f ? rcp(1.f + ex2(z2 * nl2e)) : 0.f;
    P0 = s0;
    P1 = s1;
    P2 = s2;
    r = rcp(fmaxf((s0 + s1) + s2, 1e-6f));
}

template <int RP, int NS>
__device__ __forceinline__ void pair_terms_plain(const PairVals<RP, NS> &V, const PairGeom<RP, NS> &g,
                                              PairTerms<RP, NS> &T) {
#pragma unroll
    for (int p = 0; p < RP; ++p) {
        plain_pos(V.v[2][p].x, V.v[3][p].x, V.v[4][p].x, g.m0[p].x, g.m2[p].x, T.P0[p].x,
                  T.P1[p].x, T.P2[p].x, T.r[p].x);
        plain_pos(V.v[2][p].y, V.v[3][p].y, V.v[4][p].y, g.m0[p].y, g.m2[p].y, T.P0[p].y,
                  T.P1[p].y, T.P2[p].y, T.r[p].y);
    }
#pragma unroll
    for (int i = 0; i < NS; ++i)
        plain_pos(V.s[2][i], V.s[3][i], V.s[4][i], g.m0s[i], g.m2s[i], T.P0s[i], T.P1s[i],
                  T.P2s[i], T.rs[i]);
}

// Hidden state of the lane's positions.
template <int RP, int NS>
struct PairState {
    static constexpr int RA = RP > 0 ? RP : 1;
    float2 h[RA];
    float hs[NS];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int p = 0; p < RA; ++p) h[p] = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < NS; ++i) hs[i] = 0.f;
    }
};

// One step of the recurrence.  Neighbours across lanes (within the
// half-warp): the pair block's left neighbour is the previous lane's last
// pair position (none at the line's start), its right neighbour the next
// lane's first pair position (lane 15: single 0 of lane 0).  Single i's
// neighbours are the previous / next lane's single i; lane 0's left one is
// lane 15's last pair position (i = 0) or single i-1, lane 15's right one
// lane 0's single i+1 (none after the last single).
template <int RP, int NS>
__device__ __forceinline__ void pair_recur(PairState<RP, NS> &S, const PairTerms<RP, NS> &T,
                                           const PairGeom<RP, NS> &g, int hl, bool pairs_valid) {
    constexpr unsigned FULL = 0xffffffffu;
    const int base = threadIdx.x & 16;
    const int prv = base | ((hl + 15) & 15), nxt = base | ((hl + 1) & 15);
    float leftP = 0.f, rightP = 0.f, a = 0.f;
    if constexpr (RP > 0) {
        a = __shfl_sync(FULL, S.h[RP - 1].y, prv);
        leftP = g.left_edge ? 0.f : a;
        rightP = __shfl_sync(FULL, hl == 0 ? S.hs[0] : S.h[0].x, nxt);
    }
    float sl[NS], sr[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const float c = __shfl_sync(FULL, (i > 0 && hl == 15) ? S.hs[i > 0 ? i - 1 : 0] : S.hs[i], prv);
        const float d = __shfl_sync(FULL, (i + 1 < NS && hl == 0) ? S.hs[i + 1 < NS ? i + 1 : i] : S.hs[i], nxt);
        sl[i] = (i == 0 && hl == 0) ? a : c;
        sr[i] = (i + 1 == NS && hl == 15) ? 0.f : d;
    }
    float2 hn[PairState<RP, NS>::RA];
#pragma unroll
    for (int p = 0; p < RP; ++p) {
        const float2 hc = S.h[p];
        const float2 hlf = make_float2(p == 0 ? leftP : S.h[p > 0 ? p - 1 : 0].y, hc.x);
        const float2 hrt = make_float2(hc.y, p + 1 < RP ? S.h[p + 1 < RP ? p + 1 : p].x : rightP);
        float2 N = mul2(T.P1[p], hc);
        N = fma2(T.P0[p], hlf, N);
        N = fma2(T.P2[p], hrt, N);
        hn[p] = fma2(N, T.r[p], T.bx[p]);
    }
    float hsn[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        float N = T.P1s[i] * S.hs[i];
        N = fmaf(T.P0s[i], sl[i], N);
        N = fmaf(T.P2s[i], sr[i], N);
        hsn[i] = fmaf(N, T.rs[i], T.bxs[i]);
    }
#pragma unroll
    for (int p = 0; p < RP; ++p) S.h[p] = hn[p];
    // positions past the line's end stay 0 (one of them is the right
    // neighbour of the last position); pair blocks hold such positions only
    // on lines shorter than the blocks
#pragma unroll
    for (int i = 0; i < NS; ++i) S.hs[i] = g.vs[i] ? hsn[i] : 0.f;
    if (!pairs_valid) {
#pragma unroll
        for (int p = 0; p < RP; ++p) {
            S.h[p].x = (g.vp_bits >> (2 * p)) & 1 ? S.h[p].x : 0.f;
            S.h[p].y = (g.vp_bits >> (2 * p + 1)) & 1 ? S.h[p].y : 0.f;
        }
    }
}

// Gated outputs u * h of one line into an output plane line `Y` (shared
// memory): STORE, or ADD to what the other sweep stored.  The planes hold
// the input/output element type: fp32, or bf16 for bf16 inputs (the sum of
// two directions rounded to bf16 once per sweep; the final sum of the two
// planes is formed in fp32).

template <int RP, int NS, bool ADD>
__device__ __forceinline__ void pair_emit(float *Y, int hl, const PairState<RP, NS> &S,
                                          const PairTerms<RP, NS> &T) {
    if constexpr (RP == 2) {
        float4 *a = reinterpret_cast<float4 *>(Y + 4 * hl);
        const float2 y0 = mul2(T.u[0], S.h[0]), y1 = mul2(T.u[1], S.h[1]);
        if (ADD) {
            const float4 o = *a;
            const float2 s0 = add2(y0, make_float2(o.x, o.y)), s1 = add2(y1, make_float2(o.z, o.w));
            *a = make_float4(s0.x, s0.y, s1.x, s1.y);
        } else {
            *a = make_float4(y0.x, y0.y, y1.x, y1.y);
        }
    } else {
#pragma unroll
        for (int p = 0; p < RP; ++p) {
            float2 *a = reinterpret_cast<float2 *>(Y + 2 * RP * hl + 2 * p);
            const float2 y = mul2(T.u[p], S.h[p]);
            *a = ADD ? add2(y, *a) : y;
        }
    }
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        float *a = Y + 32 * RP + 16 * i + hl;
        const float y = T.us[i] * S.hs[i];
        *a = ADD ? y + *a : y;
    }
}

template <int RP, int NS, bool ADD>
__device__ __forceinline__ void pair_emit(__nv_bfloat16 *Y, int hl, const PairState<RP, NS> &S,
                                          const PairTerms<RP, NS> &T) {
    if constexpr (RP == 2) {
        uint2 *a = reinterpret_cast<uint2 *>(Y + 4 * hl);
        float2 y0 = mul2(T.u[0], S.h[0]), y1 = mul2(T.u[1], S.h[1]);
        if (ADD) {
            const uint2 o = *a;
            y0 = add2(y0, bf16x2_f2(o.x));
            y1 = add2(y1, bf16x2_f2(o.y));
        }
        *a = make_uint2(pack_bf16x2(y0), pack_bf16x2(y1));
    } else {
#pragma unroll
        for (int p = 0; p < RP; ++p) {
            uint32_t *a = reinterpret_cast<uint32_t *>(Y + 2 * RP * hl + 2 * p);
            float2 y = mul2(T.u[p], S.h[p]);
            if (ADD) y = add2(y, bf16x2_f2(*a));
            *a = pack_bf16x2(y);
        }
    }
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        __nv_bfloat16 *a = Y + 32 * RP + 16 * i + hl;
        float y = T.us[i] * S.hs[i];
        if (ADD) y += __bfloat162float(*a);
        *a = __float2bfloat16_rn(y);
    }
}

// Output of step s: the sweep that reaches its line first stores, the other
// adds; on the middle line of an odd count both arrive together and the
// backward sweep adds after the forward one.  `wen`: this half's direction
// is enabled (else it stores nothing); `both`: both sweeps are enabled.
template <int RP, int NS, typename YT>
__device__ __forceinline__ void pair_output(YT *ybase, int yp, int s, int L, bool fwd, bool wen,
                                            bool both, int hl, const PairState<RP, NS> &S,
                                            const PairTerms<RP, NS> &T) {
    const int line = fwd ? s : L - 1 - s;
    YT *Y = ybase + line * yp;
    const int twice = 2 * s;
    if (!both || twice < L - 1) {
        if (wen) pair_emit<RP, NS, false>(Y, hl, S, T);
    } else if (twice > L - 1) {
        if (wen) pair_emit<RP, NS, true>(Y, hl, S, T);
    } else {
        if (fwd) pair_emit<RP, NS, false>(Y, hl, S, T);
        __syncwarp();
        if (!fwd) pair_emit<RP, NS, true>(Y, hl, S, T);
    }
}

__device__ __forceinline__ void pair_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(kPairThreads) : "memory");
}

// Plane index (b, c) of an item and the byte offsets of its planes.
struct PairPlane {
    uint32_t og, ow, ox;   // lambda/u plane of direction d, logit slot 0 plane, x plane
};
__device__ __forceinline__ PairPlane pair_plane(const PairParams &p, int item, int d, int es) {
    const int b = item / p.Cc, c = item - b * p.Cc;
    const uint32_t hw = static_cast<uint32_t>(p.H) * p.W * es;
    PairPlane r;
    r.og = static_cast<uint32_t>((b * p.gate_dirs + (p.gate_dirs == 4 ? d : 0)) * p.Cc + c) * hw;
    r.ow = static_cast<uint32_t>((b * 4 + d) * p.w_groups + c / p.w_cpg) * 3u * hw;
    r.ox = static_cast<uint32_t>(b * p.Cc + c) * hw;
    return r;
}

__device__ __forceinline__ const char *pair_tensor(const PairParams &p, int t) {
    return t == 0 ? p.lam : t == 1 ? p.u : t == 2 ? p.wl0 : t == 3 ? p.wl1 : t == 4 ? p.wl2 : p.x;
}

// Direction slot a half-warp reads: its own, or (when its own is not
// enabled) its partner's, whose planes are then read twice and nothing is
// stored; enabled slots only are ever read.
__device__ __forceinline__ int pair_read_dir(int dirs, int d0, int half) {
    const int own = d0 + half, other = d0 + 1 - half;
    return ((dirs >> own) & 1) ? own : other;
}

// ---------------------------------------------------------------------------
// Row lines (warp 0)
// ---------------------------------------------------------------------------
template <typename T, int RP, int NS>
struct PairRows {
    static constexpr int es = sizeof(T);
    static constexpr int NP = 2 * RP;
    static constexpr int RA = RP > 0 ? RP : 1;
    // raw words of one line: bf16 one word per pair, fp32 two; one per single
    static constexpr int KP = es == 2 ? RP : 2 * RP;
    static constexpr int KA = KP > 0 ? KP : 1;
    struct Raw {
        uint32_t p[kTensorsP][KA];
        uint32_t s[kTensorsP][NS];
    };
    // lines of lookahead in registers; the loop body is UNROLL steps, a
    // multiple of both DEPTH (the raw buffers) and 2 (the two weight sets),
    // so that every buffer is indexed statically
    static constexpr int DEPTH = (KP + NS) * kTensorsP <= 18 ? 4 : (KP + NS) * kTensorsP <= 30 ? 3 : 2;
    static constexpr int UNROLL = DEPTH % 2 ? 2 * DEPTH : DEPTH;
    static constexpr int PF_AHEAD = 16;   // lines between an L2 prefetch and its use

    const PairParams &p;
    const int hl, half;
    const bool fwd;
    const int L, M;
    PairGeom<RP, NS> g;
    bool wen, both, pairs_valid;
    int line_bytes;            // bytes between consecutive lines (+-W*es)
    // running byte offsets of the next line to load: pair block / singles
    uint32_t og, ow, ox;
    uint32_t sg[NS], sw[NS], sx[NS];
    uint32_t pf_cur, pf_next;  // lane t < 6 of each half: plane offset of tensor t (0xffffffff: none)
    int next_load;             // scan index of the next line to load

    __device__ PairRows(const PairParams &p_, int lane)
        : p(p_), hl(lane & 15), half(lane >> 4), fwd((lane >> 4) == 0), L(p_.H), M(p_.W) {
        g.init(hl, M);
        wen = (p.dirs >> half) & 1;
        both = (p.dirs & 3) == 3;
        pairs_valid = NP * 16 <= M;
        line_bytes = fwd ? M * es : -M * es;
    }

    __device__ __forceinline__ uint32_t tensor_plane(int item, int t) const {
        if (item >= p.n_items) return 0xffffffffu;
        const PairPlane pl = pair_plane(p, item, pair_read_dir(p.dirs, 0, half), es);
        const uint32_t hw = static_cast<uint32_t>(p.H) * p.W * es;
        return t < 2 ? pl.og : t < 5 ? pl.ow + static_cast<uint32_t>(t - 2) * hw : pl.ox;
    }

    __device__ __forceinline__ void set_item(int k) {
        const int item = blockIdx.x + k * gridDim.x;
        const PairPlane pl = pair_plane(p, item, pair_read_dir(p.dirs, 0, half), es);
        const uint32_t row0 = static_cast<uint32_t>(fwd ? 0 : L - 1) * M * es;
        const uint32_t cp = static_cast<uint32_t>(NP * hl) * es;
        og = pl.og + row0 + cp;
        ow = pl.ow + row0 + cp;
        ox = pl.ox + row0 + cp;
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int q = min(32 * RP + 16 * i + hl, M - 1);
            const uint32_t cs = static_cast<uint32_t>(q) * es;
            sg[i] = pl.og + row0 + cs;
            sw[i] = pl.ow + row0 + cs;
            sx[i] = pl.ox + row0 + cs;
        }
        next_load = 0;
        if (hl < kTensorsP) {
            pf_cur = tensor_plane(item, hl);
            pf_next = tensor_plane(item + gridDim.x, hl);
        }
    }

    __device__ __forceinline__ static uint32_t ld32(const char *base, uint32_t off) {
        return __ldg(reinterpret_cast<const unsigned int *>(base + off));
    }
    __device__ __forceinline__ static uint32_t ld16(const char *base, uint32_t off) {
        return __ldg(reinterpret_cast<const unsigned short *>(base + off));
    }

    // Raw words of the next line (the last line again once past it).
    __device__ __forceinline__ void load(Raw &w) {
#pragma unroll
        for (int t = 0; t < kTensorsP; ++t) {
            const char *base = pair_tensor(p, t);
            const uint32_t o = t < 2 ? og : t < 5 ? ow : ox;
#pragma unroll
            for (int k = 0; k < KP; ++k) w.p[t][k] = ld32(base, o + 4u * k);
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                const uint32_t so = t < 2 ? sg[i] : t < 5 ? sw[i] : sx[i];
                w.s[t][i] = es == 2 ? ld16(base, so) : ld32(base, so);
            }
        }
        if (++next_load < L) {
            og += line_bytes;
            ow += line_bytes;
            ox += line_bytes;
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                sg[i] += line_bytes;
                sw[i] += line_bytes;
                sx[i] += line_bytes;
            }
        }
    }

    __device__ __forceinline__ static void unpack(const Raw &w, PairVals<RP, NS> &V) {
#pragma unroll
        for (int t = 0; t < kTensorsP; ++t) {
#pragma unroll
            for (int q = 0; q < RP; ++q) {
                if constexpr (es == 2) V.v[t][q] = bf16x2_f2(w.p[t][q]);
                else V.v[t][q] = make_float2(__uint_as_float(w.p[t][2 * q]), __uint_as_float(w.p[t][2 * q + 1]));
            }
#pragma unroll
            for (int i = 0; i < NS; ++i)
                V.s[t][i] = es == 2 ? __uint_as_float(w.s[t][i] << 16) : __uint_as_float(w.s[t][i]);
        }
    }

    // L2 prefetch (TMA engine) of lines [s0, s0 + n) of the half's stream,
    // which continues into the CTA's next item.
    __device__ __forceinline__ void prefetch(int s0, int n) const {
        if (hl >= kTensorsP) return;
        const uint32_t po = s0 < L ? pf_cur : pf_next;
        const int s = s0 < L ? s0 : s0 - L;
        if (po == 0xffffffffu || s >= L) return;
        n = min(n, L - s);
        const int r0 = fwd ? s : L - s - n;
        const unsigned long long end = hl < 2 ? p.g_bytes : hl < 5 ? p.w_bytes : p.x_bytes;
        const char *base = hl < 2 ? (hl == 0 ? p.lam : p.u) : hl < 5 ? p.wl0 : p.x;
        unsigned long long a = po + static_cast<unsigned long long>(r0) * M * es;
        unsigned long long e = a + static_cast<unsigned long long>(n) * M * es;
        a &= ~15ull;
        e = (e + 15) & ~15ull;
        if (e > end) e = end & ~15ull;
        if (e > a) prefetch_l2(base + a, static_cast<uint32_t>(e - a));
    }

    template <int J>
    __device__ __forceinline__ void step(int s, PairState<RP, NS> &S, PairTerms<RP, NS> (&Tb)[2],
                                         Raw (&rb)[DEPTH], T *Yr) {
        constexpr int cur = J & 1, nx = (J + 1) & 1, buf = (J + 1) % DEPTH;
        pair_recur<RP, NS>(S, Tb[cur], g, hl, pairs_valid);
        PairVals<RP, NS> V;
        unpack(rb[buf], V);
        const bool bad = pair_terms<RP, NS>(V, g, Tb[nx]);
        load(rb[buf]);
        pair_output<RP, NS>(Yr, p.yp, s, L, fwd, wen, both, hl, S, Tb[cur]);
        if (__any_sync(0xffffffffu, bad)) pair_terms_plain<RP, NS>(V, g, Tb[nx]);
    }

    template <int J>
    __device__ __forceinline__ void steps(int s, PairState<RP, NS> &S, PairTerms<RP, NS> (&Tb)[2],
                                          Raw (&rb)[DEPTH], T *Yr) {
        if constexpr (J < UNROLL) {
            if (J == 0 || s + J < L) {
                step<J>(s + J, S, Tb, rb, Yr);
                steps<J + 1>(s, S, Tb, rb, Yr);
            }
        }
    }

    __device__ void run_item(int k, T *Yr) {
        set_item(k);
        if (k == 0) prefetch(0, PF_AHEAD);
        PairState<RP, NS> S;
        S.zero();
        PairTerms<RP, NS> Tb[2];
        Raw rb[DEPTH];
#pragma unroll
        for (int m = 0; m < DEPTH; ++m) load(rb[m]);
        {
            PairVals<RP, NS> V;
            unpack(rb[0], V);
            if (__any_sync(0xffffffffu, pair_terms<RP, NS>(V, g, Tb[0]))) pair_terms_plain<RP, NS>(V, g, Tb[0]);
        }
        load(rb[0]);
#pragma unroll 1
        for (int s = 0; s < L; s += UNROLL) {
            prefetch(s + PF_AHEAD, UNROLL);
            steps<0>(s, S, Tb, rb, Yr);
        }
    }
};

// ---------------------------------------------------------------------------
// Column lines (warp 1)
// ---------------------------------------------------------------------------
template <typename T, int RP, int NS>
struct PairCols {
    static constexpr int es = sizeof(T);
    static constexpr int NP = 2 * RP;
    static constexpr int RA = RP > 0 ? RP : 1;
    static constexpr int R = NP + NS;
    static constexpr int CH = 16 / es;        // columns per strip: 8 bf16, 4 fp32
    static constexpr int BODY = es == 2 ? 4 : 2;   // steps per 8-byte word set
    static constexpr int NB = CH / BODY;      // bodies per strip (2)
    static constexpr int NSTG = kPairStages;
    // one 8-byte read per position and tensor: (w.x, w.y) = columns of a body
    struct Words {
        uint2 w[kTensorsP][R];
    };

    const PairParams &p;
    const int hl, half;
    const bool fwd;
    const int L, M;           // L = W column lines of M = H positions
    const int nstrip;
    PairGeom<RP, NS> g;
    bool wen, both, pairs_valid;
    unsigned char *ring;      // this half's ring
    uint32_t rowoff[R];       // byte offset of position r's grid row in a stage
    uint32_t selA, selB;      // bf16 word -> first / second column in scan order
    int total;                // strips this sweep copies (all items)
    int issue_item;
    uint32_t cg, cw, cx;      // plane offsets (lambda/u, logit 0, x) of the item being copied

    __device__ PairCols(const PairParams &p_, unsigned char *smem, int lane)
        : p(p_), hl(lane & 15), half(lane >> 4), fwd((lane >> 4) == 0), L(p_.W), M(p_.H),
          nstrip((p_.W + 16 / static_cast<int>(sizeof(T)) - 1) / (16 / static_cast<int>(sizeof(T)))) {
        g.init(hl, M);
        wen = (p.dirs >> (2 + half)) & 1;
        both = (p.dirs & 12) == 12;
        pairs_valid = NP * 16 <= M;
        ring = smem + p.ring_off + half * NSTG * p.stage_bytes;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            int q = r < NP ? NP * hl + r : 32 * RP + 16 * (r - NP) + hl;
            q = min(q, M - 1);
            rowoff[r] = ring_row(q);
        }
        // a bf16 word holds columns (2m, 2m+1); right->left sweeps meet the odd one first
        selA = fwd ? 0x1044u : 0x3244u;
        selB = fwd ? 0x3244u : 0x1044u;
        issue_item = -1;
    }

    __device__ __forceinline__ unsigned char *stage(int gi) const { return ring + (gi % NSTG) * p.stage_bytes; }

    // Lowest column of strip m of the sweep.
    __device__ __forceinline__ int strip_lo(int m) const { return fwd ? m * CH : L - CH - m * CH; }

    // Copy strip gi (this half's sweep, global strip counter) into its stage
    // and commit one group (possibly empty).  Lane (i0, w) = (hl / 4, hl % 4)
    // copies word w of grid rows i0, i0 + 4, ... of the six tensors, so one
    // copy instruction moves 16 contiguous bytes of each of eight grid rows
    // (four per sweep); right->left sweeps store the words of a strip row in
    // reverse, so both sweeps meet their columns in scan order.  Words
    // outside the line (ragged last strip) are skipped.
    __device__ __forceinline__ uint32_t ring_row(int row) const {
        constexpr int grp = RP > 0 ? NP : 1;
        return static_cast<uint32_t>(row * kPairRowWords + (row / grp) * kPairSkewWords) * 4u;
    }
    __device__ __forceinline__ void issue(int gi) {
        if (gi < total) {
            const int kk = gi / nstrip, m = gi - kk * nstrip;
            const int item = blockIdx.x + kk * gridDim.x;
            if (item != issue_item) {
                issue_item = item;
                const PairPlane pl = pair_plane(p, item, pair_read_dir(p.dirs, 2, half), es);
                cg = pl.og;
                cw = pl.ow;
                cx = pl.ox;
            }
            const int w = hl & 3, i0 = hl >> 2;
            const int ws = fwd ? w : 3 - w;            // source word of slot w
            const int col = strip_lo(m) + ws * (4 / es);
            if (col >= 0 && col + 4 / es <= L) {
                const long long row_bytes = static_cast<long long>(p.W) * es;
                const long long off = static_cast<long long>(i0) * row_bytes + static_cast<long long>(col) * es;
                const char *s0 = p.lam + cg + off, *s1 = p.u + cg + off, *s2 = p.wl0 + cw + off;
                const char *s3 = p.wl1 + cw + off, *s4 = p.wl2 + cw + off, *s5 = p.x + cx + off;
                const long long step = 4 * row_bytes;
                const uint32_t sb = smem_u32(stage(gi)) + 4u * w;
#pragma unroll 1
                for (int row = i0; row < M; row += 4) {
                    const uint32_t d = sb + ring_row(row);
                    cp_async_4(d, s0);
                    cp_async_4(d + 16, s1);
                    cp_async_4(d + 32, s2);
                    cp_async_4(d + 48, s3);
                    cp_async_4(d + 64, s4);
                    cp_async_4(d + 80, s5);
                    s0 += step; s1 += step; s2 += step; s3 += step; s4 += step; s5 += step;
                }
            }
        }
        cp_async_commit();
    }

    // Wait until the strip before the newest NSTG - 1 committed ones has
    // landed (copies were made by other lanes than the readers).
    __device__ __forceinline__ void wait_stage() const {
        cp_async_wait<NSTG - 1>();
        __syncwarp();
    }

    // Word sets of body b of strip stage `sp`.
    __device__ __forceinline__ void read(const unsigned char *sp, int b, Words &Wd) const {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < kTensorsP; ++t)
                Wd.w[t][r] = *reinterpret_cast<const uint2 *>(sp + rowoff[r] + 16 * t + 8 * b);
    }

    // Column K (0 .. BODY-1, scan order) of a word set as values.
    template <int K>
    __device__ __forceinline__ void unpack(const Words &Wd, PairVals<RP, NS> &V) const {
#pragma unroll
        for (int t = 0; t < kTensorsP; ++t) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float f;
                if constexpr (es == 4) {
                    f = __uint_as_float(K == 0 ? Wd.w[t][r].x : Wd.w[t][r].y);
                } else {
                    const uint32_t word = K < 2 ? Wd.w[t][r].x : Wd.w[t][r].y;
                    f = __uint_as_float(prmt0(word, (K & 1) == 0 ? selA : selB));
                }
                if (r < NP) {
                    if (r & 1) V.v[t][r / 2].y = f;
                    else V.v[t][r / 2].x = f;
                } else {
                    V.s[t][r - NP] = f;
                }
            }
        }
    }

    // Step K of a body (n steps of it exist): recurrence with the current
    // terms, terms of the next step from `nxt` (column K+1 of this body, or
    // column 0 of the next body's words), output.
    template <int K>
    __device__ __forceinline__ void bstep(int st, PairState<RP, NS> &S, PairTerms<RP, NS> (&Tb)[2],
                                          const Words &cur, const Words &nxtw, T *Yc) {
        pair_recur<RP, NS>(S, Tb[K & 1], g, hl, pairs_valid);
        PairVals<RP, NS> V;
        if constexpr (K + 1 < BODY) unpack<K + 1>(cur, V);
        else unpack<0>(nxtw, V);
        const bool bad = pair_terms<RP, NS>(V, g, Tb[(K + 1) & 1]);
        pair_output<RP, NS>(Yc, p.yp, st, L, fwd, wen, both, hl, S, Tb[K & 1]);
        if (__any_sync(0xffffffffu, bad)) pair_terms_plain<RP, NS>(V, g, Tb[(K + 1) & 1]);
    }

    // L2 prefetch (TMA engine) of the planes the item's column sweeps read:
    // lanes 0-5 of each half take lambda, u, the three logit slots of its
    // direction and (half 0) x; one bulk prefetch of a whole plane each.
    __device__ __forceinline__ void prefetch_item(int item) const {
        if (item >= p.n_items || hl >= kTensorsP || (half == 1 && hl == kTensorsP - 1)) return;
        const PairPlane pl = pair_plane(p, item, pair_read_dir(p.dirs, 2, half), es);
        const uint32_t hw = static_cast<uint32_t>(p.H) * p.W * es;
        const uint32_t off = hl < 2 ? pl.og : hl < 5 ? pl.ow + (hl - 2) * hw : pl.ox;
        const unsigned long long end = hl < 2 ? p.g_bytes : hl < 5 ? p.w_bytes : p.x_bytes;
        const char *base = hl == 0 ? p.lam : hl == 1 ? p.u : hl < 5 ? p.wl0 : p.x;
        unsigned long long a = off & ~15u, e = (static_cast<unsigned long long>(off) + hw + 15) & ~15ull;
        if (e > end) e = end & ~15ull;
        if (e > a) prefetch_l2(base + a, static_cast<uint32_t>(e - a));
    }

    // Every column of the item whose first strip is g0.
    __device__ void run_item(int g0, T *Yc) {
        const int item = blockIdx.x + (g0 / nstrip) * gridDim.x;
        if (g0 == 0) prefetch_item(item);
        PairState<RP, NS> S;
        S.zero();
        PairTerms<RP, NS> Tb[2];
        Words A, B;
        // first strip of the item
        issue(g0 + NSTG - 1);
        wait_stage();
        read(stage(g0), 0, A);
        {
            PairVals<RP, NS> V;
            unpack<0>(A, V);
            if (__any_sync(0xffffffffu, pair_terms<RP, NS>(V, g, Tb[0]))) pair_terms_plain<RP, NS>(V, g, Tb[0]);
        }
        const int nbody = nstrip * NB;
#pragma unroll 1
        for (int bi = 0; bi < nbody; bi += 2) {
            // body bi (words A) and bi+1 (words B) of strip gi = g0 + bi / 2
            const int gi = g0 + bi / NB;
            const int st0 = bi * BODY;
            read(stage(gi), 1, B);
            bstep<0>(st0 + 0, S, Tb, A, B, Yc);
            if (st0 + 1 < L) bstep<1>(st0 + 1, S, Tb, A, B, Yc);
            if constexpr (BODY == 4) {
                if (st0 + 2 < L) bstep<2>(st0 + 2, S, Tb, A, B, Yc);
                if (st0 + 3 < L) bstep<3>(st0 + 3, S, Tb, A, B, Yc);
            }
            if (st0 + BODY >= L) break;
            // halfway through the item: the next item's planes into L2
            if (bi == 2 * (nstrip / 2)) prefetch_item(item + gridDim.x);
            // next strip: its copies were issued NSTG - 1 strips ago
            const bool more = bi + 2 < nbody;
            if (more) {
                issue(gi + NSTG);
                wait_stage();
                read(stage(gi + 1), 0, A);
            }
            const int st1 = st0 + BODY;
            bstep<0>(st1 + 0, S, Tb, B, A, Yc);
            if (st1 + 1 < L) bstep<1>(st1 + 1, S, Tb, B, A, Yc);
            if constexpr (BODY == 4) {
                if (st1 + 2 < L) bstep<2>(st1 + 2, S, Tb, B, A, Yc);
                if (st1 + 3 < L) bstep<3>(st1 + 3, S, Tb, B, A, Yc);
            }
        }
    }
};

// Sum of the row plane and the transposed column plane (in fp32),
// converted and written once.  Thread (warp w, lane j) takes grid rows
// i0 .. i0+3 (i0 = 4w, 4w + 8, ...) of column j: one 4-element read of the
// column plane (conflict-free: its line pitch is an odd number of 4-element
// units) and four reads of the row plane.
__device__ __forceinline__ void load4(const float *p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 a = *reinterpret_cast<const uint2 *>(p);
    const float2 lo = bf16x2_f2(a.x), hi = bf16x2_f2(a.y);
    v[0] = lo.x; v[1] = lo.y; v[2] = hi.x; v[3] = hi.y;
}

template <typename T>
__device__ __forceinline__ void pair_combine(const PairParams &p, const T *Yr, const T *Yc, int item) {
    const bool has_row = (p.dirs & 3) != 0, has_col = (p.dirs & 12) != 0;
    T *out = static_cast<T *>(p.out) + static_cast<size_t>(item) * p.H * p.W;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i0 = 4 * warp; i0 < p.H; i0 += 8) {
        for (int j = lane; j < p.W; j += 32) {
            float q[4] = {0.f, 0.f, 0.f, 0.f};
            if (has_col) load4(Yc + j * p.yp + i0, q);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (i0 + k < p.H) {
                    const float r = has_row ? to_f(Yr[(i0 + k) * p.yp + j]) : 0.f;
                    out[static_cast<size_t>(i0 + k) * p.W + j] = from_f<T>(r + q[k]);
                }
            }
        }
    }
}

template <typename T, int RP, int NS>
__global__ void __launch_bounds__(kPairThreads, 4) prop2d_pair_kernel(const PairParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    T *Yr = reinterpret_cast<T *>(smem);
    T *Yc = reinterpret_cast<T *>(smem + p.q_off);
    // zero the rings: slots no copy reaches (ragged strips) then hold
    // finite values where steps past a line's end read them
    {
        uint4 *z = reinterpret_cast<uint4 *>(smem + p.ring_off);
        const int n = 2 * kPairStages * p.stage_bytes / 16;
        for (int e = threadIdx.x; e < n; e += kPairThreads) z[e] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    const int n_my = blockIdx.x < p.n_items ? (p.n_items - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    if (warp == 0) {
        PairRows<T, RP, NS> rows(p, lane);
        const bool act = (p.dirs & 3) != 0;
        for (int k = 0; k < n_my; ++k) {
            if (act) rows.run_item(k, Yr);
            pair_barrier();
            pair_combine<T>(p, Yr, Yc, blockIdx.x + k * gridDim.x);
            pair_barrier();
        }
    } else {
        PairCols<T, RP, NS> cols(p, smem, lane);
        const bool act = (p.dirs & 12) != 0;
        cols.total = act ? n_my * cols.nstrip : 0;
        // prologue: the first NSTG - 1 strips
        for (int i = 0; i < kPairStages - 1; ++i) cols.issue(i);
        for (int k = 0; k < n_my; ++k) {
            if (act) cols.run_item(k * cols.nstrip, Yc);
            pair_barrier();
            pair_combine<T>(p, Yr, Yc, blockIdx.x + k * gridDim.x);
            pair_barrier();
        }
        cp_async_wait<0>();
    }
}

}  // namespace gspn
