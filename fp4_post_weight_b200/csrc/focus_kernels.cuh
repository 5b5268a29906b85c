// focus_kernels.cuh -- sm_100a kernels of the FOCUS NVFP4 weight fake-quantizer.
//
// Source of the arithmetic: model card "FOCUS NVFP4 scales for
// Llama-3.2-1B-Instruct (our reproduction)", section "What this is" (the S_b,
// c_i and w'_i equations and the rules after them) and section "Calibration"
// (AdamW on m and q); the straight-through estimator of "Technische
// Samenvatting: FOCUS ...", section "Methodologie", item 1.
//
// Work decomposition.  A tensor W[out, in] with in % 16 == 0 is a flat array of
// nblk = out*in/16 blocks: m[blk] and q[2*blk + k] index it directly, whatever
// the row length.  Work is cut into tiles of TILE_BLOCKS blocks; a persistent
// grid walks the tiles of every tensor of a table.
//
// Staging.  Each CTA runs one producer warp and NC_WARPS consumer warps over a
// ring of shared-memory stages (focus_pipeline.cuh).  For a full tile the
// producer issues one 1-D bulk copy per input array (W, dW', m, q, the AdamW
// moments), all completing on the stage's mbarrier; a partial tile (the ragged
// end of a tensor) is read by the consumers straight from global memory.  The
// prefetch depth is therefore set by the number of stages, not by registers.
//
// Inside a tile each 16-block is owned by one consumer thread: it takes the
// block's 32 bytes of W (and of dW') from the stage, its m, its two q and
// their moments, and does the block's work (A_b, x_b, S_b, the m-gradient and
// its AdamW update) once.  The forward and backward kinds store their outputs
// from registers straight to global memory (W' as two 16-byte streaming
// stores per block, the codes as 8 bytes).  The step leaves its outputs in the
// block's slots of the stage (W' over W, m, q and the moments over theirs, the
// codes and scales in two regions of their own); the producer writes a full
// tile out with one bulk copy per array once the consumers release the stage,
// and each thread of a ragged tile copies its block's out itself.
//
// Besides the FOCUS kinds (forward, backward, fused step) the same pipeline
// runs FourOverSix round to nearest and plain NVFP4 round to nearest of
// weights (KIND_F46 and KIND_RTN: W alone is staged); the
// per-token kernel (FourOverSix or NVFP4, row-major or 128x4 scales), the
// scale relayout and the standalone AdamW below are plain grid-stride kernels.
//
// Exactness.  Forward decisions (S_b, codes, w') are taken in binary32 with
// explicit round-to-nearest intrinsics (__fmul_rn / __fdiv_rn cannot be fused
// or reassociated by the compiler); sigmoid is evaluated in binary64 and
// rounded once.  The hardware conversions cvt.rn.satfinite.{e4m3x2,e2m1x2}.f32
// round to nearest even; the E4M3 input is always inside [2^-6, 448], where
// every E4M3 value is normal.  The sigmoid is evaluated with few binary64
// operations and rounded only when the rounding is certain (focus_device.cuh);
// the result equals the direct evaluation bit for bit.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "focus.h"
#include "focus_device.cuh"
#include "focus_pipeline.cuh"

namespace focus {

constexpr int NC_WARPS = 8;                      // consumer warps per CTA
constexpr int CONSUMERS = NC_WARPS * 32;         // consumer threads
constexpr int CTA_THREADS = CONSUMERS + 32;      // plus one producer warp
constexpr int THREADS = 256;                     // threads of the other kernels
constexpr int TILE_BLOCKS = CONSUMERS;           // 16-blocks per tile (4096 weights): one per consumer thread
constexpr unsigned FULL = 0xffffffffu;

// Sticky error word read by focus_get_error(): bit 0 a non-finite input,
// bit 1 a table entry skipped (an invalid tensor scale, or a pointer its
// kernel needs missing), bit 2 a non-finite gradient, bit 3 a pipeline wait
// that ran out.
// (This header is compiled into exactly one translation unit.)
__device__ unsigned int g_error_flags = 0;

enum Kind : int { KIND_FWD = 0, KIND_BWD = 1, KIND_STEP = 2, KIND_F46 = 3, KIND_RTN = 4 };

// Which inputs a kind reads besides W: dW' (and the gradient accumulators),
// and the scale parameters m and q.  FourOverSix and plain round to nearest
// read W alone.
__host__ __device__ constexpr bool has_grad(int kind) { return kind == KIND_BWD || kind == KIND_STEP; }
__host__ __device__ constexpr bool has_mq(int kind) { return kind != KIND_F46 && kind != KIND_RTN; }

// The byte offsets of the input and output regions of one shared-memory stage
// (defined with the tile engine below).
template <int KIND> struct Layout;

struct Args {
    const focus_tensor_desc *table;  // device table, or nullptr: use `one`
    int n_tensors;
    int64_t total_tiles;
    focus_tensor_desc one;           // the single tensor of the one-tensor entry points
    float one_s2;                    // its tensor scale (by value)
    float *one_scale_out;            // pack: where the tensor scale is exported (or nullptr)
    int write_wq;                    // forward and step: write W' where the descriptor has it
    int accumulate;                  // bwd: add into dm/dq; step: FOCUS_STEP_ACCUMULATE
    int write_grad;                  // step: FOCUS_STEP_WRITE_GRAD
    int pack_updated;                // step: FOCUS_STEP_PACK_UPDATED
    uint32_t *amax_ws;               // step: per-tensor max |w| (bf16 magnitude bits) for the next s2, or nullptr
    Hyper hp;
};

// The step's options fixed at compile time: SF is a mask of the SF_* bits
// (FOCUS_STEP_ACCUMULATE, _WRITE_GRAD, _PACK_UPDATED and the tensor maxima of
// focus_step_fused_amax), or SF_RUNTIME to read them from Args.  The launcher
// picks a kernel compiled for the caller's options where one exists; the
// specialised kernels carry neither the run-time tests nor the registers of
// the inputs their options leave unused (3% of the step's time, measured).
// FOCUS_STEP_WQ_UPDATED is the separate template argument WQU here, and the
// bit SF_WQU in the MXFP4 kernels.
enum : int { SF_ACC = 1, SF_WRITE_GRAD = 2, SF_PACK = 4, SF_WQU = 8, SF_AMAX = 16, SF_RUNTIME = -1 };

template <int SF>
struct StepOpt {
    static __device__ __forceinline__ bool acc(const Args &a) { return SF < 0 ? a.accumulate != 0 : (SF & SF_ACC) != 0; }
    static __device__ __forceinline__ bool write_grad(const Args &a) {
        return SF < 0 ? a.write_grad != 0 : (SF & SF_WRITE_GRAD) != 0;
    }
    static __device__ __forceinline__ bool pack(const Args &a) {
        return SF < 0 ? a.pack_updated != 0 : (SF & SF_PACK) != 0;
    }
    static __device__ __forceinline__ bool amax(const Args &a) {
        return SF < 0 ? a.amax_ws != nullptr : (SF & SF_AMAX) != 0;
    }
};

// ---------------------------------------------------------------------------
// tensor lookup
// ---------------------------------------------------------------------------

struct TensorRef {
    focus_tensor_desc d;
    int64_t nblk;
    int64_t tile_end;
    float s2;
    float den;      // fl(6 * s2)
    float rden;     // fl(1 / den)
    float den4;     // fl(4 * s2) (FourOverSix)
    float rden4;    // fl(1 / den4)
    bool den_ok;    // den inside the range where the quotient by rden is exact
    bool den46_ok;  // den and den4 both inside it
    bool ok;        // s2 usable
};

__device__ __forceinline__ void load_tensor(const Args &a, int t, TensorRef &r) {
    if (a.table) {
        r.d = a.table[t];
        r.s2 = *r.d.s2;
    } else {
        r.d = a.one;
        r.s2 = a.one_s2;
    }
    r.nblk = r.d.out * (r.d.in / 16);
    r.tile_end = r.d.tile_begin + (r.nblk + TILE_BLOCKS - 1) / TILE_BLOCKS;
    r.ok = (r.s2 > 0.0f) && finitef(r.s2);
    r.den = __fmul_rn(6.0f, r.s2);
    r.den_ok = r.ok && r.den >= 0x1p-60f && r.den <= 0x1p60f;
    r.rden = r.den_ok ? rcp_rn(r.den) : 0.0f;
    r.den4 = __fmul_rn(4.0f, r.s2);
    r.den46_ok = r.den_ok && r.den4 >= 0x1p-60f && r.den4 <= 0x1p60f;
    r.rden4 = r.den46_ok ? rcp_rn(r.den4) : 0.0f;
}

// ---------------------------------------------------------------------------
// the tile engine
// ---------------------------------------------------------------------------

// One 16-block's inputs as its consumer thread holds them.
struct Block {
    uint32_t w[8];          // W, bf16 pairs
    uint32_t g[8];          // dW', bf16 pairs
    float m, mv1, mv2;
    float q[2], qv1[2], qv2[2];
    float gm_in, gq_in[2];
    uint32_t blk;           // block index within its tensor (tensors hold fewer than 2^31 blocks)
    bool valid;
};

// A block's inputs straight from global memory (ragged tiles).
template <int KIND, int SF, class TV>
__device__ __forceinline__ void load_block_global(const TV &T, const Args &a, Block &B, uint32_t blk) {
    B.blk = blk;
    B.valid = blk < (uint32_t)T.nblk;
    if (!B.valid) {
#pragma unroll
        for (int j = 0; j < 8; ++j) B.w[j] = B.g[j] = 0u;
        B.m = 1.0f; B.mv1 = B.mv2 = 0.0f; B.gm_in = 0.0f;
#pragma unroll
        for (int k = 0; k < 2; ++k) { B.q[k] = 0.0f; B.qv1[k] = B.qv2[k] = 0.0f; B.gq_in[k] = 0.0f; }
        return;
    }
    const uint4 *W = reinterpret_cast<const uint4 *>(T.d.W) + 2u * blk;
    const uint4 w0 = __ldcs(W), w1 = __ldcs(W + 1);
    B.w[0] = w0.x; B.w[1] = w0.y; B.w[2] = w0.z; B.w[3] = w0.w;
    B.w[4] = w1.x; B.w[5] = w1.y; B.w[6] = w1.z; B.w[7] = w1.w;
    if (has_grad(KIND)) {
        const uint4 *G = reinterpret_cast<const uint4 *>(T.d.dWq) + 2u * blk;
        const uint4 g0 = __ldcs(G), g1 = __ldcs(G + 1);
        B.g[0] = g0.x; B.g[1] = g0.y; B.g[2] = g0.z; B.g[3] = g0.w;
        B.g[4] = g1.x; B.g[5] = g1.y; B.g[6] = g1.z; B.g[7] = g1.w;
    }
    if (has_mq(KIND)) {
        B.m = T.d.m[blk];
        const float2 q = reinterpret_cast<const float2 *>(T.d.q)[blk];
        B.q[0] = q.x; B.q[1] = q.y;
    }
    if (KIND == KIND_STEP) {
        B.mv1 = T.d.m_exp_avg[blk];
        B.mv2 = T.d.m_exp_avg_sq[blk];
        const float2 v1 = reinterpret_cast<const float2 *>(T.d.q_exp_avg)[blk];
        const float2 v2 = reinterpret_cast<const float2 *>(T.d.q_exp_avg_sq)[blk];
        B.qv1[0] = v1.x; B.qv1[1] = v1.y; B.qv2[0] = v2.x; B.qv2[1] = v2.y;
    }
    if (has_grad(KIND) && StepOpt<SF>::acc(a)) {
        B.gm_in = T.d.dm[blk];
        const float2 gq = reinterpret_cast<const float2 *>(T.d.dq)[blk];
        B.gq_in[0] = gq.x; B.gq_in[1] = gq.y;
    }
}

// x_b = fl(fl(A*m) / fl(6*s2)).  With |A*m| and 6*s2 in [2^-60, 2^60] the
// quotient and every intermediate of the correction stay normal, and the
// quotient comes from the tensor's reciprocal of 6*s2 (two Markstein
// corrections, correctly rounded); elsewhere from the IEEE division.
template <class TV>
__device__ __forceinline__ float scaled_max(const TV &T, float A, float m) {
    const float Am = __fmul_rn(A, m);
    const float aAm = fabsf(Am);
    if (T.den_ok && aAm <= 0x1p60f && (aAm >= 0x1p-60f || aAm == 0.0f)) return div_full(Am, T.den, T.rden);
    return div_rn_slow(Am, T.den);
}

// NVFP4 codes and E4M3 scale byte of one block for block factor m and
// sub-block logits q0, q1 (the forward's decisions only).
// The sub-block sigmoids come from sigmoid_step with the forward's binary64
// sigmoids (s0, s1 at the logits q0_old, q1_old), bit-identical to evaluating
// them afresh.  (A warp vote per sub-block between this checked code and an
// unchecked fast path, as the forward has, measured no faster here.)
template <class TV>
__device__ __forceinline__ void encode_block(const TV &T, const uint32_t *w, float A, float m, float q0, float q1,
                                             double s0, double s1, float q0_old, float q1_old, uint32_t &sbyte,
                                             uint32_t codes[2]) {
    const float x = scaled_max(T, A, m);
    float xc = (x == 0.0f) ? 1.0f : x;
    xc = fminf(fmaxf(xc, 0x1p-6f), 448.0f);
    sbyte = e4m3_byte(xc);
    const float S = e4m3_normal_f32(sbyte);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float sig = k ? sigmoid_step(s1, q1_old, q1) : sigmoid_step(s0, q0_old, q0);
        const float D = __fmul_rn(__fmul_rn(S, sig), T.s2);
        uint32_t code = 0u;
        if (D >= 0x1p-60f && D <= 0x1p60f && A <= 0x1p60f) {
            const float nr = -rcp_rn(D);
            const uint64_t D2 = f2_pack(D, D), nr2 = f2_pack(nr, nr);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint64_t y2 = div_by_f2(bf16x2_neg_f2(w[4 * k + j]), D2, nr2);
                code |= e2m1_pair(f2_lo(y2), f2_hi(y2)) << (8 * j);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                code |= e2m1_pair(div_rn_slow(bf16_lo(w[4 * k + j]), D), div_rn_slow(bf16_hi(w[4 * k + j]), D)) << (8 * j);
        }
        codes[k] = code;
    }
}

// w' = bf16(fl(fl(c*S)*s2)) of one block from its two code words and scale byte,
// to global memory, or (SO) to the block's W slot of the stage at so.
template <bool SO = false, int KIND = KIND_STEP, class TV>
__device__ __forceinline__ void store_wq_from_codes(const TV &T, uint32_t blk, const uint32_t codes[2], uint32_t sbyte,
                                                    unsigned char *so = nullptr, uint32_t lb = 0) {
    const uint16_t S_h = (uint16_t)e4m3_normal_f16_bits(sbyte);
    const uint64_t s2_2 = f2_pack(T.s2, T.s2);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t h2 = e2m1_pair_f16x2((codes[k] >> (8 * j)) & 0xffu);
            const uint64_t p = f2_mul(f2_pack(mul_f16_exact(lo16(h2), S_h), mul_f16_exact(hi16(h2), S_h)), s2_2);
            o[j] = pack_bf16x2(f2_lo(p), f2_hi(p));
        }
        if constexpr (SO)
            reinterpret_cast<uint4 *>(so + Layout<KIND>::W)[2u * lb + (uint32_t)k] = make_uint4(o[0], o[1], o[2], o[3]);
        else
            __stcs(reinterpret_cast<uint4 *>(T.d.Wq) + (2u * blk + (uint32_t)k), make_uint4(o[0], o[1], o[2], o[3]));
    }
}

// ---------------------------------------------------------------------------
// FourOverSix round to nearest (model card, section "Calibration": each
// 16-element block's scale maps the block maximum to 6 or to 4, whichever has
// the lower error; section "Perplexity": round-to-nearest FourOverSix weights)
// ---------------------------------------------------------------------------

// The scales a FourOverSix block needs from its tensor (or token) scale s:
// the quotient denominators fl(6*s), fl(4*s), their correctly rounded
// reciprocals, and whether both lie in [2^-60, 2^60], where the quotient by
// the reciprocal (div_full) is exact.
struct F46Scale {
    float s, den6, rden6, den4, rden4;
    bool den_ok;
    bool fast;   // den_ok and s in [2^-54, 2^51], so that every D = S*s (S in [2^-6, 448]) is in [2^-60, 2^60]
};

__device__ __forceinline__ bool f46_scale_fast(bool den_ok, float s) {
    return den_ok && s >= 0x1p-54f && s <= 0x1p51f;
}

__device__ __forceinline__ F46Scale f46_scale(float s) {
    F46Scale c;
    c.s = s;
    c.den6 = __fmul_rn(6.0f, s);
    c.den4 = __fmul_rn(4.0f, s);
    c.den_ok = c.den6 >= 0x1p-60f && c.den6 <= 0x1p60f && c.den4 >= 0x1p-60f && c.den4 <= 0x1p60f;
    c.rden6 = c.den_ok ? rcp_rn(c.den6) : 0.0f;
    c.rden4 = c.den_ok ? rcp_rn(c.den4) : 0.0f;
    c.fast = f46_scale_fast(c.den_ok, s);
    return c;
}

// x_T = fl(A / den) for A >= 0: the Markstein quotient where it is exact,
// the IEEE division elsewhere.
__device__ __forceinline__ float f46_x(float A, float den, float rden, bool den_ok) {
    if (den_ok && A <= 0x1p60f && (A >= 0x1p-60f || A == 0.0f)) return div_full(A, den, rden);
    return div_rn_slow(A, den);
}

// Scale byte, its value, its binary16 bits and D = fl(S*s) of target x.
struct F46Target {
    uint32_t sb;
    float D, nr;          // D and -fl(1/D) (0 when D is outside the fast range)
    uint16_t S_h;
    bool fast;
};

__device__ __forceinline__ F46Target f46_target(float x, float s, float A) {
    F46Target t;
    x = (x == 0.0f) ? 1.0f : x;
    x = fminf(fmaxf(x, 0x1p-6f), 448.0f);
    t.sb = e4m3_byte(x);
    t.S_h = (uint16_t)e4m3_normal_f16_bits(t.sb);
    t.D = __fmul_rn(e4m3_normal_f32(t.sb), s);
    t.fast = t.D >= 0x1p-60f && t.D <= 0x1p60f && A <= 0x1p60f;
    t.nr = t.fast ? -rcp_rn(t.D) : 0.0f;
    return t;
}

// Both targets of a block whose scale is fast (sc.fast) and whose maximum A
// lies in [2^-60, 2^60] or is 0, bit for bit what f46_target(f46_x(...)) gives
// each: the two scaled maxima x_6 = fl(A/fl(6s)), x_4 = fl(A/fl(4s)) as one
// packed pair (div_full's Markstein steps, lane by lane), 1 for a zero block,
// clamped below at 2^-6 (the conversion's saturation is the clamp at 448),
// both E4M3 bytes from one conversion, and D_T = fl(S_T*s) as one packed
// product, which lies in [2^-60, 2^60] by sc.fast.
__device__ __forceinline__ void f46_targets_fast(float A, const F46Scale &sc, F46Target &t6, F46Target &t4) {
    const uint64_t A2 = f2_pack(A, A);
    const uint64_t r2 = f2_pack(sc.rden6, sc.rden4);
    const uint64_t nd2 = f2_pack(-sc.den6, -sc.den4);
    uint64_t q = f2_mul(A2, r2);
    uint64_t e = f2_fma(q, nd2, A2);
    q = f2_fma(e, r2, q);
    e = f2_fma(q, nd2, A2);
    q = f2_fma(e, r2, q);
    float x6 = f2_lo(q), x4 = f2_hi(q);
    if (A == 0.0f) x6 = x4 = 1.0f;
    x6 = fmaxf(x6, 0x1p-6f);
    x4 = fmaxf(x4, 0x1p-6f);
    uint16_t sbs;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(sbs) : "f"(x4), "f"(x6));
    t6.sb = (uint32_t)sbs & 0xffu;
    t4.sb = (uint32_t)sbs >> 8;
    t6.S_h = (uint16_t)e4m3_normal_f16_bits(t6.sb);
    t4.S_h = (uint16_t)e4m3_normal_f16_bits(t4.sb);
    const uint64_t D2 = f2_mul(f2_pack(e4m3_normal_f32(t6.sb), e4m3_normal_f32(t4.sb)), f2_pack(sc.s, sc.s));
    t6.D = f2_lo(D2);
    t4.D = f2_hi(D2);
    t6.nr = -rcp_rn(t6.D);
    t4.nr = -rcp_rn(t4.D);
    t6.fast = t4.fast = true;
}

// The quotient pair y = w / D of one pair of weights under a target.  FAST:
// from the reciprocal (nw the negated pair, D2, nr2 = (D, D), (-fl(1/D), ...));
// else IEEE division.
template <bool FAST>
__device__ __forceinline__ uint64_t f46_quot(uint64_t nw, uint32_t wv, float D, uint64_t D2, uint64_t nr2) {
    if (FAST) return div_by_f2(nw, D2, nr2);
    return f2_pack(div_rn_slow(bf16_lo(wv), D), div_rn_slow(bf16_hi(wv), D));
}

// A pair's contribution to a target's squared error from its code values h2
// (binary16 pair): d' = fl(c*S*s - w) = -fl(w - c*S*s) in one rounding (c*S
// is exact), E <- fma(d', d', E), one packed lane for the even element and one
// for the odd.
__device__ __forceinline__ void f46_err(uint32_t h2, uint64_t nw, uint16_t S_h, uint64_t s_2, uint64_t &E2) {
    const uint64_t cs2 = f2_pack(mul_f16_exact(lo16(h2), S_h), mul_f16_exact(hi16(h2), S_h));
    const uint64_t d2 = f2_fma(cs2, s_2, nw);
    E2 = f2_fma(d2, d2, E2);
}

// Both targets side by side over the block's pairs: code words and errors.
// Each 8-element half is converted four pairs at a time (e2m1_quad).
template <bool FAST>
__device__ __forceinline__ void f46_both(const uint32_t *w, const F46Target &t6, const F46Target &t4, float s,
                                         uint32_t c6[2], uint32_t c4[2], float &e6, float &e4) {
    const uint64_t s_2 = f2_pack(s, s);
    const uint64_t D6 = f2_pack(t6.D, t6.D), n6 = f2_pack(t6.nr, t6.nr);
    const uint64_t D4 = f2_pack(t4.D, t4.D), n4 = f2_pack(t4.nr, t4.nr);
    uint64_t E6 = 0ull, E4 = 0ull;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        uint64_t nw[4], y[4];
        uint32_t h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            nw[j] = bf16x2_neg_f2(w[4 * k + j]);
            y[j] = f46_quot<FAST>(nw[j], w[4 * k + j], t6.D, D6, n6);
        }
        c6[k] = e2m1_quad(y, h);
#pragma unroll
        for (int j = 0; j < 4; ++j) f46_err(h[j], nw[j], t6.S_h, s_2, E6);
#pragma unroll
        for (int j = 0; j < 4; ++j) y[j] = f46_quot<FAST>(nw[j], w[4 * k + j], t4.D, D4, n4);
        c4[k] = e2m1_quad(y, h);
#pragma unroll
        for (int j = 0; j < 4; ++j) f46_err(h[j], nw[j], t4.S_h, s_2, E4);
    }
    e6 = __fadd_rn(f2_lo(E6), f2_hi(E6));
    e4 = __fadd_rn(f2_lo(E4), f2_hi(E4));
}

// Whether the target 4's squared error is strictly below the target 6's, decided
// exactly.  With alpha_i = c6_i*S6 and beta_i = c4_i*S4 (exact in binary32), the
// dequantized values are alpha_i*s and beta_i*s, and
//   e4 - e6 = sum_i (w_i - beta_i s)^2 - (w_i - alpha_i s)^2 = s (2P - sQ),
//   P = sum_i (alpha_i - beta_i) w_i,   Q = sum_i (alpha_i^2 - beta_i^2).
// S4 >= S6 and its exponent is E or E + 1, E the exponent of S6, so alpha_i and
// beta_i are integers below 2^9 times 2^(E-4): alpha - beta has at most 10
// significant bits, each term of P at most 18 (w is bf16), each term of Q at
// most 19 units of 2^(2E-8) and Q at most 23.  So every product here is exact
// in binary64, Q and s*Q (47 bits) are exact, and P is exact whenever the
// elements with a nonzero code span at most 2^31 in magnitude (always, unless
// the block scale is clamped far away from the block maximum): then 2P < sQ is
// the exact comparison.  Called for the rare near-tie blocks only, hence out of
// line.
__device__ __noinline__ bool f46_four_exact(uint4 wa, uint4 wb, uint32_t c6_0, uint32_t c6_1, uint32_t S6_h,
                                            uint32_t c4_0, uint32_t c4_1, uint32_t S4_h, float s) {
    const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    double P = 0.0, Q = 0.0;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t h6 = e2m1_pair_f16x2(((k ? c6_1 : c6_0) >> (8 * j)) & 0xffu);
            const uint32_t h4 = e2m1_pair_f16x2(((k ? c4_1 : c4_0) >> (8 * j)) & 0xffu);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const double al = mul_f16_exact(h ? hi16(h6) : lo16(h6), (uint16_t)S6_h);
                const double be = mul_f16_exact(h ? hi16(h4) : lo16(h4), (uint16_t)S4_h);
                const double wv = h ? bf16_hi(w[4 * k + j]) : bf16_lo(w[4 * k + j]);
                P = __dadd_rn(P, __dmul_rn(__dsub_rn(al, be), wv));
                Q = __dadd_rn(Q, __dsub_rn(__dmul_rn(al, al), __dmul_rn(be, be)));
            }
        }
    }
    return __dmul_rn(2.0, P) < __dmul_rn((double)s, Q);
}

// Whether a block with maximum A takes the fast arithmetic under scale sc:
// the scale is fast and A lies in [2^-60, 2^60] or is 0.
__device__ __forceinline__ bool f46_fast_range(float A, const F46Scale &sc) {
    return sc.fast && A <= 0x1p60f && (A >= 0x1p-60f || A == 0.0f);
}

// FourOverSix of one block with block maximum A (bf16 magnitude, exact) and
// scale sc.s > 0.  Returns true when the target 4 is chosen (its squared error
// strictly lower than the target 6's; a tie keeps 6); sb and codes receive the
// choice.
//
// The choice is screened with the binary32 sums e = fl(E_even + E_odd) of
// f46_both.  Each is within gamma_11 < 2^-20.5 relative of the exact error
// (one rounding in every d, two in every fused square-and-add of a lane, one in
// the final add), plus at most 2^-144 absolute where values are subnormal.  So
// when |e4 - e6| exceeds 2^-19 (e4 + e6) + 2^-140 the binary32 order is the
// exact order.  Otherwise -- a near tie, an exact tie between different
// candidates (they occur: about one block in 10^7 of Gaussian weights), or a
// non-finite sum -- the choice is taken by f46_four_exact, unless the two
// candidates are the same (equal scale bytes).
// (The warp vote on the range that rtn_block's callers take measured 2-3%
// slower here: the two-target code has more to lose in registers.)
__device__ __forceinline__ bool f46_block(const uint32_t *w, float A, const F46Scale &sc, uint32_t &sb,
                                          uint32_t codes[2]) {
    F46Target t6, t4;
    uint32_t c6[2], c4[2];
    float e6, e4;
    if (f46_fast_range(A, sc)) {
        f46_targets_fast(A, sc, t6, t4);
        f46_both<true>(w, t6, t4, sc.s, c6, c4, e6, e4);
    } else {
        t6 = f46_target(f46_x(A, sc.den6, sc.rden6, sc.den_ok), sc.s, A);
        t4 = f46_target(f46_x(A, sc.den4, sc.rden4, sc.den_ok), sc.s, A);
        if (t6.fast && t4.fast) f46_both<true>(w, t6, t4, sc.s, c6, c4, e6, e4);
        else f46_both<false>(w, t6, t4, sc.s, c6, c4, e6, e4);
    }
    bool four = e4 < e6;
    // Equal scale bytes make the two candidates identical (an exact tie: 6 is
    // kept, and e4 < e6 is false); this is the block of a tensor's or token's
    // maximum, where both scales clamp at 448.  Any other near tie is decided
    // exactly.
    if (t4.sb != t6.sb && !(fabsf(e4 - e6) > fmaf(0x1p-19f, e4 + e6, 0x1p-140f))) {
        const uint4 wa = make_uint4(w[0], w[1], w[2], w[3]), wb = make_uint4(w[4], w[5], w[6], w[7]);
        four = f46_four_exact(wa, wb, c6[0], c6[1], t6.S_h, c4[0], c4[1], t4.S_h, sc.s);
    }
    sb = four ? t4.sb : t6.sb;
    codes[0] = four ? c4[0] : c6[0];
    codes[1] = four ? c4[1] : c6[1];
    return four;
}

// NVFP4 round to nearest of one block (the target 6 alone: the card's block
// equations with m = 1 and sigmoid = 1) with block maximum A and scale sc.s > 0.
// FAST: the caller has found f46_fast_range true for this block, for every
// lane of its warp, so that the general code is not compiled into the path.
template <bool FAST = false>
__device__ __forceinline__ void rtn_block(const uint32_t *w, float A, const F46Scale &sc, uint32_t &sb,
                                          uint32_t codes[2]) {
    F46Target t6;
    if (FAST || f46_fast_range(A, sc)) {
        // as f46_target(f46_x(...)), without the range checks sc.fast makes redundant
        float x = (A == 0.0f) ? 1.0f : div_full(A, sc.den6, sc.rden6);
        t6.sb = e4m3_byte(fmaxf(x, 0x1p-6f));           // the conversion saturates at 448
        t6.S_h = (uint16_t)e4m3_normal_f16_bits(t6.sb);
        t6.D = __fmul_rn(e4m3_normal_f32(t6.sb), sc.s);
        t6.nr = -rcp_rn(t6.D);
        t6.fast = true;
    } else {
        t6 = f46_target(f46_x(A, sc.den6, sc.rden6, sc.den_ok), sc.s, A);
    }
    sb = t6.sb;
    const uint64_t D6 = f2_pack(t6.D, t6.D), n6 = f2_pack(t6.nr, t6.nr);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        uint64_t y[4];
        uint32_t h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t wv = w[4 * k + j];
            y[j] = (FAST || t6.fast) ? f46_quot<true>(bf16x2_neg_f2(wv), wv, t6.D, D6, n6)
                                     : f46_quot<false>(bf16x2_neg_f2(wv), wv, t6.D, D6, n6);
        }
        codes[k] = e2m1_quad(y, h);
    }
}

// Block maximum |w| of 16 bf16 values as bf16 magnitude bits (exact; NaN and
// infinity sort above every finite magnitude).
__device__ __forceinline__ uint32_t block_amax_bits(const uint32_t *w) {
    uint32_t am = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) am = __vmaxu2(am, w[j] & 0x7fff7fffu);
    return max(am & 0xffffu, am >> 16);
}

// The bf16 bits of w' = bf16(fl(fl(c*S)*s)) for the 16 codes of a block, as
// four 16-byte words.
__device__ __forceinline__ void wq_words(const uint32_t codes[2], uint32_t sbyte, float s, uint4 out[2]) {
    const uint16_t S_h = (uint16_t)e4m3_normal_f16_bits(sbyte);
    const uint64_t s_2 = f2_pack(s, s);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t h2 = e2m1_pair_f16x2((codes[k] >> (8 * j)) & 0xffu);
            const uint64_t p = f2_mul(f2_pack(mul_f16_exact(lo16(h2), S_h), mul_f16_exact(hi16(h2), S_h)), s_2);
            o[j] = pack_bf16x2(f2_lo(p), f2_hi(p));
        }
        out[k] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// FourOverSix (or, rtn, plain NVFP4 round to nearest) of one block of a weight
// tensor (tensor scale s2 = T.s2).
// Every lane of the warp calls it (past a ragged end with B.valid false): for
// plain round to nearest, when every valid block of the warp is in the fast
// range, the warp runs the fast code alone.
template <class TV>
__device__ __forceinline__ void compute_block_f46(const TV &T, Block &B, bool rtn) {
    const uint32_t abits = block_amax_bits(B.w);
    const float A = __uint_as_float(abits << 16);
    const bool bad = B.valid && abits >= 0x7f80u;
    F46Scale sc;
    sc.s = T.s2; sc.den6 = T.den; sc.rden6 = T.rden; sc.den4 = T.den4; sc.rden4 = T.rden4;
    sc.den_ok = T.den46_ok;
    sc.fast = f46_scale_fast(sc.den_ok, sc.s);
    const bool fast = rtn && __all_sync(FULL, !B.valid || f46_fast_range(A, sc));
    if (B.valid) {
        uint32_t sb, codes[2];
        if (!rtn) f46_block(B.w, A, sc, sb, codes);
        else if (fast) rtn_block<true>(B.w, A, sc, sb, codes);
        else rtn_block(B.w, A, sc, sb, codes);
        if (T.d.codes) {
            reinterpret_cast<uint2 *>(T.d.codes)[B.blk] = make_uint2(codes[0], codes[1]);
            T.d.scales[B.blk] = (uint8_t)sb;
        }
        if (T.d.Wq) {
            uint4 o[2];
            wq_words(codes, sb, T.s2, o);
            __stcs(reinterpret_cast<uint4 *>(T.d.Wq) + 2u * B.blk, o[0]);
            __stcs(reinterpret_cast<uint4 *>(T.d.Wq) + 2u * B.blk + 1u, o[1]);
        }
    }
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_error_flags, 1u);
}

// The forward's per-block scalars: the scaled maximum, the scale byte and
// value, and the sub-blocks' sigmoids (binary32, and the binary64 values the
// export starts from).  The divisors D = fl(fl(S*sigma)*s2) are recomputed
// where used rather than held.
struct BlockScalars {
    float x, S;
    uint32_t sbyte;
    float sig[2];
    double s64[2];
};

// The forward's scalars on the fast path, with no branch: returns whether
// each is the one the general code computes and lies where the fast
// arithmetic that follows is exact -- the scaled maximum by the reciprocal,
// the sigmoids decided, A <= 2^60 and both D in [2^-60, 2^60].  When it
// returns false the values are unspecified (never a fault) and the caller
// takes the general code.
template <class TV>
__device__ __forceinline__ bool block_scalars_fast(const TV &T, float A, float m, float q0, float q1,
                                                   BlockScalars &f) {
    const float Am = __fmul_rn(A, m);
    const float aAm = fabsf(Am);
    bool ok = T.den_ok && aAm <= 0x1p60f && (aAm >= 0x1p-60f || aAm == 0.0f) && A <= 0x1p60f;
    f.x = div_full(Am, T.den, T.rden);
    float xc = (f.x == 0.0f) ? 1.0f : f.x;
    xc = fminf(fmaxf(xc, 0x1p-6f), 448.0f);
    f.sbyte = e4m3_byte(xc);
    f.S = e4m3_normal_f32(f.sbyte);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        ok = sigmoid_fast_try(k ? q1 : q0, f.sig[k], f.s64[k]) && ok;
        const float D = __fmul_rn(__fmul_rn(f.S, f.sig[k]), T.s2);
        ok = ok && D >= 0x1p-60f && D <= 0x1p60f;
    }
    return ok;
}

// Everything of compute_block after the block maximum.  FAST: the forward's
// scalars f come from block_scalars_fast, which held for every lane of the
// warp, so the forward's per-element work runs with no range test and no
// branch.  Otherwise (a lane outside the fast range: rare) the general code,
// which tests each quantity where it is used.  Both give the same bits.
template <int KIND, bool WQU, int SF, bool FAST, bool SO, class TV>
__device__ __forceinline__ void block_body(const TV &T, const Args &a, Block &B, float A, bool bad,
                                           const BlockScalars &f, unsigned char *so, uint32_t lb) {
    using O = StepOpt<SF>;
    using L = Layout<KIND>;
    // S_b = e4m3(clamp(fl(fl(A*m)/fl(6*s2)), 2^-6, 448)), scale 1 when the scaled max is 0
    float x, S;
    uint32_t sbyte;
    if constexpr (FAST) {
        x = f.x; S = f.S; sbyte = f.sbyte;
    } else {
        x = scaled_max(T, A, B.m);
        float xc = (x == 0.0f) ? 1.0f : x;
        xc = fminf(fmaxf(xc, 0x1p-6f), 448.0f);
        sbyte = e4m3_byte(xc);
        S = e4m3_normal_f32(sbyte);
    }
    const bool inS = (x != 0.0f) && (x >= 0x1p-6f) && (x <= 448.0f);
    const uint16_t S_h = (uint16_t)e4m3_normal_f16_bits(sbyte);
    const uint64_t s2_2 = f2_pack(T.s2, T.s2);

    // (the step always writes W' where the descriptor has it)
    const bool want_wq = KIND != KIND_BWD && !WQU && (KIND == KIND_STEP || a.write_wq) && T.d.Wq != nullptr && B.valid;
    float sig[2], sq[2];
    double s64[2];                              // the forward's binary64 sigmoids, reused by the export
    uint64_t sm2 = 0ull;                        // sum of g * (in ? c - y : c), pairwise
    uint32_t codes[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        // D_k = fl(fl(S*sigmoid(q_k))*s2); y_i = fl(w_i/D_k); c_i = E2M1(clamp(y_i, -6, 6))
        if constexpr (FAST) {
            sig[k] = f.sig[k]; s64[k] = f.s64[k];
        } else {
            sig[k] = sigmoid_fast(B.q[k], s64[k]);
        }
        const float D = __fmul_rn(__fmul_rn(S, sig[k]), T.s2);
        uint64_t y2[4];
        if (FAST || (D >= 0x1p-60f && D <= 0x1p60f && A <= 0x1p60f)) {
            const float nr = -rcp_rn(D);
            const uint64_t D2 = f2_pack(D, D), nr2 = f2_pack(nr, nr);
#pragma unroll
            for (int j = 0; j < 4; ++j) y2[j] = div_by_f2(bf16x2_neg_f2(B.w[4 * k + j]), D2, nr2);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                y2[j] = f2_pack(div_rn_slow(bf16_lo(B.w[4 * k + j]), D), div_rn_slow(bf16_hi(B.w[4 * k + j]), D));
        }
        uint32_t code = 0u;
        uint32_t ch2[4];
        uint64_t cs2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t byte = e2m1_pair(f2_lo(y2[j]), f2_hi(y2[j]));
            code |= byte << (8 * j);
            ch2[j] = e2m1_pair_f16x2(byte);
            cs2[j] = f2_pack(mul_f16_exact(lo16(ch2[j]), S_h), mul_f16_exact(hi16(ch2[j]), S_h));   // c*S, exact
        }
        codes[k] = code;
        // w' = bf16(fl(fl(c*S)*s2))
        if (want_wq) {
            uint4 o;
            uint64_t p;
            p = f2_mul(cs2[0], s2_2); o.x = pack_bf16x2(f2_lo(p), f2_hi(p));
            p = f2_mul(cs2[1], s2_2); o.y = pack_bf16x2(f2_lo(p), f2_hi(p));
            p = f2_mul(cs2[2], s2_2); o.z = pack_bf16x2(f2_lo(p), f2_hi(p));
            p = f2_mul(cs2[3], s2_2); o.w = pack_bf16x2(f2_lo(p), f2_hi(p));
            if constexpr (SO) reinterpret_cast<uint4 *>(so + L::W)[2u * lb + (uint32_t)k] = o;
            else __stcs(reinterpret_cast<uint4 *>(T.d.Wq) + (2u * B.blk + (uint32_t)k), o);
        }
        sq[k] = 0.0f;
        if (has_grad(KIND)) {
            // straight-through sums, element by element: g*t with t = c - y inside the
            // clamp and c outside (c - y is exact near the code, so the sum is well
            // conditioned), and g*y inside the clamp, per sub-block
            uint64_t sq2 = 0ull;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint64_t g2 = bf16x2_f2(B.g[4 * k + j]);
                const float ylo = f2_lo(y2[j]), yhi = f2_hi(y2[j]);
                const float ilo = fabsf(ylo) <= 6.0f ? ylo : 0.0f, ihi = fabsf(yhi) <= 6.0f ? yhi : 0.0f;
                const uint64_t t2 = f2_pack(sub_f16_f32(lo16(ch2[j]), ilo), sub_f16_f32(hi16(ch2[j]), ihi));
                sm2 = f2_fma(g2, t2, sm2);
                sq2 = f2_fma(g2, f2_pack(ilo, ihi), sq2);
            }
            sq[k] = __fadd_rn(f2_lo(sq2), f2_hi(sq2));
        }
    }
    // the forward's NVFP4 codes and scale (unless the step exports the updated parameters instead)
    if (B.valid && !(KIND == KIND_STEP && O::pack(a))) {
        if constexpr (SO) {
            reinterpret_cast<uint2 *>(so + L::CODES)[lb] = make_uint2(codes[0], codes[1]);
            so[L::SCALES + lb] = (uint8_t)sbyte;
        } else {
            if (T.d.codes) {
                uint2 cc; cc.x = codes[0]; cc.y = codes[1];
                reinterpret_cast<uint2 *>(T.d.codes)[B.blk] = cc;
            }
            if (T.d.scales) T.d.scales[B.blk] = (uint8_t)sbyte;
        }
    }

    if (has_grad(KIND)) {
        // dL/dm = inS*(A/6)*sum g*t;  dL/dq_k = -(1 - sigma_k)*S*s2*sum_k g*y_in
        // (every operation rounded on its own, never contracted into a fused
        // multiply-add, so that every build of the step gives the same bits)
        float gm = inS ? __fmul_rn(__fmul_rn(A, 1.0f / 6.0f), __fadd_rn(f2_lo(sm2), f2_hi(sm2))) : 0.0f;
        float gq0 = -__fmul_rn(__fmul_rn(__fmul_rn(__fsub_rn(1.0f, sig[0]), S), T.s2), sq[0]);
        float gq1 = -__fmul_rn(__fmul_rn(__fmul_rn(__fsub_rn(1.0f, sig[1]), S), T.s2), sq[1]);
        if (O::acc(a)) {
            gm = __fadd_rn(B.gm_in, gm);
            gq0 = __fadd_rn(B.gq_in[0], gq0);
            gq1 = __fadd_rn(B.gq_in[1], gq1);
        }
        if (B.valid && !bad && !(finitef(gm) && finitef(gq0) && finitef(gq1))) atomicOr(&g_error_flags, 4u);
        if (B.valid && (KIND == KIND_BWD || O::write_grad(a))) {
            T.d.dm[B.blk] = gm;
            reinterpret_cast<float2 *>(T.d.dq)[B.blk] = make_float2(gq0, gq1);
        }
        if (KIND == KIND_STEP) {
            adamw_one(B.m, gm, B.mv1, B.mv2, a.hp.lr_m_step, a.hp.decay_m, a.hp);
            const float q_old0 = B.q[0], q_old1 = B.q[1];
            uint64_t qp = f2_pack(B.q[0], B.q[1]);
            uint64_t v1 = f2_pack(B.qv1[0], B.qv1[1]), v2 = f2_pack(B.qv2[0], B.qv2[1]);
            adamw_pair(qp, f2_pack(gq0, gq1), v1, v2, a.hp.lr_q_step, a.hp.decay_q, a.hp);
            if constexpr (SO) {                          // over the block's input slots
                reinterpret_cast<float *>(so + L::M)[lb] = B.m;
                reinterpret_cast<float *>(so + L::MV1)[lb] = B.mv1;
                reinterpret_cast<float *>(so + L::MV2)[lb] = B.mv2;
                reinterpret_cast<uint64_t *>(so + L::Q)[lb] = qp;
                reinterpret_cast<uint64_t *>(so + L::QV1)[lb] = v1;
                reinterpret_cast<uint64_t *>(so + L::QV2)[lb] = v2;
            } else if (B.valid) {
                T.d.m[B.blk] = B.m;
                T.d.m_exp_avg[B.blk] = B.mv1;
                T.d.m_exp_avg_sq[B.blk] = B.mv2;
                reinterpret_cast<float2 *>(T.d.q)[B.blk] = make_float2(f2_lo(qp), f2_hi(qp));
                reinterpret_cast<float2 *>(T.d.q_exp_avg)[B.blk] = make_float2(f2_lo(v1), f2_hi(v1));
                reinterpret_cast<float2 *>(T.d.q_exp_avg_sq)[B.blk] = make_float2(f2_lo(v2), f2_hi(v2));
            }
            // the forward of the updated m and q: NVFP4 export (what a pack after this
            // step would write) and/or W' for the next step's forward
            const bool exp_codes = O::pack(a) && T.d.codes != nullptr;
            const bool exp_wq = WQU && T.d.Wq != nullptr;
            if (B.valid && (exp_codes || exp_wq)) {
                uint32_t sb2, codes2[2];
                encode_block(T, B.w, A, B.m, f2_lo(qp), f2_hi(qp), s64[0], s64[1], q_old0, q_old1, sb2, codes2);
                if (exp_codes) {
                    if constexpr (SO) {
                        reinterpret_cast<uint2 *>(so + L::CODES)[lb] = make_uint2(codes2[0], codes2[1]);
                        so[L::SCALES + lb] = (uint8_t)sb2;
                    } else {
                        uint2 cc; cc.x = codes2[0]; cc.y = codes2[1];
                        reinterpret_cast<uint2 *>(T.d.codes)[B.blk] = cc;
                        T.d.scales[B.blk] = (uint8_t)sb2;
                    }
                }
                if (exp_wq) store_wq_from_codes<SO>(T, B.blk, codes2, sb2, so, lb);
            }
        }
    }
}

// The forward, the straight-through gradients and the AdamW update of one block.
// WQU (step only, FOCUS_STEP_WQ_UPDATED): W' is that of the updated m and q,
// a compile-time choice so that the other step variants keep its registers.
// TV is any view of a tensor with members d (descriptor), s2, den and nblk:
// the consumer warps pass the stage record in shared memory, so the
// descriptor's pointers are read where used instead of held in registers.
// Every lane of the warp calls it (past a ragged end with B.valid false).
// SO (the step's full tiles): the outputs go to the block's slots of the stage
// at so (local block lb), which the producer writes out with bulk copies;
// otherwise straight to global memory.
template <int KIND, bool WQU, int SF, bool SO = false, class TV>
__device__ __forceinline__ void compute_block(const TV &T, const Args &a, Block &B, unsigned char *so = nullptr,
                                              uint32_t lb = 0) {
    using O = StepOpt<SF>;
    if constexpr (KIND == KIND_F46 || KIND == KIND_RTN) {
        compute_block_f46(T, B, KIND == KIND_RTN);
        return;
    }
    // A_b = max |w| over the block: max of the bf16 magnitude bit patterns (a NaN
    // or an infinity sorts above every finite magnitude, which is how it is found)
    uint32_t am = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) am = __vmaxu2(am, B.w[j] & 0x7fff7fffu);
    const uint32_t abits = max(am & 0xffffu, am >> 16);
    const float A = __uint_as_float(abits << 16);
    const bool bad = B.valid && (abits >= 0x7f80u || !finitef(B.m) || !finitef(B.q[0]) || !finitef(B.q[1]));
    // The tensor maximum for the next step's s2 (focus_step_fused_amax): the warp's
    // maximum of the block maxima (the blocks past a ragged end have w = 0) into the
    // stage record in shared memory; the producer folds the stage maxima of a tensor
    // and writes them out (T is the stage record here).
    if (KIND == KIND_STEP && O::amax(a)) {
        const uint32_t wm = __reduce_max_sync(FULL, abits);
        if ((threadIdx.x & 31) == 0 && wm != 0u) atomicMax(const_cast<uint32_t *>(&T.amax), wm);
    }
    // the forward's scalars on the fast path; a warp with a lane outside it takes
    // the general code (the lanes of a warp hold neighbouring blocks of one tile)
    BlockScalars f;
    const bool fast = block_scalars_fast(T, A, B.m, B.q[0], B.q[1], f);
    if (__all_sync(FULL, fast)) block_body<KIND, WQU, SF, true, SO>(T, a, B, A, bad, f, so, lb);
    else block_body<KIND, WQU, SF, false, SO>(T, a, B, A, bad, f, so, lb);
    if (__any_sync(FULL, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_error_flags, 1u);
}

// ---------------------------------------------------------------------------
// shared-memory stage layout and pipeline depth per kind
// ---------------------------------------------------------------------------

template <int KIND>
struct Layout {
    static constexpr bool G_ = has_grad(KIND);           // dW' and the gradient accumulators
    static constexpr bool MQ = has_mq(KIND);             // m and q
    static constexpr bool ST = KIND == KIND_STEP;        // AdamW moments
    static constexpr uint32_t W = 0;
    static constexpr uint32_t G = W + TILE_BLOCKS * 32;
    static constexpr uint32_t M = G + (G_ ? TILE_BLOCKS * 32 : 0);
    static constexpr uint32_t Q = M + (MQ ? TILE_BLOCKS * 4 : 0);
    static constexpr uint32_t MV1 = Q + (MQ ? TILE_BLOCKS * 8 : 0);
    static constexpr uint32_t MV2 = MV1 + (ST ? TILE_BLOCKS * 4 : 0);
    static constexpr uint32_t QV1 = MV2 + (ST ? TILE_BLOCKS * 4 : 0);
    static constexpr uint32_t QV2 = QV1 + (ST ? TILE_BLOCKS * 8 : 0);
    static constexpr uint32_t GM = QV2 + (ST ? TILE_BLOCKS * 8 : 0);
    static constexpr uint32_t GQ = GM + (G_ ? TILE_BLOCKS * 4 : 0);
    static constexpr uint32_t IN_END = GQ + (G_ ? TILE_BLOCKS * 8 : 0);  // end of the inputs
    // the step's outputs that have no input slot to take over: codes and scales
    static constexpr uint32_t CODES = IN_END;
    static constexpr uint32_t SCALES = CODES + (ST ? TILE_BLOCKS * 8 : 0);
    static constexpr uint32_t BYTES = SCALES + (ST ? TILE_BLOCKS : 0);     // one stage
    // bytes the bulk copies of one full tile deliver
    static __device__ __forceinline__ uint32_t tx_bytes(bool accumulate) {
        return (accumulate || !G_) ? IN_END : GM;
    }
};

template <int KIND> struct Depth;
template <> struct Depth<KIND_FWD> { static constexpr int STAGES = 6, MIN_CTAS = 3; };
template <> struct Depth<KIND_BWD> { static constexpr int STAGES = 3, MIN_CTAS = 3; };
template <> struct Depth<KIND_STEP> { static constexpr int STAGES = 2, MIN_CTAS = 3; };
template <> struct Depth<KIND_F46> { static constexpr int STAGES = 8, MIN_CTAS = 3; };
template <> struct Depth<KIND_RTN> { static constexpr int STAGES = 8, MIN_CTAS = 3; };

template <int KIND>
constexpr uint32_t stage_smem_bytes() { return Depth<KIND>::STAGES * Layout<KIND>::BYTES; }

enum : uint32_t { MODE_BULK = 0, MODE_DIRECT = 1, MODE_SKIP = 2 };

// The producer's record of one staged tile, read by the consumers from shared
// memory: the tile's tensor (descriptor, s2, fl(6*s2), block count) and place.
struct StageInfo {
    focus_tensor_desc d;
    int64_t nblk;
    float s2;
    float den;
    float rden;
    uint32_t den_ok;
    uint32_t first;    // first block of the tile within the tensor
    uint32_t nb;       // blocks in the tile
    uint32_t mode;     // MODE_*
    float den4;        // FourOverSix: fl(4*s2), its reciprocal, both quotients exact by reciprocal
    float rden4;
    uint32_t den46_ok;
    uint32_t tensor;   // index of the tile's tensor in the table
    uint32_t amax;     // fused step with s2 for the next step: max |w| bits of the tile (consumers' smem atomics)
};

// The running tensor maximum the producer keeps for focus_step_fused_amax: the
// stage maxima of consecutive tiles of one tensor are folded in a register and
// written with one global atomic when the tensor changes (about one atomic per
// CTA and tensor, instead of one per warp and tile, which contended at L2).
struct AmaxFold {
    uint32_t tensor = 0xffffffffu;
    uint32_t v = 0u;
    __device__ __forceinline__ void add(uint32_t *ws, uint32_t t, uint32_t x) {
        if (t != tensor) {
            flush(ws);
            tensor = t;
            v = 0u;
        }
        v = max(v, x);
    }
    __device__ __forceinline__ void flush(uint32_t *ws) {
        if (tensor != 0xffffffffu && v != 0u) atomicMax(ws + tensor, v);
    }
};

// A block's inputs from a staged tile (local block lb of the tile).
template <int KIND, int SF>
__device__ __forceinline__ void load_block_smem(const Args &a, const unsigned char *stage, Block &B, uint32_t lb,
                                                uint32_t blk) {
    using L = Layout<KIND>;
    B.blk = blk;
    B.valid = true;
    const uint4 *W = reinterpret_cast<const uint4 *>(stage + L::W) + 2u * lb;
    const uint4 w0 = W[0], w1 = W[1];
    B.w[0] = w0.x; B.w[1] = w0.y; B.w[2] = w0.z; B.w[3] = w0.w;
    B.w[4] = w1.x; B.w[5] = w1.y; B.w[6] = w1.z; B.w[7] = w1.w;
    if (has_grad(KIND)) {
        const uint4 *G = reinterpret_cast<const uint4 *>(stage + L::G) + 2u * lb;
        const uint4 g0 = G[0], g1 = G[1];
        B.g[0] = g0.x; B.g[1] = g0.y; B.g[2] = g0.z; B.g[3] = g0.w;
        B.g[4] = g1.x; B.g[5] = g1.y; B.g[6] = g1.z; B.g[7] = g1.w;
    }
    if (has_mq(KIND)) {
        B.m = reinterpret_cast<const float *>(stage + L::M)[lb];
        const float2 q = reinterpret_cast<const float2 *>(stage + L::Q)[lb];
        B.q[0] = q.x; B.q[1] = q.y;
    }
    if (KIND == KIND_STEP) {
        B.mv1 = reinterpret_cast<const float *>(stage + L::MV1)[lb];
        B.mv2 = reinterpret_cast<const float *>(stage + L::MV2)[lb];
        const float2 v1 = reinterpret_cast<const float2 *>(stage + L::QV1)[lb];
        const float2 v2 = reinterpret_cast<const float2 *>(stage + L::QV2)[lb];
        B.qv1[0] = v1.x; B.qv1[1] = v1.y; B.qv2[0] = v2.x; B.qv2[1] = v2.y;
    }
    if (has_grad(KIND) && StepOpt<SF>::acc(a)) {
        B.gm_in = reinterpret_cast<const float *>(stage + L::GM)[lb];
        const float2 gq = reinterpret_cast<const float2 *>(stage + L::GQ)[lb];
        B.gq_in[0] = gq.x; B.gq_in[1] = gq.y;
    } else {
        B.gm_in = 0.0f; B.gq_in[0] = B.gq_in[1] = 0.0f;
    }
}

// Next tensor holding `tile`, scanning forward from T (tiles only increase).
// Returns false when the table has no tensor for it.
__device__ __forceinline__ bool seek_tensor(const Args &a, int64_t tile, int &t, TensorRef &T, bool &have) {
    if (have && tile < T.tile_end) return true;
    const int n = a.table ? a.n_tensors : 1;
    if (have && t + 1 < n) ++t;
    for (;;) {
        load_tensor(a, t, T);
        if (tile < T.tile_end || t + 1 >= n) break;
        ++t;
    }
    have = true;
    return tile < T.tile_end;
}

// The outputs a full tile of the step left in its stage, written to global
// memory with bulk copies (one group): W' over W, the parameters and moments
// over theirs, the codes and scales from their own regions.  Each array the
// descriptor has is written whole: the step writes every block of a full tile.
__device__ __forceinline__ void store_step_tile(const StageInfo &inf, const unsigned char *stage) {
    using L = Layout<KIND_STEP>;
    const focus_tensor_desc &d = inf.d;
    const uint32_t f = inf.first;
    if (d.Wq) bulk_s2g(reinterpret_cast<uint4 *>(d.Wq) + 2u * f, smem_u32(stage + L::W), TILE_BLOCKS * 32);
    if (d.codes) {
        bulk_s2g(d.codes + 8u * f, smem_u32(stage + L::CODES), TILE_BLOCKS * 8);
        bulk_s2g(d.scales + f, smem_u32(stage + L::SCALES), TILE_BLOCKS);
    }
    bulk_s2g(d.m + f, smem_u32(stage + L::M), TILE_BLOCKS * 4);
    bulk_s2g(d.m_exp_avg + f, smem_u32(stage + L::MV1), TILE_BLOCKS * 4);
    bulk_s2g(d.m_exp_avg_sq + f, smem_u32(stage + L::MV2), TILE_BLOCKS * 4);
    bulk_s2g(d.q + 2u * f, smem_u32(stage + L::Q), TILE_BLOCKS * 8);
    bulk_s2g(d.q_exp_avg + 2u * f, smem_u32(stage + L::QV1), TILE_BLOCKS * 8);
    bulk_s2g(d.q_exp_avg_sq + 2u * f, smem_u32(stage + L::QV2), TILE_BLOCKS * 8);
    bulk_commit();
}

// The producer: one thread feeding the ring (and, for the step, writing the
// outputs of each full tile from its stage before the stage takes the next).
template <int KIND, int SF>
__device__ __forceinline__ void produce(const Args &a, unsigned char *smem, uint64_t *full, uint64_t *empty,
                                        StageInfo *info) {
    using L = Layout<KIND>;
    using O = StepOpt<SF>;
    constexpr int S = Depth<KIND>::STAGES;
    int t = 0;
    TensorRef T;
    bool have = false;
    uint32_t pending = 0;             // stages whose last use was filled by bulk copies
    uint32_t pending_parity = 0;      // and the parity of that use
    uint32_t it = 0;
    bool timed_out = false;
    AmaxFold fold;
    for (int64_t tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++it) {
        const uint32_t st = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!mbar_wait(smem_u32(&empty[st]), ph ^ 1u)) {
            atomicOr(&g_error_flags, 8u);
            timed_out = true;
            break;
        }
        pending &= ~(1u << st);       // the consumers released it: its copies have landed
        StageInfo &inf = info[st];
        if (KIND == KIND_STEP && O::amax(a)) {
            if (it >= (uint32_t)S) fold.add(a.amax_ws, inf.tensor, inf.amax);   // the stage's previous tile
            inf.amax = 0u;
        }
        // the previous tile's outputs leave the stage before those regions are
        // filled again (the regions no output uses are refilled at once)
        bool read_wait = false;
        if (KIND == KIND_STEP && it >= (uint32_t)S && inf.mode == MODE_BULK) {
            store_step_tile(inf, smem + st * L::BYTES);
            read_wait = true;
        }
        const bool found = seek_tensor(a, tile, t, T, have);
        const uint32_t first = found ? (uint32_t)(tile - T.d.tile_begin) * TILE_BLOCKS : 0u;
        const int64_t left = T.nblk - (int64_t)first;
        const uint32_t nb = found ? (uint32_t)(left < TILE_BLOCKS ? left : TILE_BLOCKS) : 0u;
        // a descriptor without a pointer this kernel needs (a table prepared for
        // another purpose) is skipped and reported, never dereferenced
        bool complete = T.d.W != nullptr && (!has_mq(KIND) || (T.d.m != nullptr && T.d.q != nullptr));
        if (has_grad(KIND)) complete = complete && T.d.dWq != nullptr;
        if (KIND == KIND_BWD || O::acc(a) || O::write_grad(a)) complete = complete && T.d.dm != nullptr && T.d.dq != nullptr;
        if (KIND == KIND_STEP)
            complete = complete && T.d.m_exp_avg && T.d.m_exp_avg_sq && T.d.q_exp_avg && T.d.q_exp_avg_sq;
        if (KIND != KIND_BWD && T.d.codes != nullptr) complete = complete && T.d.scales != nullptr;
        const bool usable = found && T.ok && (complete || T.nblk == 0);
        const uint32_t mode = !usable ? MODE_SKIP : (nb == (uint32_t)TILE_BLOCKS ? MODE_BULK : MODE_DIRECT);
        if (found && !(T.ok && complete)) atomicOr(&g_error_flags, 2u);
        inf.d = T.d;
        inf.nblk = T.nblk;
        inf.s2 = T.s2;
        inf.den = T.den;
        inf.rden = T.rden;
        inf.den_ok = T.den_ok ? 1u : 0u;
        inf.den4 = T.den4;
        inf.rden4 = T.rden4;
        inf.den46_ok = T.den46_ok ? 1u : 0u;
        inf.tensor = (uint32_t)t;
        inf.first = first;
        inf.nb = nb;
        inf.mode = mode;
        const uint32_t bar = smem_u32(&full[st]);
        if (mode == MODE_BULK) {
            unsigned char *stage = smem + st * L::BYTES;
            const uint32_t f = first;
            mbar_arrive_expect_tx(bar, L::tx_bytes(O::acc(a)));
            if (has_grad(KIND))
                bulk_g2s(smem_u32(stage + L::G), reinterpret_cast<const uint4 *>(T.d.dWq) + 2u * f, TILE_BLOCKS * 32,
                         bar);
            if (has_grad(KIND) && O::acc(a)) {
                bulk_g2s(smem_u32(stage + L::GM), T.d.dm + f, TILE_BLOCKS * 4, bar);
                bulk_g2s(smem_u32(stage + L::GQ), T.d.dq + 2u * f, TILE_BLOCKS * 8, bar);
            }
            if (read_wait) bulk_wait_read();
            bulk_g2s(smem_u32(stage + L::W), reinterpret_cast<const uint4 *>(T.d.W) + 2u * f, TILE_BLOCKS * 32, bar);
            if (has_mq(KIND)) {
                bulk_g2s(smem_u32(stage + L::M), T.d.m + f, TILE_BLOCKS * 4, bar);
                bulk_g2s(smem_u32(stage + L::Q), T.d.q + 2u * f, TILE_BLOCKS * 8, bar);
            }
            if (KIND == KIND_STEP) {
                bulk_g2s(smem_u32(stage + L::MV1), T.d.m_exp_avg + f, TILE_BLOCKS * 4, bar);
                bulk_g2s(smem_u32(stage + L::MV2), T.d.m_exp_avg_sq + f, TILE_BLOCKS * 4, bar);
                bulk_g2s(smem_u32(stage + L::QV1), T.d.q_exp_avg + 2u * f, TILE_BLOCKS * 8, bar);
                bulk_g2s(smem_u32(stage + L::QV2), T.d.q_exp_avg_sq + 2u * f, TILE_BLOCKS * 8, bar);
            }
            pending |= 1u << st;
            pending_parity = (pending_parity & ~(1u << st)) | (ph << st);
        } else {
            // (a ragged tile's consumers write their outputs into the stage)
            if (read_wait) bulk_wait_read();
            mbar_arrive(bar);
        }
    }
    // The last uses of the stages: wait (bounded) until the consumers have
    // released them, fold in their tensor maxima and write the running maximum,
    // and write the outputs of the full tiles; then wait until every bulk store
    // has completed.
    if (KIND == KIND_STEP && !timed_out) {
        for (uint32_t j = it > (uint32_t)S ? it - (uint32_t)S : 0u; j < it; ++j) {
            const uint32_t st = j % S;
            if (!mbar_wait(smem_u32(&empty[st]), (j / S) & 1u)) {
                atomicOr(&g_error_flags, 8u);
                break;
            }
            if (O::amax(a)) fold.add(a.amax_ws, info[st].tensor, info[st].amax);
            if (info[st].mode == MODE_BULK) store_step_tile(info[st], smem + st * L::BYTES);
        }
        if (O::amax(a)) fold.flush(a.amax_ws);
    }
    if (KIND == KIND_STEP) bulk_wait_all();
    // Before the CTA may exit, every bulk copy it issued must have landed (normally
    // the consumers already waited for all of them; this matters after a timeout).
    for (int st = 0; st < S; ++st)
        if ((pending >> st) & 1u)
            if (!mbar_wait(smem_u32(&full[st]), (pending_parity >> st) & 1u)) atomicOr(&g_error_flags, 8u);
}

// A ragged tile's block of the step: its outputs, left in the block's slots
// of the stage, to global memory (what store_step_tile does for a full tile;
// nothing for the blocks past the tensor's end).
template <bool WQU, int SF>
__device__ __forceinline__ void copy_out_step_block(const StageInfo &T, const Args &a, const Block &B,
                                                    const unsigned char *so, uint32_t lb) {
    using L = Layout<KIND_STEP>;
    if (!B.valid) return;
    const uint32_t blk = B.blk;
    if (T.d.Wq) {
        __stcs(reinterpret_cast<uint4 *>(T.d.Wq) + 2u * blk, reinterpret_cast<const uint4 *>(so + L::W)[2u * lb]);
        __stcs(reinterpret_cast<uint4 *>(T.d.Wq) + 2u * blk + 1u, reinterpret_cast<const uint4 *>(so + L::W)[2u * lb + 1u]);
    }
    if (T.d.codes) {
        reinterpret_cast<uint2 *>(T.d.codes)[blk] = reinterpret_cast<const uint2 *>(so + L::CODES)[lb];
        T.d.scales[blk] = so[L::SCALES + lb];
    }
    T.d.m[blk] = reinterpret_cast<const float *>(so + L::M)[lb];
    T.d.m_exp_avg[blk] = reinterpret_cast<const float *>(so + L::MV1)[lb];
    T.d.m_exp_avg_sq[blk] = reinterpret_cast<const float *>(so + L::MV2)[lb];
    reinterpret_cast<uint64_t *>(T.d.q)[blk] = reinterpret_cast<const uint64_t *>(so + L::Q)[lb];
    reinterpret_cast<uint64_t *>(T.d.q_exp_avg)[blk] = reinterpret_cast<const uint64_t *>(so + L::QV1)[lb];
    reinterpret_cast<uint64_t *>(T.d.q_exp_avg_sq)[blk] = reinterpret_cast<const uint64_t *>(so + L::QV2)[lb];
}

// The consumers: NC_WARPS warps computing from the ring.
template <int KIND, bool WQU, int SF>
__device__ __forceinline__ void consume(const Args &a, unsigned char *smem, uint64_t *full, uint64_t *empty,
                                        const StageInfo *info) {
    using L = Layout<KIND>;
    constexpr int S = Depth<KIND>::STAGES;
    const int lane = threadIdx.x & 31;
    uint32_t it = 0;
    for (int64_t tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++it) {
        const uint32_t st = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!mbar_wait(smem_u32(&full[st]), ph)) {
            if (lane == 0) atomicOr(&g_error_flags, 8u);
            break;
        }
        const StageInfo &inf = info[st];
        const uint32_t mode = inf.mode;
        if (mode != MODE_SKIP) {
            unsigned char *stage = smem + st * L::BYTES;
            const uint32_t lb = threadIdx.x;
            Block B;
            if (mode == MODE_BULK) load_block_smem<KIND, SF>(a, stage, B, lb, inf.first + lb);
            else load_block_global<KIND, SF>(inf, a, B, inf.first + lb);
            if constexpr (KIND == KIND_STEP) {
                // the step leaves its outputs in the stage: the producer writes a
                // full tile out with bulk copies, each thread a ragged tile's block
                // (the stage is free: a ragged tile was read from global memory)
                compute_block<KIND, WQU, SF, true>(inf, a, B, stage, lb);
                if (mode == MODE_BULK) fence_proxy_async_smem();
                else copy_out_step_block<WQU, SF>(inf, a, B, stage, lb);
            } else {
                compute_block<KIND, WQU, SF>(inf, a, B);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[st]));
    }
}

template <int KIND, bool WQU = false, int SF = SF_RUNTIME>
__global__ void __launch_bounds__(CTA_THREADS, Depth<KIND>::MIN_CTAS) pipe_kernel(const Args a) {
    constexpr int S = Depth<KIND>::STAGES;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[S];
    __shared__ __align__(8) uint64_t empty[S];
    __shared__ StageInfo info[S];
    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(smem_u32(&full[st]), 1);
            mbar_init(smem_u32(&empty[st]), NC_WARPS);
        }
        mbar_fence_init();
        if (a.one_scale_out && blockIdx.x == 0) *a.one_scale_out = a.one_s2;
    }
    __syncthreads();
    if (threadIdx.x >= CONSUMERS) {
        if (threadIdx.x == CONSUMERS) produce<KIND, SF>(a, smem, full, empty, info);
        return;
    }
    consume<KIND, WQU, SF>(a, smem, full, empty, info);
}

// ---------------------------------------------------------------------------
// s2 = amax(|W|)/2688: per-tile maxima, then one CTA per tensor
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(THREADS) amax_tiles_kernel(const Args a, uint32_t *partial) {
    __shared__ uint32_t red[THREADS / 32];
    int t = 0;
    TensorRef T;
    bool have = false;
    for (int64_t tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x) {
        if (!have || tile >= T.tile_end) {
            const int n = a.table ? a.n_tensors : 1;
            if (have && t + 1 < n) ++t;
            for (;;) {
                T.d = a.table ? a.table[t] : a.one;
                T.nblk = T.d.out * (T.d.in / 16);
                T.tile_end = T.d.tile_begin + (T.nblk + TILE_BLOCKS - 1) / TILE_BLOCKS;
                if (tile < T.tile_end || t + 1 >= n) break;
                ++t;
            }
            have = true;
            if (tile >= T.tile_end) break;      // uniform across the CTA: no barrier is skipped by some threads only
        }
        // TILE_BLOCKS blocks x 32 bytes per tile: two 16-byte loads per thread
        const int64_t first_sb = (tile - T.d.tile_begin) * TILE_BLOCKS * 2;
        const int64_t nsb = 2 * T.nblk;
        uint32_t mx = 0;
#pragma unroll
        for (int u = 0; u < 2 * TILE_BLOCKS / THREADS; ++u) {
            const int64_t sb = first_sb + u * THREADS + threadIdx.x;
            if (sb < nsb) {
                const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(T.d.W) + sb);
                const uint32_t m2 = __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                                             __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu));
                mx = max(mx, max(m2 & 0xffffu, m2 >> 16));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(FULL, mx, o));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
        __syncthreads();
        if (threadIdx.x < 32) {
            uint32_t v = threadIdx.x < THREADS / 32 ? red[threadIdx.x] : 0u;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(FULL, v, o));
            if (threadIdx.x == 0) partial[tile] = v;
        }
        __syncthreads();
    }
}

// One CTA per tensor: max of its tiles' maxima, s2 = fl(A / 2688).
__global__ void __launch_bounds__(THREADS) s2_finish_kernel(const Args a, const uint32_t *partial, float *one_out) {
    __shared__ uint32_t red[THREADS / 32];
    const focus_tensor_desc d = a.table ? a.table[blockIdx.x] : a.one;
    const int64_t nblk = d.out * (d.in / 16);
    const int64_t ntiles = (nblk + TILE_BLOCKS - 1) / TILE_BLOCKS;
    uint32_t mx = 0;
    for (int64_t i = threadIdx.x; i < ntiles; i += THREADS) mx = max(mx, partial[d.tile_begin + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(FULL, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint32_t v = threadIdx.x < THREADS / 32 ? red[threadIdx.x] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(FULL, v, o));
        if (threadIdx.x == 0) {
            if (v >= 0x7f80u) atomicOr(&g_error_flags, 1u);
            const float A = __uint_as_float(v << 16);
            const float s2 = __fdiv_rn(A, 2688.0f);
            if (a.table) *d.s2 = s2;
            else *one_out = s2;
        }
    }
}

// ---------------------------------------------------------------------------
// FourOverSix with one scale per token (model card, section "Calibration",
// activation bullet): s_t = fl(max_row |x| / 2688), then every block of the
// row as for the weights.  One CTA per row and loop: the first pass reads the
// row from HBM for its maximum, the second reads it again (from L2) and
// writes codes, scales and, when asked, the dequantized row.  A row whose
// maximum is 0 has s_t = 0: block scales 0x38 (1.0), codes 0, values 0.
// ---------------------------------------------------------------------------

constexpr int ROW_THREADS = 128;               // threads of the per-token kernel: 8 rows in flight per SM (12% faster than 256)

// Byte of scale (r, c) in the 128x4-atom layout of sm_100 block-scaled GEMMs
// (rows padded to 128, columns to 4; `groups` = column groups of 4): atoms of
// 128 rows x 4 columns, 512 bytes, stored band by band with the column groups
// inner; inside an atom, byte 16*(r mod 32) + 4*((r div 32) mod 4) + (c mod 4).
__device__ __forceinline__ int64_t swizzled_offset(int64_t r, int64_t c, int64_t groups) {
    return (((r >> 7) * groups + (c >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (c & 3);
}

// SWZ: the block scales go straight into the 128x4-atom layout (`scales` holds
// the padded buffer), and the CTAs that draw a padding row, or a row's padding
// columns, write them 0.  RTN: plain NVFP4 round to nearest (the target 6
// alone) instead of FourOverSix.
template <bool SWZ, bool RTN = false>
__global__ void __launch_bounds__(ROW_THREADS) f46_rows_kernel(const uint16_t *__restrict__ X, int64_t rows, int64_t cols,
                                                           float *__restrict__ row_scales, uint8_t *__restrict__ codes,
                                                           uint8_t *__restrict__ scales, uint16_t *__restrict__ Xq) {
    __shared__ uint32_t red[ROW_THREADS / 32];
    const int64_t chunks = cols / 8;          // 16-byte words of a row
    const int64_t nb = cols / 16;
    const int64_t groups = (nb + 3) / 4;      // SWZ: column groups of the padded layout
    const int64_t rows_out = SWZ ? (rows + 127) / 128 * 128 : rows;
    for (int64_t r = blockIdx.x; r < rows_out; r += gridDim.x) {
        if (SWZ && r >= rows) {                // a padding row: its words of every column group are 0
            for (int64_t g = threadIdx.x; g < groups; g += ROW_THREADS)
                *reinterpret_cast<uint32_t *>(scales + swizzled_offset(r, 4 * g, groups)) = 0u;
            continue;
        }
        const uint4 *xr = reinterpret_cast<const uint4 *>(X + r * cols);
        uint32_t mx = 0u;
        for (int64_t c = threadIdx.x; c < chunks; c += ROW_THREADS) {
            const uint4 v = xr[c];
            const uint32_t m2 = __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                                         __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu));
            mx = max(mx, max(m2 & 0xffffu, m2 >> 16));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(FULL, mx, o));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
        __syncthreads();
        uint32_t amax = 0u;
#pragma unroll
        for (int w = 0; w < ROW_THREADS / 32; ++w) amax = max(amax, red[w]);
        __syncthreads();                       // red is rewritten by the next row
        if (amax >= 0x7f80u) {                 // a non-finite value: flag it, write nothing of the row
            if (threadIdx.x == 0) atomicOr(&g_error_flags, 1u);
            continue;
        }
        const float s = __fdiv_rn(__uint_as_float(amax << 16), 2688.0f);
        if (threadIdx.x == 0) row_scales[r] = s;
        const F46Scale sc = f46_scale(s);
        for (int64_t b = threadIdx.x; b < nb; b += ROW_THREADS) {
            const int64_t blk = r * nb + b;
            uint32_t sb = 0x38u, cw[2] = {0u, 0u};
            uint4 o[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
            if (s != 0.0f) {
                const uint4 v0 = xr[2 * b], v1 = xr[2 * b + 1];
                const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                if (RTN) rtn_block(w, __uint_as_float(block_amax_bits(w) << 16), sc, sb, cw);
                else f46_block(w, __uint_as_float(block_amax_bits(w) << 16), sc, sb, cw);
                if (Xq) wq_words(cw, sb, s, o);
            }
            reinterpret_cast<uint2 *>(codes)[blk] = make_uint2(cw[0], cw[1]);
            scales[SWZ ? swizzled_offset(r, b, groups) : blk] = (uint8_t)sb;
            if (Xq) {
                __stcs(reinterpret_cast<uint4 *>(Xq) + 2 * blk, o[0]);
                __stcs(reinterpret_cast<uint4 *>(Xq) + 2 * blk + 1, o[1]);
            }
        }
        if (SWZ)                               // the row's padding columns (at most 3)
            for (int64_t c = nb + threadIdx.x; c < 4 * groups; c += ROW_THREADS) scales[swizzled_offset(r, c, groups)] = 0u;
    }
}

// ---------------------------------------------------------------------------
// E4M3 scale factors [rows][cols] (row-major, one byte per 16-element block)
// -> the 128x4-atom layout the sm_100 block-scaled tensor-core GEMM reads:
// rows padded to 128 and columns to 4, atoms of 128 rows x 4 columns (512
// bytes) stored band by band (column groups inner), scale (r, c) of an atom
// at byte 16*(r mod 32) + 4*(r div 32) + c.  One thread per 4-byte output
// word (one row's 4 scales): the writes are coalesced; padding is written 0.
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(THREADS) scales_swizzle_kernel(const uint8_t *__restrict__ lin, int64_t rows,
                                                                 int64_t cols, uint32_t *__restrict__ out,
                                                                 int64_t words) {
    const int64_t groups = (cols + 3) / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < words; wi += stride) {
        const int64_t atom = wi >> 7;                       // 128 words per atom
        const uint32_t in = (uint32_t)wi & 127u;            // word 4*(r mod 32) + (r div 32) of the atom
        const int64_t r = (atom / groups) * 128 + 32 * (in & 3u) + (in >> 2);
        const int64_t c0 = (atom % groups) * 4;
        uint32_t v = 0u;
        if (r < rows) {
            const uint8_t *src = lin + r * cols + c0;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (c0 + c < cols) v |= (uint32_t)src[c] << (8 * c);
        }
        out[wi] = v;
    }
}

// s2 = fl(A / 2688) of every tensor from the maxima a step accumulated
// (focus_step_fused_amax), one thread per tensor; the workspace word is
// cleared for the next step.
__global__ void __launch_bounds__(THREADS) s2_from_amax_kernel(const focus_tensor_desc *table, int n,
                                                               uint32_t *amax_ws) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n) return;
    const uint32_t v = amax_ws[t];
    if (v >= 0x7f80u) atomicOr(&g_error_flags, 1u);
    *table[t].s2 = __fdiv_rn(__uint_as_float(v << 16), 2688.0f);
    amax_ws[t] = 0u;
}

// ---------------------------------------------------------------------------
// standalone AdamW over a flat vector, four parameters per thread and loop
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(THREADS) adamw_kernel(float *__restrict__ p, const float *__restrict__ g,
                                                        float *__restrict__ v1, float *__restrict__ v2,
                                                        int64_t n, float step_size, float decay, Hyper h) {
    const int64_t n4 = n / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 P = reinterpret_cast<float4 *>(p)[i];
        const float4 G = __ldcs(reinterpret_cast<const float4 *>(g) + i);
        float4 A = reinterpret_cast<float4 *>(v1)[i];
        float4 B = reinterpret_cast<float4 *>(v2)[i];
        adamw_one(P.x, G.x, A.x, B.x, step_size, decay, h);
        adamw_one(P.y, G.y, A.y, B.y, step_size, decay, h);
        adamw_one(P.z, G.z, A.z, B.z, step_size, decay, h);
        adamw_one(P.w, G.w, A.w, B.w, step_size, decay, h);
        reinterpret_cast<float4 *>(p)[i] = P;
        reinterpret_cast<float4 *>(v1)[i] = A;
        reinterpret_cast<float4 *>(v2)[i] = B;
    }
    // the n % 4 tail
    const int64_t i = 4 * n4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (blockIdx.x == 0 && i < n) {
        float P = p[i], A = v1[i], B = v2[i];
        adamw_one(P, g[i], A, B, step_size, decay, h);
        p[i] = P; v1[i] = A; v2[i] = B;
    }
}

}  // namespace focus
