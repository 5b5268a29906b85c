// focus_mx.cuh -- the MXFP4 variant of the FOCUS quantizer on sm_100a.
//
// Sources: "Technische Samenvatting: FOCUS ...", section "Probleemstelling"
// (MXFP4: one E8M0 scale per 32 values) and section "Methodologie", items 2
// and 3 (quantization scale = hardware scale x learnable coefficient; each
// hardware block of 32 is cut into sub-blocks of 8 with a coefficient each);
// the structure of the card's equations ("FOCUS NVFP4 scales for
// Llama-3.2-1B-Instruct", section "What this is").  Per 32-block b with
// sub-blocks k = 0..3 (no tensor scale):
//   x_b  = fl(A_b * m_b)
//   S_b  = 2^(floor(log2 x_b) - 2), exponent clamped to [-127, 127] (E8M0;
//          the OCP Microscaling rule on the scaled maximum); 1 when x_b == 0
//   D_k  = fl(S_b * sigmoid(q_k));  y_i = fl(w_i / D_k)
//   c_i  = E2M1_rne(clamp(y_i, -6, 6));  w'_i = bf16(fl(c_i * S_b))
// Straight-through: dm_b = [x_b >= 2^-125] (A_b/4) sum g (in ? c - y : c)
// (32 exact products summed in binary64, rounded once), dq_k = -(1 - sigma_k)
// S_b sum_k in g y (binary32).
//
// Work decomposition: one thread per 32-block; W and dW' arrive as four
// 16-byte loads each, m as one float, q and its moments as one float4 each.
// No shared-memory staging: a thread has 128 bytes of loads in flight, enough
// at full occupancy.  mx_kernel strides over the blocks of one tensor;
// mx_multi_kernel walks the tiles (4096 weights, 128 blocks) of a table of
// tensors, one launch for a whole model.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "focus_kernels.cuh"

namespace focus {

struct MxArgs {
    const uint16_t *W;
    const uint16_t *dWq;
    uint16_t *Wq;              // nullable
    float *m, *q;              // [nblk], [4*nblk]
    float *m_ea, *m_eas, *q_ea, *q_eas;
    uint8_t *codes;            // nullable: [nblk] x 16 bytes
    uint8_t *scales;           // nullable: [nblk] E8M0 bytes
    float *dm, *dq;            // bwd outputs; step: accumulators / gradient outputs
    int64_t nblk;
    int accumulate;
    int write_grad;
    int pack_updated;          // step, export build: codes+scales of the UPDATED m and q
    int wq_updated;            // step, export build: W' of the UPDATED m and q
    Hyper hp;
};

// The MXFP4 step's options fixed at compile time (SF: the SF_* bits of the
// NVFP4 step, SF_WQU for FOCUS_STEP_WQ_UPDATED) or read from MxArgs
// (SF_RUNTIME); see StepOpt.
template <int SF>
struct MxOpt {
    static __device__ __forceinline__ bool acc(const MxArgs &a) { return SF < 0 ? a.accumulate != 0 : (SF & SF_ACC) != 0; }
    static __device__ __forceinline__ bool write_grad(const MxArgs &a) {
        return SF < 0 ? a.write_grad != 0 : (SF & SF_WRITE_GRAD) != 0;
    }
    static __device__ __forceinline__ bool pack(const MxArgs &a) {
        return SF < 0 ? a.pack_updated != 0 : (SF & SF_PACK) != 0;
    }
    static __device__ __forceinline__ bool wqu(const MxArgs &a) {
        return SF < 0 ? a.wq_updated != 0 : (SF & SF_WQU) != 0;
    }
};

// E8M0 exponent of the scaled maximum x (see the header comment) and S = 2^e.
__device__ __forceinline__ int mx_exponent(float x) {
    if (x == 0.0f) return 0;
    if (!(x >= 0x1p-126f)) return -127;                  // negative, subnormal: below the clamp
    const int e = (int)((__float_as_uint(x) >> 23) & 0xffu) - 127 - 2;
    return e < -127 ? -127 : e;
}
__device__ __forceinline__ float pow2f(int e) {           // 2^e for e in [-127, 127]
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : 0x1p-127f;
}

// The export of one 32-block from the UPDATED m and q (qn): the same
// arithmetic as the forward below, so the result is bit for bit what the
// forward writes when run after the step.  Codes and scale when pack_updated,
// W' when wq_updated.  The block's W is read again here (the step's first
// read left it in L1) rather than held in sixteen registers across the
// update.
template <int SF>
__device__ __forceinline__ void mx_encode(const MxArgs &a, int64_t blk, float A, float m, const float *qn) {
    const bool want_codes = MxOpt<SF>::pack(a) && a.codes != nullptr;
    const bool want_wq = MxOpt<SF>::wqu(a) && a.Wq != nullptr;
    if (!want_codes && !want_wq) return;
    uint32_t w[16];
    {
        const uint4 *Wp = reinterpret_cast<const uint4 *>(a.W) + 4 * blk;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 v = __ldg(Wp + j);
            w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
        }
    }
    if (!finitef(m) || !finitef(qn[0]) || !finitef(qn[1]) || !finitef(qn[2]) || !finitef(qn[3]))
        atomicOr(&g_error_flags, 1u);
    const float x = __fmul_rn(A, m);
    const int e = mx_exponent(x);
    const float S = pow2f(e);
    const uint64_t S2 = f2_pack(S, S);
    uint32_t codes[4];
    float sg[4];                                  // as in mx_block: one warp vote for the fast sigmoids
    {
        bool ok = true;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            double s64u;
            ok = sigmoid_fast_try(qn[k], sg[k], s64u) && ok;
        }
        if (!__all_sync(__activemask(), ok)) {
#pragma unroll
            for (int k = 0; k < 4; ++k) sg[k] = sigmoid_rn(qn[k]);
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float D = __fmul_rn(S, sg[k]);
        uint64_t y2[4];
        if (D >= 0x1p-60f && D <= 0x1p60f && A <= 0x1p60f) {
            const float nr = -rcp_rn(D);
            const uint64_t D2 = f2_pack(D, D), nr2 = f2_pack(nr, nr);
#pragma unroll
            for (int j = 0; j < 4; ++j) y2[j] = div_by_f2(bf16x2_neg_f2(w[4 * k + j]), D2, nr2);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                y2[j] = f2_pack(div_rn_slow(bf16_lo(w[4 * k + j]), D), div_rn_slow(bf16_hi(w[4 * k + j]), D));
        }
        uint32_t code = 0u, o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t byte = e2m1_pair(f2_lo(y2[j]), f2_hi(y2[j]));
            code |= byte << (8 * j);
            if (want_wq) {
                const uint32_t h2 = e2m1_pair_f16x2(byte);
                const float c0 = __half2float(__ushort_as_half(lo16(h2)));
                const float c1 = __half2float(__ushort_as_half(hi16(h2)));
                const uint64_t p = f2_mul(f2_pack(c0, c1), S2);
                o[j] = pack_bf16x2(f2_lo(p), f2_hi(p));
            }
        }
        codes[k] = code;
        if (want_wq) __stcs(reinterpret_cast<uint4 *>(a.Wq) + 4 * blk + k, make_uint4(o[0], o[1], o[2], o[3]));
    }
    if (want_codes) {
        reinterpret_cast<uint4 *>(a.codes)[blk] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        a.scales[blk] = (uint8_t)(e + 127);
    }
}

// One 32-block of the tensor `a` describes.  EXPORT (step only): the codes,
// scale and/or W' are those of the updated m and q (mx_encode) instead of the
// forward's, a compile-time choice so that the plain step keeps its registers.
template <int KIND, bool EXPORT = false, int SF = SF_RUNTIME>
__device__ __forceinline__ void mx_block(const MxArgs &a, int64_t blk) {
    using O = MxOpt<SF>;
    {
        uint32_t w[16], g[16];
        const uint4 *Wp = reinterpret_cast<const uint4 *>(a.W) + 4 * blk;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 v = EXPORT ? __ldg(Wp + j) : __ldcs(Wp + j);    // the export reads it again
            w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
        }
        if (KIND != KIND_FWD) {
            const uint4 *Gp = reinterpret_cast<const uint4 *>(a.dWq) + 4 * blk;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = __ldcs(Gp + j);
                g[4 * j] = v.x; g[4 * j + 1] = v.y; g[4 * j + 2] = v.z; g[4 * j + 3] = v.w;
            }
        }
        float m = a.m[blk];
        float4 q4 = reinterpret_cast<const float4 *>(a.q)[blk];
        float qk[4] = {q4.x, q4.y, q4.z, q4.w};

        uint32_t am = 0u;
#pragma unroll
        for (int j = 0; j < 16; ++j) am = __vmaxu2(am, w[j] & 0x7fff7fffu);
        const uint32_t abits = max(am & 0xffffu, am >> 16);
        const float A = __uint_as_float(abits << 16);
        bool bad = abits >= 0x7f80u || !finitef(m) || !finitef(qk[0]) || !finitef(qk[1]) || !finitef(qk[2]) ||
                   !finitef(qk[3]);

        const float x = __fmul_rn(A, m);
        const int e = mx_exponent(x);
        const float S = pow2f(e);
        const bool inS = x >= 0x1p-125f;
        const uint64_t S2 = f2_pack(S, S);

        // the sub-blocks' sigmoids: in the step, the table-driven evaluation when it
        // decides the rounding for every sub-block of every active lane (one warp
        // vote), else the direct binary64 evaluation for the warp (the same bits
        // either way; the forward and backward kernels keep the direct one, which
        // fits their registers better)
        float sig[4], sq[4];
        {
            bool ok = KIND == KIND_STEP;
            if (KIND == KIND_STEP) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    double s64u;
                    ok = sigmoid_fast_try(qk[k], sig[k], s64u) && ok;
                }
            }
            if (!__all_sync(__activemask(), ok)) {
#pragma unroll
                for (int k = 0; k < 4; ++k) sig[k] = sigmoid_rn(qk[k]);
            }
        }
        double sm = 0.0;              // sum of g*(in ? c - y : c): exact products, binary64 sum (a block's
                                      // gradient may nearly cancel, and AdamW at step 1 compares it with eps)
        uint32_t codes[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float D = __fmul_rn(S, sig[k]);
            uint64_t y2[4];
            if (D >= 0x1p-60f && D <= 0x1p60f && A <= 0x1p60f) {
                const float nr = -rcp_rn(D);
                const uint64_t D2 = f2_pack(D, D), nr2 = f2_pack(nr, nr);
#pragma unroll
                for (int j = 0; j < 4; ++j) y2[j] = div_by_f2(bf16x2_neg_f2(w[4 * k + j]), D2, nr2);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    y2[j] = f2_pack(div_rn_slow(bf16_lo(w[4 * k + j]), D), div_rn_slow(bf16_hi(w[4 * k + j]), D));
            }
            uint32_t code = 0u, o[4];
            uint64_t sq2 = 0ull;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t byte = e2m1_pair(f2_lo(y2[j]), f2_hi(y2[j]));
                code |= byte << (8 * j);
                const uint32_t h2 = e2m1_pair_f16x2(byte);
                const float c0 = __half2float(__ushort_as_half(lo16(h2)));
                const float c1 = __half2float(__ushort_as_half(hi16(h2)));
                if (KIND != KIND_BWD) {
                    const uint64_t p = f2_mul(f2_pack(c0, c1), S2);          // c*S: exact (a power of two)
                    o[j] = pack_bf16x2(f2_lo(p), f2_hi(p));
                }
                if (KIND != KIND_FWD) {
                    const float ylo = f2_lo(y2[j]), yhi = f2_hi(y2[j]);
                    const float ilo = fabsf(ylo) <= 6.0f ? ylo : 0.0f, ihi = fabsf(yhi) <= 6.0f ? yhi : 0.0f;
                    const uint64_t g2 = bf16x2_f2(g[4 * k + j]);
                    sm = fma((double)f2_lo(g2), (double)__fsub_rn(c0, ilo), sm);
                    sm = fma((double)f2_hi(g2), (double)__fsub_rn(c1, ihi), sm);
                    sq2 = f2_fma(g2, f2_pack(ilo, ihi), sq2);
                }
            }
            codes[k] = code;
            if (KIND != KIND_BWD && a.Wq && !(EXPORT && O::wqu(a)))
                __stcs(reinterpret_cast<uint4 *>(a.Wq) + 4 * blk + k, make_uint4(o[0], o[1], o[2], o[3]));
            sq[k] = (KIND != KIND_FWD) ? __fadd_rn(f2_lo(sq2), f2_hi(sq2)) : 0.0f;
        }
        if (KIND != KIND_BWD && a.codes && !(EXPORT && O::pack(a))) {
            reinterpret_cast<uint4 *>(a.codes)[blk] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            a.scales[blk] = (uint8_t)(e + 127);
        }
        if (KIND != KIND_FWD) {
            float gm = inS ? (float)((double)A * 0.25 * sm) : 0.0f;
            float gq[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) gq[k] = -__fmul_rn(__fmul_rn(__fsub_rn(1.0f, sig[k]), S), sq[k]);
            if (O::acc(a)) {
                gm = __fadd_rn(a.dm[blk], gm);
                const float4 p = reinterpret_cast<const float4 *>(a.dq)[blk];
                gq[0] = __fadd_rn(p.x, gq[0]); gq[1] = __fadd_rn(p.y, gq[1]);
                gq[2] = __fadd_rn(p.z, gq[2]); gq[3] = __fadd_rn(p.w, gq[3]);
            }
            if (!bad && !(finitef(gm) && finitef(gq[0]) && finitef(gq[1]) && finitef(gq[2]) && finitef(gq[3])))
                atomicOr(&g_error_flags, 4u);
            if (KIND == KIND_BWD || O::write_grad(a)) {
                a.dm[blk] = gm;
                reinterpret_cast<float4 *>(a.dq)[blk] = make_float4(gq[0], gq[1], gq[2], gq[3]);
            }
            if (KIND == KIND_STEP) {
                float v1 = a.m_ea[blk], v2 = a.m_eas[blk];
                adamw_one(m, gm, v1, v2, a.hp.lr_m_step, a.hp.decay_m, a.hp);
                a.m[blk] = m; a.m_ea[blk] = v1; a.m_eas[blk] = v2;
                const float4 e1 = reinterpret_cast<const float4 *>(a.q_ea)[blk];
                const float4 e2 = reinterpret_cast<const float4 *>(a.q_eas)[blk];
                uint64_t p01 = f2_pack(qk[0], qk[1]), p23 = f2_pack(qk[2], qk[3]);
                uint64_t a01 = f2_pack(e1.x, e1.y), a23 = f2_pack(e1.z, e1.w);
                uint64_t b01 = f2_pack(e2.x, e2.y), b23 = f2_pack(e2.z, e2.w);
                adamw_pair(p01, f2_pack(gq[0], gq[1]), a01, b01, a.hp.lr_q_step, a.hp.decay_q, a.hp);
                adamw_pair(p23, f2_pack(gq[2], gq[3]), a23, b23, a.hp.lr_q_step, a.hp.decay_q, a.hp);
                reinterpret_cast<float4 *>(a.q)[blk] = make_float4(f2_lo(p01), f2_hi(p01), f2_lo(p23), f2_hi(p23));
                reinterpret_cast<float4 *>(a.q_ea)[blk] = make_float4(f2_lo(a01), f2_hi(a01), f2_lo(a23), f2_hi(a23));
                reinterpret_cast<float4 *>(a.q_eas)[blk] = make_float4(f2_lo(b01), f2_hi(b01), f2_lo(b23), f2_hi(b23));
                if (EXPORT) {
                    const float qn[4] = {f2_lo(p01), f2_hi(p01), f2_lo(p23), f2_hi(p23)};
                    mx_encode<SF>(a, blk, A, m, qn);
                }
            }
        }
        if (bad) atomicOr(&g_error_flags, 1u);
    }
}

template <int KIND, bool EXPORT = false>
__global__ void __launch_bounds__(THREADS) mx_kernel(const MxArgs a) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < a.nblk; blk += stride)
        mx_block<KIND, EXPORT>(a, blk);
}

// ---------------------------------------------------------------------------
// Many tensors in one launch.  The table uses focus_tensor_desc with the
// MXFP4 shapes (m [out][in/32], q [out][in/8], scales [out][in/32]); its
// tile_begin fields count tiles of MX_TILE_BLOCKS 32-blocks (4096 weights).
// Each CTA keeps the descriptor of its current tensor in shared memory as an
// MxArgs, refreshed by thread 0 when the CTA's next tile lies past it (a
// CTA-uniform test, so the barriers around it are reached by every thread).
// ---------------------------------------------------------------------------

constexpr int MX_TILE_BLOCKS = 128;        // 32-blocks per tile, one per thread

struct MxMultiArgs {
    const focus_tensor_desc *table;
    int n_tensors;
    int64_t total_tiles;
    int accumulate;
    int write_grad;
    int pack_updated;
    int wq_updated;
    Hyper hp;
};

template <int KIND, bool EXPORT = false, int SF = SF_RUNTIME>
__global__ void __launch_bounds__(MX_TILE_BLOCKS, 7) mx_multi_kernel(const MxMultiArgs g) {
    const bool acc = SF < 0 ? g.accumulate != 0 : (SF & SF_ACC) != 0;
    const bool write_grad = SF < 0 ? g.write_grad != 0 : (SF & SF_WRITE_GRAD) != 0;
    __shared__ MxArgs sa;
    __shared__ int64_t s_range[2];          // tiles [first, end) of the current tensor
    int t = 0;                              // thread 0's table cursor
    int64_t first = 0, end = 0;
    for (int64_t tile = blockIdx.x; tile < g.total_tiles; tile += gridDim.x) {
        if (tile >= end) {
            __syncthreads();                // every thread is done with the previous descriptor
            if (threadIdx.x == 0) {
                focus_tensor_desc d;
                int64_t nb = 0, e = 0;
                for (;;) {
                    d = g.table[t];
                    nb = d.out * (d.in / 32);
                    e = d.tile_begin + (nb + MX_TILE_BLOCKS - 1) / MX_TILE_BLOCKS;
                    if (tile < e || t + 1 >= g.n_tensors) break;
                    ++t;
                }
                // a descriptor without a pointer the call needs is skipped and reported
                bool ok = d.W != nullptr && d.m != nullptr && d.q != nullptr;
                if (KIND != KIND_FWD) ok = ok && d.dWq != nullptr;
                if (KIND == KIND_STEP)
                    ok = ok && d.m_exp_avg && d.m_exp_avg_sq && d.q_exp_avg && d.q_exp_avg_sq;
                if (KIND == KIND_BWD || acc || write_grad) ok = ok && d.dm && d.dq;
                if ((d.codes == nullptr) != (d.scales == nullptr)) ok = false;
                if (!ok && nb > 0) atomicOr(&g_error_flags, 2u);
                sa.W = d.W; sa.dWq = d.dWq; sa.Wq = d.Wq;
                sa.m = d.m; sa.q = d.q;
                sa.m_ea = d.m_exp_avg; sa.m_eas = d.m_exp_avg_sq; sa.q_ea = d.q_exp_avg; sa.q_eas = d.q_exp_avg_sq;
                sa.codes = d.codes; sa.scales = d.scales;
                sa.dm = d.dm; sa.dq = d.dq;
                sa.nblk = ok ? nb : 0;
                sa.accumulate = g.accumulate;
                sa.write_grad = g.write_grad;
                sa.pack_updated = g.pack_updated;
                sa.wq_updated = g.wq_updated;
                sa.hp = g.hp;
                s_range[0] = d.tile_begin;
                s_range[1] = e;
            }
            __syncthreads();
            first = s_range[0];
            end = s_range[1];
            if (tile >= end) break;         // past the last tensor (uniform): nothing left
        }
        const int64_t blk = (tile - first) * MX_TILE_BLOCKS + threadIdx.x;
        if (tile >= first && blk < sa.nblk) mx_block<KIND, EXPORT, SF>(sa, blk);
    }
}

}  // namespace focus
