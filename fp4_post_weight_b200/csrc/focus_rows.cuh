// focus_rows.cuh -- the per-token quantizers (FourOverSix, or plain NVFP4 round
// to nearest) over one or more activation tensors in one launch, rows staged
// in shared memory.
//
// Model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct (our
// reproduction)", section "Calibration" (activation bullet: FourOverSix with
// one FP32 scale per token) and section "Perplexity" (the NVFP4 baseline: one
// scale per token).  For every row (token) r of X [tokens, hidden]:
//   s_r = fl(max_row |x| / 2688);  every 16-block as the weights' quantizer
//   with s_r in place of s2 (FourOverSix: the target 6 or 4 of the lower
//   squared error; NVFP4: the target 6);  a row of zeros has s_r = 0, scale
//   bytes 0x38, codes 0 and values 0.
//
// Work decomposition.  A CTA takes bundles U = blockIdx.x, blockIdx.x + grid,
// ... of the table's rows: consecutive rows of one entry, as many as fit 256
// threads with at most 4 blocks each (4 rows of 4096 values, 1 of 14336; with
// the 128x4 scale layout an entry's rows are padded to a multiple of 128 and a
// padding row only writes its scale words 0).  The CTA is 8 consumer warps and
// one producer warp.  The producer (one thread) stages the bundles in shared
// memory, two buffers in turn, each with one 1-D bulk copy (completion counted
// in bytes on the buffer's full barrier) once the 8 consumer warps have
// released the buffer's previous bundle (its empty barrier counts their
// arrivals), so the table walk and the copies never hold up a consumer warp.
// X is read from HBM once and both passes over a row read shared memory: the
// first computes the block maxima and each row's maximum (warp reduction, then
// one barrier of the consumer warps per bundle), the second quantizes every
// block.  The threads of a row own its blocks in turn (consecutive threads,
// consecutive 32-byte blocks) and keep their maxima in their own slots of a
// shared array between the passes.  Rows up to RS_MAX_HIDDEN values; longer
// rows take f46_rows_kernel.
//
// Every wait is bounded (focus_pipeline.cuh).  The consumers decide to stop
// uniformly through their bundle barrier; the producer stops when a release
// does not come in time, and before it exits waits (bounded) for every copy
// it issued whose release it has not seen.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "focus.h"
#include "focus_kernels.cuh"
#include "focus_pipeline.cuh"

namespace focus {

constexpr int RS_THREADS = 256;                           // 8 consumer warps per CTA
constexpr int RS_CTA_THREADS = RS_THREADS + 32;           // plus a producer warp
constexpr int RS_BPT = 4;                                 // blocks per thread at most
constexpr int64_t RS_MAX_HIDDEN = 16 * RS_THREADS * RS_BPT;   // 16384 values per row
constexpr float RCP_2688 = 1.0f / 2688.0f;                    // correctly rounded (evaluated at compile time)

// The activation tensors of one launch.  Each entry uses focus_tensor_desc
// fields as: W = X [out = tokens, in = hidden] bf16, s2 = token scales
// [tokens] (written), codes [tokens][hidden/2], scales (row-major
// [tokens][hidden/16], or the 128x4-atom buffer), Wq = X' (nullable),
// tile_begin = the entry's first bundle in the launch's numbering (below).
struct RowArgs {
    const focus_tensor_desc *table;  // device table, or nullptr: use `one`
    int n_tensors;
    int64_t total_rows;              // bundles of rows (rs_bundles) over all entries
    int64_t max_in;                  // the staging buffers hold rows of at most this many values
    focus_tensor_desc one;
};

// Rows are taken in bundles of consecutive rows of one entry: a row of nb
// blocks gets rs_tpr(nb) threads (a power of two from 32 to RS_THREADS, at
// most RS_BPT blocks each), and a bundle holds RS_THREADS / rs_tpr(nb) rows,
// at most RS_BPT * RS_THREADS blocks (32 KB of X).  A row of 4096 values is
// one of a bundle of 4 (64 threads each); a row of 14336 is a bundle of its
// own.  The entries' tile_begin count bundles.
__host__ __device__ constexpr int64_t rs_tpr(int64_t nb) {
    int64_t t = 32;
    while (t < RS_THREADS && t * RS_BPT < nb) t *= 2;
    return t;
}
__host__ __device__ constexpr int64_t rs_rows_per_bundle(int64_t nb) { return RS_THREADS / rs_tpr(nb); }
__host__ __device__ constexpr int64_t rs_bundles(int64_t rows_out, int64_t nb) {
    return (rows_out + rs_rows_per_bundle(nb) - 1) / rs_rows_per_bundle(nb);
}

// The record of a staged bundle, written by the producer before it completes
// the buffer's full barrier phase and read by the consumers after waiting on it.
struct RowStage {
    float *ts;          // token scales of the bundle's entry
    uint8_t *codes;
    uint8_t *scales;
    uint16_t *xq;
    int64_t r0;         // first row of the bundle within its entry
    int64_t nb;         // 16-blocks per row
    int64_t groups;     // column groups of 4 scales (128x4 layout)
    uint32_t rows;      // rows in the bundle (data rows, then padding rows of the 128x4 layout)
    uint32_t data;      // data rows in the bundle (staged)
    uint32_t tpr;       // threads per row
    uint32_t skip;      // 1: nothing to do (an entry wider than the buffers, or past the table)
};

// The producer: fill the record of bundle U and stage its data rows into `dst`
// (one bulk copy, the rows being consecutive in X; completion on `bar`;
// returns true), or, for a bundle without data rows or a skipped one,
// complete the barrier's phase without data (returns false).  An entry wider
// than the buffers is skipped and reported.
// (The entry of U is found by scanning the table forward from entry t, which
// the caller keeps: a CTA's bundles only increase.  The descriptor is read
// again for every bundle rather than held in registers across the loop.)
template <bool SWZ>
__device__ __forceinline__ bool stage_bundle(const RowArgs &a, int64_t U, int &t, unsigned char *dst, uint64_t *bar,
                                             RowStage &rec) {
    const uint32_t b = smem_u32(bar);
    const int n = a.table ? a.n_tensors : 1;
    focus_tensor_desc d;
    int64_t rows_out = 0, end;
    for (;;) {
        d = a.table ? a.table[t] : a.one;
        rows_out = (d.out > 0 && d.in > 0) ? (SWZ ? (d.out + 127) / 128 * 128 : d.out) : 0;
        end = d.tile_begin + rs_bundles(rows_out, d.in / 16);
        if (U < end || t + 1 >= n) break;
        ++t;
    }
    rec.skip = 1u;
    if (U < end) {
        const int64_t nb = d.in / 16;
        const int64_t rpb = rs_rows_per_bundle(nb);
        const int64_t r0 = (U - d.tile_begin) * rpb;
        const int64_t rows = rows_out - r0 < rpb ? rows_out - r0 : rpb;
        const int64_t data = d.out - r0 < 0 ? 0 : (d.out - r0 < rows ? d.out - r0 : rows);
        rec.ts = d.s2;
        rec.codes = d.codes;
        rec.scales = d.scales;
        rec.xq = d.Wq;
        rec.r0 = r0;
        rec.nb = nb;
        rec.groups = (nb + 3) / 4;
        rec.rows = (uint32_t)rows;
        rec.data = (uint32_t)data;
        rec.tpr = (uint32_t)rs_tpr(nb);
        if (d.in > a.max_in) {
            if (r0 == 0) atomicOr(&g_error_flags, 2u);
        } else {
            rec.skip = 0u;
            if (data > 0) {
                const uint32_t bytes = (uint32_t)(data * d.in * 2);
                mbar_arrive_expect_tx(b, bytes);
                bulk_g2s(smem_u32(dst), d.W + r0 * d.in, bytes, b);
                return true;
            }
        }
    }
    mbar_arrive(b);
    return false;
}

// Named barrier 1 over the consumer warps (the producer warp never takes
// part): every consumer thread arrives with `pred`; returns whether any of
// them passed true.
__device__ __forceinline__ bool consumers_sync_or(bool pred) {
    uint32_t r;
    asm volatile("{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, 1, %2, p; selp.u32 %0, 1, 0, q; }"
                 : "=r"(r)
                 : "r"((uint32_t)pred), "n"(RS_THREADS)
                 : "memory");
    return r != 0;
}

// swizzled_offset in 32-bit arithmetic: a tensor of this kernel has fewer than
// 2^31 blocks in rows of at most 1024, so its padded 128x4 buffer (rows rounded
// up to 128, columns to 4) holds fewer than 2^32 bytes.
__device__ __forceinline__ uint32_t swizzled_offset32(uint32_t r, uint32_t c, uint32_t groups) {
    return (((r >> 7) * groups + (c >> 2)) << 9) + ((r & 31u) << 4) + (((r >> 5) & 3u) << 2) + (c & 3u);
}

// Pass 2 of one consumer thread over its row of a staged bundle: the row's
// scale from the warps' maxima, then this thread's blocks (b = li + j*tpr).
// (Row indices fit 32 bits: a tensor holds fewer than 2^31 blocks.)
template <bool SWZ, bool RTN>
__device__ __forceinline__ void quantize_row_part(const RowStage &rec, const unsigned char *row, const uint32_t *red,
                                                  const uint32_t *amax_s, int tid, uint32_t ri, uint32_t li,
                                                  bool data) {
    const uint32_t tpr = rec.tpr;
    const uint32_t r = (uint32_t)rec.r0 + ri;
    const uint32_t groups = (uint32_t)rec.groups;
    uint8_t *const scales = rec.scales;
    if (!data) {                            // a padding row of the 128x4 layout: its words are 0
        if (SWZ)
            for (uint32_t g = li; g < groups; g += tpr)
                *reinterpret_cast<uint32_t *>(scales + swizzled_offset32(r, 4u * g, groups)) = 0u;
        return;
    }
    const uint32_t nbu = (uint32_t)rec.nb;
    uint32_t amax = 0u;
    const uint32_t wpr = tpr / 32u, w0 = ri * wpr;
    for (uint32_t w = 0; w < wpr; ++w) amax = max(amax, red[w0 + w]);
    if (amax >= 0x7f80u) {                  // a non-finite value: flag it, write nothing of the row
        if (li == 0) atomicOr(&g_error_flags, 1u);
        return;
    }
    const float A_row = __uint_as_float(amax << 16);
    // s = fl(A_row / 2688): the twice-corrected quotient by the correctly rounded
    // 1/2688 (bit-identical to the IEEE division while nothing underflows)
    const float s = A_row >= 0x1p-100f ? div_full(A_row, 2688.0f, RCP_2688) : div_rn_slow(A_row, 2688.0f);
    if (li == 0) rec.ts[r] = s;
    // this thread's blocks (a tensor holds fewer than 2^31 blocks, so block
    // indices fit 32 bits)
    const uint32_t jn = li < nbu ? (nbu - 1u - li) / tpr + 1u : 0u;
    const uint32_t base = r * nbu;
    uint2 *const codes = reinterpret_cast<uint2 *>(rec.codes);
    uint4 *const xq = reinterpret_cast<uint4 *>(rec.xq);
    if (s == 0.0f) {                        // a row of zeros: scale bytes 0x38, codes 0, values 0
        for (uint32_t j = 0; j < jn; ++j) {
            const uint32_t b = li + j * tpr, blk = base + b;
            codes[blk] = make_uint2(0u, 0u);
            scales[SWZ ? swizzled_offset32(r, b, groups) : blk] = 0x38u;
            if (xq) {
                __stcs(xq + 2ull * blk, make_uint4(0u, 0u, 0u, 0u));
                __stcs(xq + 2ull * blk + 1, make_uint4(0u, 0u, 0u, 0u));
            }
        }
    } else {
        const F46Scale sc = f46_scale(s);
        // the warp's lanes take the same number of iterations (the first lane's,
        // the most), so that for round to nearest each can vote for the fast code
        const uint32_t jw = RTN ? __shfl_sync(FULL, jn, 0) : jn;
#pragma unroll 1
        for (uint32_t j = 0; j < jw; ++j) {
            const uint32_t b = li + j * tpr, blk = base + b;
            const bool mine = j < jn;
            const float Ab = mine ? __uint_as_float(amax_s[j * RS_THREADS + tid] << 16) : 0.0f;
            const bool fast = RTN && __all_sync(FULL, !mine || f46_fast_range(Ab, sc));
            if (!mine) continue;
            const uint4 *p = reinterpret_cast<const uint4 *>(row) + 2u * b;
            const uint4 v0 = p[0], v1 = p[1];
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            uint32_t sb, cw[2];
            if (!RTN) f46_block(w, Ab, sc, sb, cw);
            else if (fast) rtn_block<true>(w, Ab, sc, sb, cw);
            else rtn_block(w, Ab, sc, sb, cw);
            codes[blk] = make_uint2(cw[0], cw[1]);
            scales[SWZ ? swizzled_offset32(r, b, groups) : blk] = (uint8_t)sb;
            if (xq) {
                uint4 o[2];
                wq_words(cw, sb, s, o);
                __stcs(xq + 2ull * blk, o[0]);
                __stcs(xq + 2ull * blk + 1, o[1]);
            }
        }
    }
    if (SWZ)                                // the row's padding columns (at most 3)
        for (uint32_t c = nbu + li; c < 4u * groups; c += tpr)
            scales[swizzled_offset32(r, c, groups)] = 0u;
}

// The producer warp's lane 0: stages the CTA's bundles into the two buffers in
// turn, each once the consumer warps have released the buffer's previous
// bundle, then waits (bounded) for any copy it issued whose release it has not
// seen, so that no copy is in flight when the CTA exits.
template <bool SWZ>
__device__ __forceinline__ void rows_produce(const RowArgs &a, unsigned char *smem, uint32_t stage_bytes,
                                             uint64_t *full, uint64_t *empty, RowStage *info) {
    int tn = 0;                      // cursor over the table
    uint32_t pending = 0, pending_parity = 0;
    uint32_t it = 0;
    for (int64_t U = blockIdx.x; U < a.total_rows; U += gridDim.x, ++it) {
        const uint32_t st = it & 1u, ph = (it >> 1) & 1u;
        if (!mbar_wait(smem_u32(&empty[st]), ph ^ 1u)) {
            atomicOr(&g_error_flags, 8u);
            break;
        }
        pending &= ~(1u << st);      // released: its copy had landed
        if (stage_bundle<SWZ>(a, U, tn, smem + st * stage_bytes, &full[st], info[st])) {
            pending |= 1u << st;
            pending_parity = (pending_parity & ~(1u << st)) | (ph << st);
        }
    }
    for (uint32_t st = 0; st < 2; ++st)
        if ((pending >> st) & 1u)
            if (!mbar_wait(smem_u32(&full[st]), (pending_parity >> st) & 1u)) atomicOr(&g_error_flags, 8u);
}

// Three CTAs of 288 threads per SM (72 registers a thread at most: the
// FourOverSix kernels spill 4 and 16 bytes at that bound).
template <bool SWZ, bool RTN>
__global__ void __launch_bounds__(RS_CTA_THREADS, 3) rows_staged_kernel(const RowArgs a, uint32_t stage_bytes) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[2];
    __shared__ __align__(8) uint64_t empty[2];
    __shared__ RowStage info[2];
    __shared__ uint32_t red[2][RS_THREADS / 32];
    __shared__ uint32_t amax_s[RS_BPT * RS_THREADS];   // block maxima; each thread keeps only its own
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        for (int st = 0; st < 2; ++st) {
            mbar_init(smem_u32(&full[st]), 1);
            mbar_init(smem_u32(&empty[st]), RS_THREADS / 32);
        }
        mbar_fence_init();
    }
    __syncthreads();
    if (tid >= RS_THREADS) {
        if (tid == RS_THREADS) rows_produce<SWZ>(a, smem, stage_bytes, full, empty, info);
        return;
    }
    uint32_t it = 0;
    for (int64_t U = blockIdx.x; U < a.total_rows; U += gridDim.x, ++it) {
        const uint32_t st = it & 1u, ph = (it >> 1) & 1u;
        const unsigned char *bundle = smem + st * stage_bytes;
        const bool ok = mbar_wait(smem_u32(&full[st]), ph);
        const RowStage &rec = info[st];
        const bool skip = !ok || rec.skip != 0u;
        // this thread's row of the bundle and its place in it
        const uint32_t tpr = rec.tpr;
        const uint32_t ri = (uint32_t)tid / tpr, li = (uint32_t)tid % tpr;
        const uint32_t nbu = (uint32_t)rec.nb;
        const bool data = !skip && ri < rec.data;
        const unsigned char *row = bundle + (size_t)ri * nbu * 32u;
        // pass 1: the block maxima of this thread's blocks and their maximum
        uint32_t mx = 0u;
        if (data) {
#pragma unroll 2
            for (int j = 0; j < RS_BPT; ++j) {
                const uint32_t b = li + (uint32_t)j * tpr;
                if (b < nbu) {
                    const uint4 *p = reinterpret_cast<const uint4 *>(row) + 2u * b;
                    const uint4 v0 = p[0], v1 = p[1];
                    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                    const uint32_t ab = block_amax_bits(w);
                    amax_s[j * RS_THREADS + tid] = ab;
                    mx = max(mx, ab);
                }
            }
        }
        mx = __reduce_max_sync(FULL, mx);       // a warp's lanes belong to one row (tpr >= 32)
        if (lane == 0) red[st][warp] = mx;
        // the row maxima are complete (and a wait that ran out stops every consumer here)
        if (consumers_sync_or(!ok)) {
            if (tid == 0) atomicOr(&g_error_flags, 8u);
            break;
        }
        if (!skip && ri < rec.rows)
            quantize_row_part<SWZ, RTN>(rec, row, red[st], amax_s, tid, ri, li, data);
        // this warp is done with the buffer and its record
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[st]));
    }
}

}  // namespace focus
