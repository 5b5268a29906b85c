// focus_capi.cu -- the extern "C" boundary of libfocus.so (declared in focus.h).
//
// Every entry point checks its arguments on the host, then enqueues kernels on
// the caller's stream; nothing is allocated and nothing synchronizes except
// focus_get_error().  Launch sizes: a persistent grid of (SM count) x (CTAs
// resident per SM, from the occupancy calculator), cached per device.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "focus.h"
#include "focus_trace.cuh"
#include "focus_kernels.cuh"
#include "focus_mx.cuh"
#include "focus_rows.cuh"

namespace focus {

static_assert(sizeof(focus_tensor_desc) == 144, "descriptor layout is part of the ABI");

namespace {

constexpr int MAX_DEVICES = 64;

static_assert(SF_ACC == (int)FOCUS_STEP_ACCUMULATE && SF_WRITE_GRAD == (int)FOCUS_STEP_WRITE_GRAD &&
                  SF_PACK == (int)FOCUS_STEP_PACK_UPDATED && SF_WQU == (int)FOCUS_STEP_WQ_UPDATED &&
                  (SF_AMAX & 15) == 0,
              "the step kernels' option bits are the FOCUS_STEP_* flags, plus one for the tensor maxima");

// The step kernels: one per FOCUS_STEP_WQ_UPDATED setting that reads the other
// options at run time, and ones compiled for the option sets of a calibration
// loop: the step with the export and the tensor maxima, with either alone or
// neither, and the last micro-batch's step (accumulate, W' of the update).
constexpr int STEP_KERNELS = 7;
template <bool WQU, int SF>
constexpr int step_kernel_index() {
    return !WQU ? (SF == SF_RUNTIME ? 0 : SF == (SF_PACK | SF_AMAX) ? 2 : SF == SF_PACK ? 3 : SF == SF_AMAX ? 4
                                                                                      : SF == 0 ? 5 : -1)
                : (SF == SF_RUNTIME ? 1 : SF == SF_ACC ? 6 : -1);
}

template <int KIND, bool WQU = false, int SF = SF_RUNTIME>
int pipe_occupancy() {
    cudaFuncSetAttribute(pipe_kernel<KIND, WQU, SF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)stage_smem_bytes<KIND>());
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, pipe_kernel<KIND, WQU, SF>, CTA_THREADS,
                                                  stage_smem_bytes<KIND>());
    return occ;
}

struct DeviceInfo {
    int sms = 0;
    int occ_step[STEP_KERNELS] = {};   // by step_kernel_index
    int occ_fwd = 0, occ_bwd = 0, occ_f46 = 0, occ_rtn = 0,
        occ_rows = 0, occ_rows_swz = 0, occ_amax = 0, occ_adam = 0;
    int occ_rows_rtn[2] = {0, 0};   // per-token NVFP4: row-major scales, 128x4 layout
    int occ_mx[3] = {0, 0, 0}, occ_mx_multi[3] = {0, 0, 0}, occ_mx_export = 0;
    int occ_mx_multi_export[3] = {0, 0, 0};   // run-time options; export and W' of the update; export alone
};

std::once_flag g_once[MAX_DEVICES];
DeviceInfo g_info[MAX_DEVICES];

int device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return FOCUS_ERR_CUDA;
    std::call_once(g_once[dev], [dev] {
        DeviceInfo &d = g_info[dev];
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        d.occ_fwd = pipe_occupancy<KIND_FWD>();
        d.occ_bwd = pipe_occupancy<KIND_BWD>();
        d.occ_f46 = pipe_occupancy<KIND_F46>();
        d.occ_rtn = pipe_occupancy<KIND_RTN>();
        d.occ_step[step_kernel_index<false, SF_RUNTIME>()] = pipe_occupancy<KIND_STEP, false, SF_RUNTIME>();
        d.occ_step[step_kernel_index<true, SF_RUNTIME>()] = pipe_occupancy<KIND_STEP, true, SF_RUNTIME>();
        d.occ_step[step_kernel_index<false, SF_PACK | SF_AMAX>()] = pipe_occupancy<KIND_STEP, false, SF_PACK | SF_AMAX>();
        d.occ_step[step_kernel_index<false, SF_PACK>()] = pipe_occupancy<KIND_STEP, false, SF_PACK>();
        d.occ_step[step_kernel_index<false, SF_AMAX>()] = pipe_occupancy<KIND_STEP, false, SF_AMAX>();
        d.occ_step[step_kernel_index<false, 0>()] = pipe_occupancy<KIND_STEP, false, 0>();
        d.occ_step[step_kernel_index<true, SF_ACC>()] = pipe_occupancy<KIND_STEP, true, SF_ACC>();
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_rows, f46_rows_kernel<false>, ROW_THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_rows_swz, f46_rows_kernel<true>, ROW_THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_rows_rtn[0], f46_rows_kernel<false, true>, ROW_THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_rows_rtn[1], f46_rows_kernel<true, true>, ROW_THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_amax, amax_tiles_kernel, THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_adam, adamw_kernel, THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx[0], mx_kernel<KIND_FWD>, THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx[1], mx_kernel<KIND_BWD>, THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx[2], mx_kernel<KIND_STEP>, THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx_multi[0], mx_multi_kernel<KIND_FWD>,
                                                      MX_TILE_BLOCKS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx_multi[1], mx_multi_kernel<KIND_BWD>,
                                                      MX_TILE_BLOCKS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx_multi[2], mx_multi_kernel<KIND_STEP>,
                                                      MX_TILE_BLOCKS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx_export, mx_kernel<KIND_STEP, true>, THREADS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx_multi_export[1],
                                                      mx_multi_kernel<KIND_STEP, true, SF_PACK | SF_WQU>,
                                                      MX_TILE_BLOCKS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx_multi_export[2], mx_multi_kernel<KIND_STEP, true, SF_PACK>,
                                                      MX_TILE_BLOCKS, 0);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.occ_mx_multi_export[0], mx_multi_kernel<KIND_STEP, true>,
                                                      MX_TILE_BLOCKS, 0);
    });
    DeviceInfo &d = g_info[dev];
    bool step_ok = true;
    for (int k = 0; k < STEP_KERNELS; ++k) step_ok = step_ok && d.occ_step[k] > 0;
    if (d.sms <= 0 || d.occ_fwd <= 0 || d.occ_bwd <= 0 || !step_ok || d.occ_f46 <= 0 || d.occ_rtn <= 0 ||
        d.occ_rows <= 0 || d.occ_rows_swz <= 0 || d.occ_rows_rtn[0] <= 0 || d.occ_rows_rtn[1] <= 0 || d.occ_amax <= 0 || d.occ_adam <= 0 || d.occ_mx[0] <= 0 ||
        d.occ_mx[1] <= 0 || d.occ_mx[2] <= 0 || d.occ_mx_multi[0] <= 0 || d.occ_mx_multi[1] <= 0 ||
        d.occ_mx_multi[2] <= 0 || d.occ_mx_export <= 0 || d.occ_mx_multi_export[0] <= 0 ||
        d.occ_mx_multi_export[1] <= 0 || d.occ_mx_multi_export[2] <= 0)
        return FOCUS_ERR_CUDA;
    *out = &d;
    return FOCUS_OK;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A tensor holds at most 2^31 - 2^16 blocks (about 3.4e10 weights), so that
// block and sub-block indices within it fit 32-bit arithmetic in the kernels.
constexpr int64_t MAX_BLOCKS = (INT64_C(1) << 31) - (INT64_C(1) << 16);

int check_shape(int64_t out, int64_t in) {
    if (out < 0 || in < 0 || (in % 16) != 0) return FOCUS_ERR_SHAPE;
    if (in > 0 && out > MAX_BLOCKS / (in / 16 > 0 ? in / 16 : 1)) return FOCUS_ERR_SHAPE;
    return FOCUS_OK;
}

int check_s2(float s2) { return (s2 > 0.0f && std::isfinite(s2)) ? FOCUS_OK : FOCUS_ERR_VALUE; }

int64_t tiles_of(int64_t out, int64_t in) {
    const int64_t nblk = out * (in / 16);
    return (nblk + TILE_BLOCKS - 1) / TILE_BLOCKS;
}

int64_t grid_for(int64_t tiles, int sms, int occ) {
    int64_t g = (int64_t)sms * occ;
    return tiles < g ? tiles : g;
}

int launch_status() {
    return cudaGetLastError() == cudaSuccess ? FOCUS_OK : FOCUS_ERR_CUDA;
}

focus_tensor_desc one_desc(const uint16_t *W, const uint16_t *dWq, uint16_t *Wq, const float *m, const float *q,
                           int64_t out, int64_t in) {
    focus_tensor_desc d;
    std::memset(&d, 0, sizeof d);
    d.W = W;
    d.dWq = dWq;
    d.Wq = Wq;
    d.m = const_cast<float *>(m);
    d.q = const_cast<float *>(q);
    d.out = out;
    d.in = in;
    d.block_begin = 0;
    d.tile_begin = 0;
    return d;
}

Hyper make_hyper(float lr_m, float lr_q, float beta1, float beta2, float eps, float wd, int64_t step) {
    const double bc1 = 1.0 - std::pow((double)beta1, (double)step);
    const double bc2 = 1.0 - std::pow((double)beta2, (double)step);
    Hyper h;
    h.lr_m_step = (float)((double)lr_m / bc1);
    h.lr_q_step = (float)((double)lr_q / bc1);
    h.decay_m = (float)(1.0 - (double)lr_m * wd);
    h.decay_q = (float)(1.0 - (double)lr_q * wd);
    h.beta1 = beta1;
    h.one_m_beta1 = (float)(1.0 - (double)beta1);
    h.beta2 = beta2;
    h.one_m_beta2 = (float)(1.0 - (double)beta2);
    h.inv_bc2_sqrt = (float)(1.0 / std::sqrt(bc2));
    h.eps = eps;
    return h;
}

int check_hyper(float lr, float beta1, float beta2, float eps, float wd, int64_t step) {
    if (!(lr >= 0.0f) || !std::isfinite(lr)) return FOCUS_ERR_VALUE;
    if (!(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f)) return FOCUS_ERR_VALUE;
    if (!(eps >= 0.0f) || !std::isfinite(eps) || !(wd >= 0.0f) || !std::isfinite(wd)) return FOCUS_ERR_VALUE;
    if (step < 1) return FOCUS_ERR_VALUE;
    return FOCUS_OK;
}

}  // namespace
}  // namespace focus

using namespace focus;

namespace {
template <int KIND, bool WQU = false, int SF = SF_RUNTIME>
int launch_on(const Args &a, cudaStream_t s) {
    static_assert(KIND == KIND_STEP ? step_kernel_index<WQU, SF>() >= 0 : (!WQU && SF == SF_RUNTIME),
                  "a pipe_kernel instance that device_info does not set up");
    DeviceInfo *di;
    int rc = device_info(&di);
    if (rc) return rc;
    if (a.total_tiles == 0 && !a.one_scale_out) return FOCUS_OK;
    int occ;
    if constexpr (KIND == KIND_STEP) occ = di->occ_step[step_kernel_index<WQU, SF>()];
    else occ = KIND == KIND_FWD ? di->occ_fwd : KIND == KIND_BWD ? di->occ_bwd : KIND == KIND_RTN ? di->occ_rtn
                                                                                             : di->occ_f46;
    int64_t grid = grid_for(a.total_tiles, di->sms, occ);
    if (grid < 1) grid = 1;   // the pack of an empty tensor still writes its tensor scale
    pipe_kernel<KIND, WQU, SF><<<(unsigned)grid, CTA_THREADS, stage_smem_bytes<KIND>(), s>>>(a);
    return launch_status();
}

int check_shape_mx(int64_t out, int64_t in) {
    if (out < 0 || in < 0 || (in % 32) != 0) return FOCUS_ERR_SHAPE;
    if (in > 0 && out > MAX_BLOCKS / (in / 32 > 0 ? in / 32 : 1)) return FOCUS_ERR_SHAPE;
    return FOCUS_OK;
}

template <int KIND, bool EXPORT = false>
int launch_mx(const MxArgs &a, cudaStream_t s) {
    DeviceInfo *di;
    int rc = device_info(&di);
    if (rc) return rc;
    if (a.nblk == 0) return FOCUS_OK;
    const int occ = EXPORT ? di->occ_mx_export : di->occ_mx[KIND];
    const int64_t grid = grid_for((a.nblk + THREADS - 1) / THREADS, di->sms, occ);
    mx_kernel<KIND, EXPORT><<<(unsigned)grid, THREADS, 0, s>>>(a);
    return launch_status();
}

template <int KIND>
int launch_mx_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, int accumulate, int write_grad,
                    const Hyper &hp, cudaStream_t s, int pack_updated = 0, int wq_updated = 0) {
    if (n < 0 || total_tiles < 0) return FOCUS_ERR_VALUE;
    if (n == 0 || total_tiles == 0) return FOCUS_OK;
    if (!descs_dev) return FOCUS_ERR_NULL;
    if (!aligned16(descs_dev)) return FOCUS_ERR_ALIGN;
    DeviceInfo *di;
    int rc = device_info(&di);
    if (rc) return rc;
    MxMultiArgs a{};
    a.table = descs_dev;
    a.n_tensors = n;
    a.total_tiles = total_tiles;
    a.accumulate = accumulate;
    a.write_grad = write_grad;
    a.pack_updated = pack_updated;
    a.wq_updated = wq_updated;
    a.hp = hp;
    if constexpr (KIND == KIND_STEP) {
        if (pack_updated || wq_updated) {
            // the export kernels compiled for the options of a calibration loop where
            // they apply (no accumulation, no gradient output), else the run-time one
            const int v = (accumulate || write_grad || !pack_updated) ? 0 : (wq_updated ? 1 : 2);
            const int64_t grid = grid_for(total_tiles, di->sms, di->occ_mx_multi_export[v]);
            if (v == 1) mx_multi_kernel<KIND, true, SF_PACK | SF_WQU><<<(unsigned)grid, MX_TILE_BLOCKS, 0, s>>>(a);
            else if (v == 2) mx_multi_kernel<KIND, true, SF_PACK><<<(unsigned)grid, MX_TILE_BLOCKS, 0, s>>>(a);
            else mx_multi_kernel<KIND, true><<<(unsigned)grid, MX_TILE_BLOCKS, 0, s>>>(a);
            return launch_status();
        }
    }
    const int64_t grid = grid_for(total_tiles, di->sms, di->occ_mx_multi[KIND]);
    mx_multi_kernel<KIND><<<(unsigned)grid, MX_TILE_BLOCKS, 0, s>>>(a);
    return launch_status();
}

int launch_s2(const Args &a, uint32_t *partial, float *one_out, int n_finish, cudaStream_t s) {
    DeviceInfo *di;
    int rc = device_info(&di);
    if (rc) return rc;
    if (a.total_tiles > 0) {
        const int64_t grid = grid_for(a.total_tiles, di->sms, di->occ_amax);
        amax_tiles_kernel<<<(unsigned)grid, THREADS, 0, s>>>(a, partial);
        if ((rc = launch_status())) return rc;
    }
    if (n_finish > 0) {
        s2_finish_kernel<<<(unsigned)n_finish, THREADS, 0, s>>>(a, partial, one_out);
        return launch_status();
    }
    return FOCUS_OK;
}
}  // namespace

// ---------------------------------------------------------------------------
// s2 without a caller workspace
//
// Some callers of this library have no way to hand it device memory: a
// runtime whose fixed memory pool owns every device allocation and forbids
// any other, or a latency-critical path that must never enter cudaMalloc (it
// can synchronize the device).  focus_s2_noalloc serves them: its per-tile
// maxima live in the array below, which is part of the library's device image
// (every GPU that loads the library keeps it until the process exits), so the
// call allocates nothing.  One word per 4096-weight tile: NOALLOC_TILES words
// cover a tensor of FOCUS_S2_NOALLOC_MAX_WEIGHTS weights.  The amax kernel
// writes every word the finishing kernel reads, so nothing has to be cleared
// between calls; two calls whose work overlaps on the GPU share the array and
// race.
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t NOALLOC_TILES = FOCUS_S2_NOALLOC_MAX_WEIGHTS / (TILE_BLOCKS * 16);
static_assert(NOALLOC_TILES * TILE_BLOCKS * 16 == FOCUS_S2_NOALLOC_MAX_WEIGHTS, "whole tiles");

static __device__ __align__(256) uint32_t g_s2_noalloc_scratch[NOALLOC_TILES];

std::mutex g_noalloc_mutex;
uint32_t *g_noalloc_ptr[MAX_DEVICES];   // the array's device address on each device, once found

// The scratch array's device address on device `dev` (current), or nullptr when
// the lookup fails.  A successful lookup is kept; a failed one (for instance
// inside a stream capture, where the lookup may be refused) is retried by the
// next call, and its error is taken off the runtime's error state so that the
// next entry point does not report it as its own launch failure.
uint32_t *noalloc_scratch(int dev) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_s2_noalloc_scratch) == cudaSuccess) {
            g_noalloc_ptr[dev] = static_cast<uint32_t *>(p);
        } else {
            (void)cudaGetLastError();
        }
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" {

const char *focus_status_string(int status) {
    switch (status) {
    case FOCUS_OK: return "FOCUS_OK";
    case FOCUS_ERR_NULL: return "FOCUS_ERR_NULL: a required pointer is NULL";
    case FOCUS_ERR_SHAPE: return "FOCUS_ERR_SHAPE: in must be a multiple of 16, sizes non-negative";
    case FOCUS_ERR_ALIGN: return "FOCUS_ERR_ALIGN: tensor base addresses must be 16-byte aligned";
    case FOCUS_ERR_VALUE: return "FOCUS_ERR_VALUE: a scalar argument is out of range";
    case FOCUS_ERR_WORKSPACE: return "FOCUS_ERR_WORKSPACE: workspace missing or too small";
    case FOCUS_ERR_CUDA: return "FOCUS_ERR_CUDA: a CUDA call or launch failed";
    case FOCUS_ERR_NONFINITE_INPUT: return "FOCUS_ERR_NONFINITE_INPUT: a kernel met a non-finite input";
    case FOCUS_ERR_DEVICE_TIMEOUT: return "FOCUS_ERR_DEVICE_TIMEOUT: a kernel's pipeline wait ran out";
    default: return "FOCUS_ERR_UNKNOWN";
    }
}

const char *focus_version(void) { return "0.1.0"; }

size_t focus_s2_workspace_bytes(int64_t out, int64_t in) {
    if (check_shape(out, in)) return 0;
    const int64_t t = tiles_of(out, in);
    return (size_t)(t > 0 ? t : 1) * sizeof(uint32_t);
}

int focus_s2(const uint16_t *W, int64_t out, int64_t in, float *s2_dev, void *ws_dev, size_t ws_bytes,
             focus_stream_t stream) {
    FOCUS_RANGE();
    int rc = check_shape(out, in);
    if (rc) return rc;
    if (!s2_dev || !ws_dev || (!W && out * in > 0)) return FOCUS_ERR_NULL;
    if (!aligned16(W) || !aligned16(ws_dev)) return FOCUS_ERR_ALIGN;
    if (ws_bytes < focus_s2_workspace_bytes(out, in)) return FOCUS_ERR_WORKSPACE;
    Args a{};
    a.table = nullptr;
    a.n_tensors = 1;
    a.one = one_desc(W, nullptr, nullptr, nullptr, nullptr, out, in);
    a.total_tiles = tiles_of(out, in);
    return launch_s2(a, static_cast<uint32_t *>(ws_dev), s2_dev, 1, (cudaStream_t)stream);
}

int focus_s2_noalloc(const uint16_t *W, int64_t out, int64_t in, float *s2_dev, focus_stream_t stream) {
    FOCUS_RANGE();
    int rc = check_shape(out, in);
    if (rc) return rc;
    if (!s2_dev || (!W && out * in > 0)) return FOCUS_ERR_NULL;
    if (!aligned16(W)) return FOCUS_ERR_ALIGN;
    const int64_t tiles = tiles_of(out, in);
    if (tiles > NOALLOC_TILES) return FOCUS_ERR_WORKSPACE;   // larger than the built-in scratch covers
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return FOCUS_ERR_CUDA;
    // The first call on a device, with that device current, looks up the device
    // address of the scratch array (its name in host code is only a stand-in).
    uint32_t *scratch = noalloc_scratch(dev);
    if (scratch == nullptr) return FOCUS_ERR_CUDA;
    Args a{};
    a.table = nullptr;
    a.n_tensors = 1;
    a.one = one_desc(W, nullptr, nullptr, nullptr, nullptr, out, in);
    a.total_tiles = tiles;
    return launch_s2(a, scratch, s2_dev, 1, (cudaStream_t)stream);
}

int focus_fwd(const uint16_t *W, const float *m, const float *q, float s2, int64_t out, int64_t in, uint16_t *Wq,
              focus_stream_t stream) {
    FOCUS_RANGE();
    int rc = check_shape(out, in);
    if (rc) return rc;
    if ((rc = check_s2(s2))) return rc;
    if (out * in == 0) return FOCUS_OK;
    if (!W || !m || !q || !Wq) return FOCUS_ERR_NULL;
    if (!aligned16(W) || !aligned16(m) || !aligned16(q) || !aligned16(Wq)) return FOCUS_ERR_ALIGN;
    Args a{};
    a.one = one_desc(W, nullptr, Wq, m, q, out, in);
    a.write_wq = 1;
    a.one_s2 = s2;
    a.n_tensors = 1;
    a.total_tiles = tiles_of(out, in);
    return launch_on<KIND_FWD>(a, (cudaStream_t)stream);
}

int focus_pack_nvfp4(const uint16_t *W, const float *m, const float *q, float s2, int64_t out, int64_t in,
                     uint8_t *codes, uint8_t *scales, float *tensor_scale_dev, focus_stream_t stream) {
    FOCUS_RANGE();
    int rc = check_shape(out, in);
    if (rc) return rc;
    if ((rc = check_s2(s2))) return rc;
    if (!tensor_scale_dev) return FOCUS_ERR_NULL;
    if (out * in > 0) {
        if (!W || !m || !q || !codes || !scales) return FOCUS_ERR_NULL;
        if (!aligned16(W) || !aligned16(m) || !aligned16(q) || !aligned16(codes) || !aligned16(scales))
            return FOCUS_ERR_ALIGN;
    }
    Args a{};
    a.one_scale_out = tensor_scale_dev;
    a.one = one_desc(W, nullptr, nullptr, m, q, out, in);
    a.one.codes = codes;
    a.one.scales = scales;
    a.one_s2 = s2;
    a.n_tensors = 1;
    a.total_tiles = tiles_of(out, in);
    return launch_on<KIND_FWD>(a, (cudaStream_t)stream);
}

int focus_ste_bwd(const uint16_t *W, const uint16_t *dWq, const float *m, const float *q, float s2, int64_t out,
                  int64_t in, float *dm, float *dq, int accumulate, focus_stream_t stream) {
    FOCUS_RANGE();
    int rc = check_shape(out, in);
    if (rc) return rc;
    if ((rc = check_s2(s2))) return rc;
    if (accumulate != 0 && accumulate != 1) return FOCUS_ERR_VALUE;
    if (out * in == 0) return FOCUS_OK;
    if (!W || !dWq || !m || !q || !dm || !dq) return FOCUS_ERR_NULL;
    if (!aligned16(W) || !aligned16(dWq) || !aligned16(m) || !aligned16(q) || !aligned16(dm) || !aligned16(dq))
        return FOCUS_ERR_ALIGN;
    Args a{};
    a.one = one_desc(W, dWq, nullptr, m, q, out, in);
    a.one.dm = dm;
    a.one.dq = dq;
    a.one_s2 = s2;
    a.n_tensors = 1;
    a.accumulate = accumulate;
    a.total_tiles = tiles_of(out, in);
    return launch_on<KIND_BWD>(a, (cudaStream_t)stream);
}

int focus_adamw_step(float *p, const float *g, float *exp_avg, float *exp_avg_sq, int64_t n, float lr, float beta1,
                     float beta2, float eps, float weight_decay, int64_t step, focus_stream_t stream) {
    FOCUS_RANGE();
    if (n < 0) return FOCUS_ERR_SHAPE;
    int rc = check_hyper(lr, beta1, beta2, eps, weight_decay, step);
    if (rc) return rc;
    if (n == 0) return FOCUS_OK;
    if (!p || !g || !exp_avg || !exp_avg_sq) return FOCUS_ERR_NULL;
    if (!aligned16(p) || !aligned16(g) || !aligned16(exp_avg) || !aligned16(exp_avg_sq)) return FOCUS_ERR_ALIGN;
    DeviceInfo *di;
    if ((rc = device_info(&di))) return rc;
    const Hyper h = make_hyper(lr, lr, beta1, beta2, eps, weight_decay, step);
    const int64_t per_cta = (int64_t)THREADS * 4;
    const int64_t grid = grid_for((n + per_cta - 1) / per_cta, di->sms, di->occ_adam);
    adamw_kernel<<<(unsigned)(grid > 0 ? grid : 1), THREADS, 0, (cudaStream_t)stream>>>(
        p, g, exp_avg, exp_avg_sq, n, h.lr_m_step, h.decay_m, h);
    return launch_status();
}

int focus_table_prepare(focus_tensor_desc *d, int n, int purpose, int64_t *total_tiles) {
    FOCUS_RANGE();
    if (!d || !total_tiles) return FOCUS_ERR_NULL;
    if (n < 0 || purpose < 0 || purpose > FOCUS_PURPOSE_ACT_SWIZZLED) return FOCUS_ERR_VALUE;
    int64_t tiles = 0, blocks = 0;
    if (purpose == FOCUS_PURPOSE_ACT || purpose == FOCUS_PURPOSE_ACT_SWIZZLED) {
        // activation tensors for the per-token calls: W = X, s2 = token scales;
        // tile_begin is the entry's first bundle of rows (rows padded to 128 for the
        // 128x4 layout; rs_bundles gives an entry's bundles)
        int64_t rows = 0;
        for (int i = 0; i < n; ++i) {
            focus_tensor_desc &e = d[i];
            int rc = check_shape(e.out, e.in);
            if (rc) return rc;
            if (e.in > RS_MAX_HIDDEN) return FOCUS_ERR_SHAPE;
            if (e.out * e.in > 0) {
                if (!e.W || !e.s2 || !e.codes || !e.scales) return FOCUS_ERR_NULL;
                const void *ptrs[] = {e.W, e.s2, e.codes, e.scales, e.Wq};
                for (const void *p : ptrs)
                    if (p && !aligned16(p)) return FOCUS_ERR_ALIGN;
            }
            e.block_begin = blocks;
            e.tile_begin = rows;
            blocks += e.out * (e.in / 16);
            if (e.out * e.in > 0)
                rows += rs_bundles(purpose == FOCUS_PURPOSE_ACT_SWIZZLED ? (e.out + 127) / 128 * 128 : e.out, e.in / 16);
        }
        *total_tiles = rows;
        return FOCUS_OK;
    }
    if (purpose == FOCUS_PURPOSE_MX) {
        for (int i = 0; i < n; ++i) {
            focus_tensor_desc &e = d[i];
            int rc = check_shape_mx(e.out, e.in);
            if (rc) return rc;
            const int64_t nblk = e.out * (e.in / 32);
            if (nblk > 0) {
                if (!e.W || !e.m || !e.q) return FOCUS_ERR_NULL;
                const void *ptrs[] = {e.W, e.m, e.q, e.Wq, e.codes, e.scales, e.dm, e.dq, e.dWq,
                                      e.m_exp_avg, e.m_exp_avg_sq, e.q_exp_avg, e.q_exp_avg_sq};
                for (const void *p : ptrs)
                    if (p && !aligned16(p)) return FOCUS_ERR_ALIGN;
                if ((e.codes == nullptr) != (e.scales == nullptr)) return FOCUS_ERR_NULL;
                if ((e.dm == nullptr) != (e.dq == nullptr)) return FOCUS_ERR_NULL;
            }
            e.block_begin = blocks;
            e.tile_begin = tiles;
            blocks += nblk;
            tiles += (nblk + MX_TILE_BLOCKS - 1) / MX_TILE_BLOCKS;
        }
        *total_tiles = tiles;
        return FOCUS_OK;
    }
    for (int i = 0; i < n; ++i) {
        focus_tensor_desc &e = d[i];
        int rc = check_shape(e.out, e.in);
        if (rc) return rc;
        if (!e.s2) return FOCUS_ERR_NULL;
        if (!aligned16(e.s2)) return FOCUS_ERR_ALIGN;
        const int64_t nblk = e.out * (e.in / 16);
        if (nblk > 0) {
            if (!e.W) return FOCUS_ERR_NULL;
            if (purpose != 3 && (!e.m || !e.q)) return FOCUS_ERR_NULL;
            if (purpose == 3 && !e.codes && !e.Wq) return FOCUS_ERR_NULL;     // FourOverSix writes something
            const void *ptrs[] = {e.W, e.m, e.q, e.Wq, e.codes, e.scales, e.dm, e.dq, e.dWq,
                                  e.m_exp_avg, e.m_exp_avg_sq, e.q_exp_avg, e.q_exp_avg_sq};
            for (const void *p : ptrs)
                if (p && !aligned16(p)) return FOCUS_ERR_ALIGN;
            if ((e.codes == nullptr) != (e.scales == nullptr)) return FOCUS_ERR_NULL;
            if (purpose == 1 && (!e.dWq || !e.m_exp_avg || !e.m_exp_avg_sq || !e.q_exp_avg || !e.q_exp_avg_sq))
                return FOCUS_ERR_NULL;
            if (purpose == 2 && (!e.dWq || !e.dm || !e.dq)) return FOCUS_ERR_NULL;
            if ((e.dm == nullptr) != (e.dq == nullptr)) return FOCUS_ERR_NULL;
        }
        e.block_begin = blocks;
        e.tile_begin = tiles;
        blocks += nblk;
        tiles += (nblk + TILE_BLOCKS - 1) / TILE_BLOCKS;
    }
    *total_tiles = tiles;
    return FOCUS_OK;
}

size_t focus_s2_multi_workspace_bytes(int64_t total_tiles) {
    return (size_t)(total_tiles > 0 ? total_tiles : 1) * sizeof(uint32_t);
}

int focus_s2_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, void *ws_dev, size_t ws_bytes,
                   focus_stream_t stream) {
    FOCUS_RANGE();
    if (n < 0 || total_tiles < 0) return FOCUS_ERR_VALUE;
    if (n == 0) return FOCUS_OK;
    if (!descs_dev || !ws_dev) return FOCUS_ERR_NULL;
    if (!aligned16(descs_dev) || !aligned16(ws_dev)) return FOCUS_ERR_ALIGN;
    if (ws_bytes < focus_s2_multi_workspace_bytes(total_tiles)) return FOCUS_ERR_WORKSPACE;
    Args a{};
    a.table = descs_dev;
    a.n_tensors = n;
    a.total_tiles = total_tiles;
    return launch_s2(a, static_cast<uint32_t *>(ws_dev), nullptr, n, (cudaStream_t)stream);
}

static int step_fused(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, const focus_hparams *hp,
                      int64_t step, unsigned flags, uint32_t *amax_ws, focus_stream_t stream) {
    if (n < 0 || total_tiles < 0) return FOCUS_ERR_VALUE;
    if (!hp) return FOCUS_ERR_NULL;
    int rc = check_hyper(hp->lr_m, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step);
    if (rc) return rc;
    if ((rc = check_hyper(hp->lr_q, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step))) return rc;
    if (flags & ~(unsigned)(FOCUS_STEP_ACCUMULATE | FOCUS_STEP_WRITE_GRAD | FOCUS_STEP_PACK_UPDATED |
                            FOCUS_STEP_WQ_UPDATED))
        return FOCUS_ERR_VALUE;
    if (n == 0) return FOCUS_OK;
    if (!descs_dev) return FOCUS_ERR_NULL;
    if (!aligned16(descs_dev)) return FOCUS_ERR_ALIGN;
    Args a{};
    a.table = descs_dev;
    a.n_tensors = n;
    a.total_tiles = total_tiles;
    a.write_wq = 1;
    a.accumulate = (flags & FOCUS_STEP_ACCUMULATE) ? 1 : 0;
    a.write_grad = (flags & FOCUS_STEP_WRITE_GRAD) ? 1 : 0;
    a.pack_updated = (flags & FOCUS_STEP_PACK_UPDATED) ? 1 : 0;
    a.amax_ws = amax_ws;
    a.hp = make_hyper(hp->lr_m, hp->lr_q, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step);
    // the kernel compiled for these options where there is one (FOCUS_STEP_WRITE_GRAD
    // always takes the kernel that reads them at run time)
    const cudaStream_t s = (cudaStream_t)stream;
    const int sf = (int)(flags & (FOCUS_STEP_ACCUMULATE | FOCUS_STEP_WRITE_GRAD | FOCUS_STEP_PACK_UPDATED)) |
                   (amax_ws ? SF_AMAX : 0);
    if (flags & FOCUS_STEP_WQ_UPDATED) {
        if (sf == SF_ACC) return launch_on<KIND_STEP, true, SF_ACC>(a, s);
        return launch_on<KIND_STEP, true>(a, s);
    }
    switch (sf) {
    case SF_PACK | SF_AMAX: return launch_on<KIND_STEP, false, SF_PACK | SF_AMAX>(a, s);
    case SF_PACK: return launch_on<KIND_STEP, false, SF_PACK>(a, s);
    case SF_AMAX: return launch_on<KIND_STEP, false, SF_AMAX>(a, s);
    case 0: return launch_on<KIND_STEP, false, 0>(a, s);
    default: return launch_on<KIND_STEP>(a, s);
    }
}

int focus_step_fused(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, const focus_hparams *hp,
                     int64_t step, unsigned flags, focus_stream_t stream) {
    FOCUS_RANGE();
    return step_fused(descs_dev, n, total_tiles, hp, step, flags, nullptr, stream);
}

int focus_step_fused_amax(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, const focus_hparams *hp,
                          int64_t step, unsigned flags, uint32_t *amax_ws, focus_stream_t stream) {
    FOCUS_RANGE();
    if (n > 0 && !amax_ws) return FOCUS_ERR_NULL;
    if (!aligned16(amax_ws)) return FOCUS_ERR_ALIGN;
    return step_fused(descs_dev, n, total_tiles, hp, step, flags, amax_ws, stream);
}

int focus_s2_from_amax(const focus_tensor_desc *descs_dev, int n, uint32_t *amax_ws, focus_stream_t stream) {
    FOCUS_RANGE();
    if (n < 0) return FOCUS_ERR_VALUE;
    if (n == 0) return FOCUS_OK;
    if (!descs_dev || !amax_ws) return FOCUS_ERR_NULL;
    if (!aligned16(descs_dev) || !aligned16(amax_ws)) return FOCUS_ERR_ALIGN;
    s2_from_amax_kernel<<<(unsigned)((n + THREADS - 1) / THREADS), THREADS, 0, (cudaStream_t)stream>>>(descs_dev, n,
                                                                                                      amax_ws);
    return launch_status();
}

int focus_fwd_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, focus_stream_t stream) {
    FOCUS_RANGE();
    if (n < 0 || total_tiles < 0) return FOCUS_ERR_VALUE;
    if (n == 0) return FOCUS_OK;
    if (!descs_dev) return FOCUS_ERR_NULL;
    if (!aligned16(descs_dev)) return FOCUS_ERR_ALIGN;
    Args a{};
    a.table = descs_dev;
    a.n_tensors = n;
    a.total_tiles = total_tiles;
    a.write_wq = 1;
    return launch_on<KIND_FWD>(a, (cudaStream_t)stream);
}

int focus_ste_bwd_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, int accumulate,
                        focus_stream_t stream) {
    FOCUS_RANGE();
    if (n < 0 || total_tiles < 0) return FOCUS_ERR_VALUE;
    if (accumulate != 0 && accumulate != 1) return FOCUS_ERR_VALUE;
    if (n == 0) return FOCUS_OK;
    if (!descs_dev) return FOCUS_ERR_NULL;
    if (!aligned16(descs_dev)) return FOCUS_ERR_ALIGN;
    Args a{};
    a.table = descs_dev;
    a.n_tensors = n;
    a.total_tiles = total_tiles;
    a.accumulate = accumulate;
    return launch_on<KIND_BWD>(a, (cudaStream_t)stream);
}

int focus_pack_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, focus_stream_t stream) {
    FOCUS_RANGE();
    if (n < 0 || total_tiles < 0) return FOCUS_ERR_VALUE;
    if (n == 0) return FOCUS_OK;
    if (!descs_dev) return FOCUS_ERR_NULL;
    if (!aligned16(descs_dev)) return FOCUS_ERR_ALIGN;
    Args a{};
    a.table = descs_dev;
    a.n_tensors = n;
    a.total_tiles = total_tiles;
    return launch_on<KIND_FWD>(a, (cudaStream_t)stream);
}

}  // extern "C"

namespace {
int weight_f46(const uint16_t *W, int64_t out, int64_t in, float s2, uint8_t *codes, uint8_t *scales, uint16_t *Wq,
               int rtn, cudaStream_t stream) {
    int rc = check_shape(out, in);
    if (rc) return rc;
    if ((rc = check_s2(s2))) return rc;
    if ((codes == nullptr) != (scales == nullptr)) return FOCUS_ERR_NULL;
    if (!codes && !Wq) return FOCUS_ERR_NULL;
    if (out * in == 0) return FOCUS_OK;
    if (!W) return FOCUS_ERR_NULL;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(scales) || !aligned16(Wq)) return FOCUS_ERR_ALIGN;
    Args a{};
    a.one = one_desc(W, nullptr, Wq, nullptr, nullptr, out, in);
    a.one.codes = codes;
    a.one.scales = scales;
    a.one_s2 = s2;
    a.n_tensors = 1;
    a.total_tiles = tiles_of(out, in);
    return rtn ? launch_on<KIND_RTN>(a, stream) : launch_on<KIND_F46>(a, stream);
}

int weight_f46_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, int rtn, cudaStream_t stream) {
    if (n < 0 || total_tiles < 0) return FOCUS_ERR_VALUE;
    if (n == 0) return FOCUS_OK;
    if (!descs_dev) return FOCUS_ERR_NULL;
    if (!aligned16(descs_dev)) return FOCUS_ERR_ALIGN;
    Args a{};
    a.table = descs_dev;
    a.n_tensors = n;
    a.total_tiles = total_tiles;
    return rtn ? launch_on<KIND_RTN>(a, stream) : launch_on<KIND_F46>(a, stream);
}
}  // namespace

extern "C" {

int focus_fouroversix_weight(const uint16_t *W, int64_t out, int64_t in, float s2, uint8_t *codes, uint8_t *scales,
                             uint16_t *Wq, focus_stream_t stream) {
    FOCUS_RANGE();
    return weight_f46(W, out, in, s2, codes, scales, Wq, 0, (cudaStream_t)stream);
}

int focus_fouroversix_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, focus_stream_t stream) {
    FOCUS_RANGE();
    return weight_f46_multi(descs_dev, n, total_tiles, 0, (cudaStream_t)stream);
}

int focus_nvfp4_weight(const uint16_t *W, int64_t out, int64_t in, float s2, uint8_t *codes, uint8_t *scales,
                       uint16_t *Wq, focus_stream_t stream) {
    FOCUS_RANGE();
    return weight_f46(W, out, in, s2, codes, scales, Wq, 1, (cudaStream_t)stream);
}

int focus_nvfp4_weight_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_tiles, focus_stream_t stream) {
    FOCUS_RANGE();
    return weight_f46_multi(descs_dev, n, total_tiles, 1, (cudaStream_t)stream);
}

}  // extern "C"

namespace {
// The staged per-token kernel over the rows of `a` (one entry or a device
// table), buffers sized for rows of a.max_in values.
template <bool SWZ, bool RTN>
int launch_rows_staged_t(const RowArgs &a, cudaStream_t stream) {
    static std::once_flag once[MAX_DEVICES];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return FOCUS_ERR_CUDA;
    std::call_once(once[dev], [] {
        cudaFuncSetAttribute(rows_staged_kernel<SWZ, RTN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(2 * RS_MAX_HIDDEN * 2));
    });
    DeviceInfo *di;
    int rc = device_info(&di);
    if (rc) return rc;
    // one stage holds a bundle of rows: at most RS_BPT * RS_THREADS blocks (32 KB)
    const uint32_t stage = (uint32_t)(RS_MAX_HIDDEN * 2);
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rows_staged_kernel<SWZ, RTN>, RS_CTA_THREADS,
                                                      2 * stage) != cudaSuccess ||
        occ <= 0)
        return FOCUS_ERR_CUDA;
    const int64_t grid = grid_for(a.total_rows, di->sms, occ);
    if (grid <= 0) return FOCUS_OK;
    rows_staged_kernel<SWZ, RTN><<<(unsigned)grid, RS_CTA_THREADS, 2 * stage, stream>>>(a, stage);
    return launch_status();
}

int launch_rows_staged(const RowArgs &a, bool rtn, bool swz, cudaStream_t stream) {
    if (swz && rtn) return launch_rows_staged_t<true, true>(a, stream);
    if (swz) return launch_rows_staged_t<true, false>(a, stream);
    if (rtn) return launch_rows_staged_t<false, true>(a, stream);
    return launch_rows_staged_t<false, false>(a, stream);
}

// The per-token quantizers over a prepared table of activation tensors.
int act_rows_multi(const focus_tensor_desc *descs_dev, int n, int64_t total_rows, int64_t max_hidden, bool rtn,
                   bool swz, cudaStream_t stream) {
    if (n < 0 || total_rows < 0) return FOCUS_ERR_VALUE;
    if (n == 0 || total_rows == 0) return FOCUS_OK;
    if (!descs_dev) return FOCUS_ERR_NULL;
    if (max_hidden < 16 || max_hidden % 16 != 0 || max_hidden > RS_MAX_HIDDEN) return FOCUS_ERR_SHAPE;
    RowArgs a{};
    a.table = descs_dev;
    a.n_tensors = n;
    a.total_rows = total_rows;
    a.max_in = max_hidden;
    return launch_rows_staged(a, rtn, swz, stream);
}

// The per-token quantizers: FourOverSix or NVFP4 round to nearest (rtn), the
// block scales row-major or in the 128x4-atom layout (swz: scales_bytes is
// the caller's buffer size).
int act_rows(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales, uint8_t *codes,
             uint8_t *scales, size_t scales_bytes, uint16_t *Xq, bool rtn, bool swz, cudaStream_t stream) {
    int rc = check_shape(tokens, hidden);
    if (rc) return rc;
    if (tokens * hidden == 0) return FOCUS_OK;
    if (!X || !token_scales || !codes || !scales) return FOCUS_ERR_NULL;
    if (!aligned16(X) || !aligned16(token_scales) || !aligned16(codes) || !aligned16(scales) || !aligned16(Xq))
        return FOCUS_ERR_ALIGN;
    if (swz && scales_bytes < focus_scales_swizzled_bytes(tokens, hidden / 16)) return FOCUS_ERR_WORKSPACE;
    if (hidden <= RS_MAX_HIDDEN) {                  // rows staged in shared memory
        RowArgs a{};
        a.table = nullptr;
        a.n_tensors = 1;
        a.total_rows = rs_bundles(swz ? (tokens + 127) / 128 * 128 : tokens, hidden / 16);
        a.max_in = hidden;
        a.one = one_desc(X, nullptr, Xq, nullptr, nullptr, tokens, hidden);
        a.one.s2 = token_scales;
        a.one.codes = codes;
        a.one.scales = scales;
        return launch_rows_staged(a, rtn, swz, stream);
    }
    DeviceInfo *di;
    if ((rc = device_info(&di))) return rc;
    const int64_t rows_out = swz ? (tokens + 127) / 128 * 128 : tokens;
    const int occ = rtn ? di->occ_rows_rtn[swz ? 1 : 0] : (swz ? di->occ_rows_swz : di->occ_rows);
    const int64_t grid = grid_for(rows_out, di->sms, occ);
    const unsigned g = (unsigned)grid;
    if (swz && rtn) f46_rows_kernel<true, true><<<g, ROW_THREADS, 0, stream>>>(X, tokens, hidden, token_scales, codes,
                                                                            scales, Xq);
    else if (swz) f46_rows_kernel<true><<<g, ROW_THREADS, 0, stream>>>(X, tokens, hidden, token_scales, codes,
                                                                      scales, Xq);
    else if (rtn) f46_rows_kernel<false, true><<<g, ROW_THREADS, 0, stream>>>(X, tokens, hidden, token_scales, codes,
                                                                             scales, Xq);
    else f46_rows_kernel<false><<<g, ROW_THREADS, 0, stream>>>(X, tokens, hidden, token_scales, codes, scales, Xq);
    return launch_status();
}
}  // namespace

extern "C" {

int focus_fouroversix_act(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales, uint8_t *codes,
                          uint8_t *scales, uint16_t *Xq, focus_stream_t stream) {
    FOCUS_RANGE();
    return act_rows(X, tokens, hidden, token_scales, codes, scales, 0, Xq, false, false, (cudaStream_t)stream);
}

int focus_fouroversix_act_swizzled(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales,
                                   uint8_t *codes, uint8_t *scales_swz, size_t scales_bytes, uint16_t *Xq,
                                   focus_stream_t stream) {
    FOCUS_RANGE();
    return act_rows(X, tokens, hidden, token_scales, codes, scales_swz, scales_bytes, Xq, false, true,
                    (cudaStream_t)stream);
}

int focus_nvfp4_act(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales, uint8_t *codes,
                    uint8_t *scales, uint16_t *Xq, focus_stream_t stream) {
    FOCUS_RANGE();
    return act_rows(X, tokens, hidden, token_scales, codes, scales, 0, Xq, true, false, (cudaStream_t)stream);
}

int focus_nvfp4_act_swizzled(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales, uint8_t *codes,
                             uint8_t *scales_swz, size_t scales_bytes, uint16_t *Xq, focus_stream_t stream) {
    FOCUS_RANGE();
    return act_rows(X, tokens, hidden, token_scales, codes, scales_swz, scales_bytes, Xq, true, true,
                    (cudaStream_t)stream);
}

int focus_fouroversix_act_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_rows,
                                int64_t max_hidden, int swizzled, focus_stream_t stream) {
    FOCUS_RANGE();
    return act_rows_multi(descs_dev, n_tensors, total_rows, max_hidden, false, swizzled != 0, (cudaStream_t)stream);
}

int focus_nvfp4_act_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_rows, int64_t max_hidden,
                          int swizzled, focus_stream_t stream) {
    FOCUS_RANGE();
    return act_rows_multi(descs_dev, n_tensors, total_rows, max_hidden, true, swizzled != 0, (cudaStream_t)stream);
}

int focus_mx_fwd(const uint16_t *W, const float *m, const float *q, int64_t out, int64_t in, uint16_t *Wq,
                 uint8_t *codes, uint8_t *scales, focus_stream_t stream) {
    FOCUS_RANGE();
    int rc = check_shape_mx(out, in);
    if (rc) return rc;
    if ((codes == nullptr) != (scales == nullptr)) return FOCUS_ERR_NULL;
    if (!Wq && !codes) return FOCUS_ERR_NULL;
    if (out * in == 0) return FOCUS_OK;
    if (!W || !m || !q) return FOCUS_ERR_NULL;
    if (!aligned16(W) || !aligned16(m) || !aligned16(q) || !aligned16(Wq) || !aligned16(codes) || !aligned16(scales))
        return FOCUS_ERR_ALIGN;
    MxArgs a{};
    a.W = W; a.m = const_cast<float *>(m); a.q = const_cast<float *>(q);
    a.Wq = Wq; a.codes = codes; a.scales = scales;
    a.nblk = out * (in / 32);
    return launch_mx<KIND_FWD>(a, (cudaStream_t)stream);
}

int focus_mx_ste_bwd(const uint16_t *W, const uint16_t *dWq, const float *m, const float *q, int64_t out, int64_t in,
                     float *dm, float *dq, int accumulate, focus_stream_t stream) {
    FOCUS_RANGE();
    int rc = check_shape_mx(out, in);
    if (rc) return rc;
    if (accumulate != 0 && accumulate != 1) return FOCUS_ERR_VALUE;
    if (out * in == 0) return FOCUS_OK;
    if (!W || !dWq || !m || !q || !dm || !dq) return FOCUS_ERR_NULL;
    if (!aligned16(W) || !aligned16(dWq) || !aligned16(m) || !aligned16(q) || !aligned16(dm) || !aligned16(dq))
        return FOCUS_ERR_ALIGN;
    MxArgs a{};
    a.W = W; a.dWq = dWq; a.m = const_cast<float *>(m); a.q = const_cast<float *>(q);
    a.dm = dm; a.dq = dq; a.accumulate = accumulate;
    a.nblk = out * (in / 32);
    return launch_mx<KIND_BWD>(a, (cudaStream_t)stream);
}

int focus_mx_step(const uint16_t *W, const uint16_t *dWq, float *m, float *q, float *m_exp_avg, float *m_exp_avg_sq,
                  float *q_exp_avg, float *q_exp_avg_sq, int64_t out, int64_t in, const focus_hparams *hp,
                  int64_t step, unsigned flags, uint16_t *Wq, float *dm, float *dq, focus_stream_t stream) {
    FOCUS_RANGE();
    int rc = check_shape_mx(out, in);
    if (rc) return rc;
    if (!hp) return FOCUS_ERR_NULL;
    if ((rc = check_hyper(hp->lr_m, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step))) return rc;
    if ((rc = check_hyper(hp->lr_q, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step))) return rc;
    if (flags & ~(unsigned)(FOCUS_STEP_ACCUMULATE | FOCUS_STEP_WRITE_GRAD | FOCUS_STEP_WQ_UPDATED))
        return FOCUS_ERR_VALUE;
    if (out * in == 0) return FOCUS_OK;
    if (!W || !dWq || !m || !q || !m_exp_avg || !m_exp_avg_sq || !q_exp_avg || !q_exp_avg_sq) return FOCUS_ERR_NULL;
    if ((flags & (FOCUS_STEP_ACCUMULATE | FOCUS_STEP_WRITE_GRAD)) && (!dm || !dq)) return FOCUS_ERR_NULL;
    const void *ptrs[] = {W, dWq, m, q, m_exp_avg, m_exp_avg_sq, q_exp_avg, q_exp_avg_sq, Wq, dm, dq};
    for (const void *p : ptrs)
        if (!aligned16(p)) return FOCUS_ERR_ALIGN;
    MxArgs a{};
    a.W = W; a.dWq = dWq; a.Wq = Wq; a.m = m; a.q = q;
    a.m_ea = m_exp_avg; a.m_eas = m_exp_avg_sq; a.q_ea = q_exp_avg; a.q_eas = q_exp_avg_sq;
    a.dm = dm; a.dq = dq;
    a.accumulate = (flags & FOCUS_STEP_ACCUMULATE) ? 1 : 0;
    a.write_grad = (flags & FOCUS_STEP_WRITE_GRAD) ? 1 : 0;
    a.wq_updated = (flags & FOCUS_STEP_WQ_UPDATED) ? 1 : 0;
    a.hp = make_hyper(hp->lr_m, hp->lr_q, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step);
    a.nblk = out * (in / 32);
    if (a.wq_updated) return launch_mx<KIND_STEP, true>(a, (cudaStream_t)stream);
    return launch_mx<KIND_STEP>(a, (cudaStream_t)stream);
}


int focus_mx_fwd_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                       focus_stream_t stream) {
    FOCUS_RANGE();
    return launch_mx_multi<KIND_FWD>(descs_dev, n_tensors, total_tiles, 0, 0, Hyper{}, (cudaStream_t)stream);
}

int focus_mx_ste_bwd_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles, int accumulate,
                           focus_stream_t stream) {
    FOCUS_RANGE();
    if (accumulate != 0 && accumulate != 1) return FOCUS_ERR_VALUE;
    return launch_mx_multi<KIND_BWD>(descs_dev, n_tensors, total_tiles, accumulate, 0, Hyper{},
                                     (cudaStream_t)stream);
}

int focus_mx_step_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                        const focus_hparams *hp, int64_t step, unsigned flags, focus_stream_t stream) {
    FOCUS_RANGE();
    if (!hp) return FOCUS_ERR_NULL;
    int rc;
    if ((rc = check_hyper(hp->lr_m, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step))) return rc;
    if ((rc = check_hyper(hp->lr_q, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step))) return rc;
    if (flags & ~(unsigned)(FOCUS_STEP_ACCUMULATE | FOCUS_STEP_WRITE_GRAD | FOCUS_STEP_PACK_UPDATED |
                            FOCUS_STEP_WQ_UPDATED))
        return FOCUS_ERR_VALUE;
    return launch_mx_multi<KIND_STEP>(descs_dev, n_tensors, total_tiles, (flags & FOCUS_STEP_ACCUMULATE) ? 1 : 0,
                                      (flags & FOCUS_STEP_WRITE_GRAD) ? 1 : 0,
                                      make_hyper(hp->lr_m, hp->lr_q, hp->beta1, hp->beta2, hp->eps,
                                                 hp->weight_decay, step),
                                      (cudaStream_t)stream, (flags & FOCUS_STEP_PACK_UPDATED) ? 1 : 0,
                                      (flags & FOCUS_STEP_WQ_UPDATED) ? 1 : 0);
}

size_t focus_scales_swizzled_bytes(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0) return 0;
    return (size_t)(((rows + 127) / 128) * 128) * (size_t)(((cols + 3) / 4) * 4);
}

int focus_scales_swizzle(const uint8_t *scales, int64_t rows, int64_t cols, uint8_t *out, size_t out_bytes,
                         focus_stream_t stream) {
    FOCUS_RANGE();
    if (rows < 0 || cols < 0) return FOCUS_ERR_SHAPE;
    const size_t need = focus_scales_swizzled_bytes(rows, cols);
    if (need == 0) return FOCUS_OK;
    if (!out || (!scales && rows * cols > 0)) return FOCUS_ERR_NULL;
    if (!aligned16(out) || !aligned16(scales)) return FOCUS_ERR_ALIGN;
    if (out_bytes < need) return FOCUS_ERR_WORKSPACE;
    DeviceInfo *di;
    int rc = device_info(&di);
    if (rc) return rc;
    const int64_t words = (int64_t)(need / 4);
    const int64_t grid = grid_for((words + THREADS - 1) / THREADS, di->sms, 8);
    scales_swizzle_kernel<<<(unsigned)grid, THREADS, 0, (cudaStream_t)stream>>>(scales, rows, cols,
                                                                               reinterpret_cast<uint32_t *>(out), words);
    return launch_status();
}

int focus_get_error(focus_stream_t stream) {
    FOCUS_RANGE();
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FOCUS_ERR_CUDA;
    unsigned int flags = 0;
    if (cudaMemcpyFromSymbol(&flags, g_error_flags, sizeof flags) != cudaSuccess) return FOCUS_ERR_CUDA;
    if (flags) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_error_flags, &zero, sizeof zero) != cudaSuccess) return FOCUS_ERR_CUDA;
        return (flags & 8u) ? FOCUS_ERR_DEVICE_TIMEOUT : FOCUS_ERR_NONFINITE_INPUT;
    }
    return FOCUS_OK;
}

}  // extern "C"
