// focus_host.cu -- the fused step over tensors held in HOST memory.
//
// A runtime layer above the device entry points of focus_capi.cu: it owns no
// kernels.  For each tensor it uploads the step's inputs into one of
// HOST_SLOTS device slots carved from the caller's workspace, runs s2 (when
// asked), the fused step with the tensor maximum and s2 for the next step on
// the caller's stream, and reads the updated parameters and outputs back.
// Two copy streams (upload, read-back) and per-slot events let the upload of
// tensor i+1 and the read-back of tensor i-1 run while tensor i is stepped.
// Every copy is one cudaMemcpyAsync of one contiguous buffer.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include <cuda_runtime.h>

#include "focus.h"
#include "focus_trace.cuh"

namespace {

constexpr int HOST_SLOTS = 3;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Byte offsets of one slot's buffers for tensors of up to `n` weights.
struct SlotLayout {
    size_t desc, s2, amax, partial, W, dWq, Wq, m, q, mea, meas, qea, qeas, codes, scales, bytes;
};

SlotLayout slot_layout(int64_t n) {
    SlotLayout L;
    size_t o = 0;
    auto take = [&o](size_t b) {
        const size_t r = o;
        o += align256(b);
        return r;
    };
    const size_t w = static_cast<size_t>(n), nb = w / 16;
    L.desc = take(sizeof(focus_tensor_desc));
    L.s2 = take(16);
    L.amax = take(16);
    L.partial = take(focus_s2_workspace_bytes(1, n));   // the s2 pass's per-tile maxima (n % 16 == 0)
    L.W = take(2 * w);
    L.dWq = take(2 * w);
    L.Wq = take(2 * w);
    L.m = take(4 * nb);
    L.q = take(8 * nb);
    L.mea = take(4 * nb);
    L.meas = take(4 * nb);
    L.qea = take(8 * nb);
    L.qeas = take(8 * nb);
    L.codes = take(w / 2);
    L.scales = take(nb);
    L.bytes = o;
    return L;
}

// The library's shape rule (in % 16 == 0, sizes non-negative, block count in
// range): the s2 workspace query answers 0 exactly for shapes it rejects.
bool shape_ok(const focus_tensor_desc &h) { return focus_s2_workspace_bytes(h.out, h.in) != 0; }

int64_t max_weights(const focus_tensor_desc *h, int n) {
    int64_t mx = 0;
    for (int i = 0; i < n; ++i) mx = h[i].out * h[i].in > mx ? h[i].out * h[i].in : mx;
    return mx;
}

// Streams and events of one call, released on every exit path.
struct CallResources {
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t entry = nullptr;
    cudaEvent_t in_done[HOST_SLOTS] = {}, step_done[HOST_SLOTS] = {}, out_done[HOST_SLOTS] = {};
    bool ok = true;
    CallResources() {
        ok = cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&entry, cudaEventDisableTiming) == cudaSuccess;
        for (int s = 0; s < HOST_SLOTS && ok; ++s)
            ok = cudaEventCreateWithFlags(&in_done[s], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&step_done[s], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&out_done[s], cudaEventDisableTiming) == cudaSuccess;
    }
    ~CallResources() {
        if (up) cudaStreamSynchronize(up);
        if (down) cudaStreamSynchronize(down);
        for (int s = 0; s < HOST_SLOTS; ++s) {
            if (in_done[s]) cudaEventDestroy(in_done[s]);
            if (step_done[s]) cudaEventDestroy(step_done[s]);
            if (out_done[s]) cudaEventDestroy(out_done[s]);
        }
        if (entry) cudaEventDestroy(entry);
        if (up) cudaStreamDestroy(up);
        if (down) cudaStreamDestroy(down);
    }
};

}  // namespace

extern "C" {

size_t focus_step_host_workspace_bytes(const focus_tensor_desc *host_descs, int n_tensors) {
    if (!host_descs || n_tensors <= 0) return 0;
    for (int i = 0; i < n_tensors; ++i)
        if (!shape_ok(host_descs[i])) return 0;
    const int64_t mx = max_weights(host_descs, n_tensors);
    return mx > 0 ? HOST_SLOTS * slot_layout(mx).bytes : 0;
}

int focus_step_host(const focus_tensor_desc *h, int n, const focus_hparams *hp, int64_t step, unsigned flags,
                    void *ws_dev, size_t ws_bytes, focus_stream_t stream) {
    FOCUS_RANGE();
    if (n < 0) return FOCUS_ERR_VALUE;
    if (!hp) return FOCUS_ERR_NULL;
    if (flags & ~(unsigned)(FOCUS_STEP_PACK_UPDATED | FOCUS_STEP_WQ_UPDATED | FOCUS_HOST_S2_FIRST))
        return FOCUS_ERR_VALUE;
    if (n == 0) return FOCUS_OK;
    if (!h) return FOCUS_ERR_NULL;
    // host-side checks of every entry before anything is enqueued
    for (int i = 0; i < n; ++i) {
        const focus_tensor_desc &e = h[i];
        if (!shape_ok(e)) return FOCUS_ERR_SHAPE;
        if (e.out * e.in == 0) continue;
        if (!e.W || !e.dWq || !e.m || !e.q || !e.m_exp_avg || !e.m_exp_avg_sq || !e.q_exp_avg || !e.q_exp_avg_sq ||
            !e.s2)
            return FOCUS_ERR_NULL;
        if ((e.codes == nullptr) != (e.scales == nullptr)) return FOCUS_ERR_NULL;
        if (e.dm || e.dq) return FOCUS_ERR_VALUE;            // no gradient buffers on this path
        if (!(flags & FOCUS_HOST_S2_FIRST) && !(*e.s2 > 0.0f && std::isfinite(*e.s2))) return FOCUS_ERR_VALUE;
    }
    const size_t need = focus_step_host_workspace_bytes(h, n);
    if (need == 0) return FOCUS_OK;                           // every tensor is empty
    if (!ws_dev) return FOCUS_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(ws_dev) % 256 != 0) return FOCUS_ERR_ALIGN;
    if (ws_bytes < need) return FOCUS_ERR_WORKSPACE;

    const SlotLayout L = slot_layout(max_weights(h, n));
    unsigned char *ws = static_cast<unsigned char *>(ws_dev);
    const cudaStream_t comp = (cudaStream_t)stream;
    CallResources R;
    if (!R.ok) return FOCUS_ERR_CUDA;
    std::vector<focus_tensor_desc> dd(n);     // the device descriptors (host copies, uploaded per tensor)
    std::vector<int> slot_of(n, -1);
    const unsigned step_flags = flags & (FOCUS_STEP_PACK_UPDATED | FOCUS_STEP_WQ_UPDATED);
    int rc = FOCUS_OK;
    bool cuda_ok = cudaEventRecord(R.entry, comp) == cudaSuccess && cudaStreamWaitEvent(R.up, R.entry, 0) == cudaSuccess;
    for (int s = 0; s < HOST_SLOTS && cuda_ok; ++s)   // the maxima start at 0; s2_from_amax clears them after use
        cuda_ok = cudaMemsetAsync(ws + s * L.bytes + L.amax, 0, 16, R.up) == cudaSuccess;

    auto copy = [&cuda_ok](void *dst, const void *src, size_t bytes, cudaMemcpyKind kind, cudaStream_t s) {
        if (cuda_ok && bytes) cuda_ok = cudaMemcpyAsync(dst, src, bytes, kind, s) == cudaSuccess;
    };
    auto upload_and_step = [&](int i, int use) {
        const focus_tensor_desc &e = h[i];
        const int s = use % HOST_SLOTS;
        unsigned char *b = ws + s * L.bytes;
        const size_t w = static_cast<size_t>(e.out * e.in), nb = w / 16;
        focus_tensor_desc &d = dd[i];
        std::memset(&d, 0, sizeof d);
        d.W = reinterpret_cast<const uint16_t *>(b + L.W);
        d.dWq = reinterpret_cast<const uint16_t *>(b + L.dWq);
        d.Wq = e.Wq ? reinterpret_cast<uint16_t *>(b + L.Wq) : nullptr;
        d.m = reinterpret_cast<float *>(b + L.m);
        d.q = reinterpret_cast<float *>(b + L.q);
        d.m_exp_avg = reinterpret_cast<float *>(b + L.mea);
        d.m_exp_avg_sq = reinterpret_cast<float *>(b + L.meas);
        d.q_exp_avg = reinterpret_cast<float *>(b + L.qea);
        d.q_exp_avg_sq = reinterpret_cast<float *>(b + L.qeas);
        d.s2 = reinterpret_cast<float *>(b + L.s2);
        d.codes = e.codes ? b + L.codes : nullptr;
        d.scales = e.codes ? b + L.scales : nullptr;
        d.out = e.out;
        d.in = e.in;
        int64_t tiles = 0;
        if (rc == FOCUS_OK) rc = focus_table_prepare(&d, 1, 1, &tiles);
        slot_of[i] = s;
        if (rc != FOCUS_OK) return;
        // upload: after the slot's previous read-back
        if (use >= HOST_SLOTS && cuda_ok) cuda_ok = cudaStreamWaitEvent(R.up, R.out_done[s], 0) == cudaSuccess;
        copy(b + L.desc, &d, sizeof d, cudaMemcpyHostToDevice, R.up);
        copy(b + L.W, e.W, 2 * w, cudaMemcpyHostToDevice, R.up);
        copy(b + L.dWq, e.dWq, 2 * w, cudaMemcpyHostToDevice, R.up);
        copy(b + L.m, e.m, 4 * nb, cudaMemcpyHostToDevice, R.up);
        copy(b + L.q, e.q, 8 * nb, cudaMemcpyHostToDevice, R.up);
        copy(b + L.mea, e.m_exp_avg, 4 * nb, cudaMemcpyHostToDevice, R.up);
        copy(b + L.meas, e.m_exp_avg_sq, 4 * nb, cudaMemcpyHostToDevice, R.up);
        copy(b + L.qea, e.q_exp_avg, 8 * nb, cudaMemcpyHostToDevice, R.up);
        copy(b + L.qeas, e.q_exp_avg_sq, 8 * nb, cudaMemcpyHostToDevice, R.up);
        if (!(flags & FOCUS_HOST_S2_FIRST)) copy(b + L.s2, e.s2, sizeof(float), cudaMemcpyHostToDevice, R.up);
        if (cuda_ok) cuda_ok = cudaEventRecord(R.in_done[s], R.up) == cudaSuccess;
        // step on the caller's stream
        if (cuda_ok) cuda_ok = cudaStreamWaitEvent(comp, R.in_done[s], 0) == cudaSuccess;
        if (!cuda_ok) return;
        const focus_tensor_desc *dev_desc = reinterpret_cast<const focus_tensor_desc *>(b + L.desc);
        if (flags & FOCUS_HOST_S2_FIRST)
            rc = focus_s2_multi(dev_desc, 1, tiles, b + L.partial, focus_s2_multi_workspace_bytes(tiles), stream);
        if (rc == FOCUS_OK)
            rc = focus_step_fused_amax(dev_desc, 1, tiles, hp, step, step_flags,
                                       reinterpret_cast<uint32_t *>(b + L.amax), stream);
        if (rc == FOCUS_OK) rc = focus_s2_from_amax(dev_desc, 1, reinterpret_cast<uint32_t *>(b + L.amax), stream);
        if (rc == FOCUS_OK && cuda_ok) cuda_ok = cudaEventRecord(R.step_done[s], comp) == cudaSuccess;
    };
    auto read_back = [&](int i) {
        const focus_tensor_desc &e = h[i];
        const int s = slot_of[i];
        unsigned char *b = ws + s * L.bytes;
        const size_t w = static_cast<size_t>(e.out * e.in), nb = w / 16;
        if (cuda_ok) cuda_ok = cudaStreamWaitEvent(R.down, R.step_done[s], 0) == cudaSuccess;
        copy(e.m, b + L.m, 4 * nb, cudaMemcpyDeviceToHost, R.down);
        copy(e.q, b + L.q, 8 * nb, cudaMemcpyDeviceToHost, R.down);
        copy(e.m_exp_avg, b + L.mea, 4 * nb, cudaMemcpyDeviceToHost, R.down);
        copy(e.m_exp_avg_sq, b + L.meas, 4 * nb, cudaMemcpyDeviceToHost, R.down);
        copy(e.q_exp_avg, b + L.qea, 8 * nb, cudaMemcpyDeviceToHost, R.down);
        copy(e.q_exp_avg_sq, b + L.qeas, 8 * nb, cudaMemcpyDeviceToHost, R.down);
        copy(e.s2, b + L.s2, sizeof(float), cudaMemcpyDeviceToHost, R.down);
        if (e.Wq) copy(e.Wq, b + L.Wq, 2 * w, cudaMemcpyDeviceToHost, R.down);
        if (e.codes) {
            copy(e.codes, b + L.codes, w / 2, cudaMemcpyDeviceToHost, R.down);
            copy(e.scales, b + L.scales, nb, cudaMemcpyDeviceToHost, R.down);
        }
        if (cuda_ok) cuda_ok = cudaEventRecord(R.out_done[s], R.down) == cudaSuccess;
    };
    // Enqueue order: the upload and step of tensor i before the read-back of tensor
    // i-1, so that a blocking read-back (pageable host memory) does not hold back
    // the next upload.
    int use = 0, prev = -1;
    for (int i = 0; i < n && rc == FOCUS_OK && cuda_ok; ++i) {
        if (h[i].out * h[i].in == 0) continue;
        upload_and_step(i, use++);
        if (rc != FOCUS_OK || !cuda_ok) break;
        if (prev >= 0) read_back(prev);
        prev = i;
    }
    if (rc == FOCUS_OK && cuda_ok && prev >= 0) read_back(prev);
    // the call returns with every result in host memory
    if (cudaStreamSynchronize(R.up) != cudaSuccess) cuda_ok = false;
    if (cudaStreamSynchronize(comp) != cudaSuccess) cuda_ok = false;
    if (cudaStreamSynchronize(R.down) != cudaSuccess) cuda_ok = false;
    if (rc != FOCUS_OK) return rc;
    return cuda_ok ? FOCUS_OK : FOCUS_ERR_CUDA;
}

}  // extern "C"
