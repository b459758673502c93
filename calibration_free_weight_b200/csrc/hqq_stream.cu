// hqq_stream.cu -- hqq_quantize_stream: quantise a list of matrices held in
// host memory, streaming them through one GPU.
//
// The pages quantise a model layer by layer on the GPU and move data only
// once per layer (techreport.ngo, "Weight-only quantization without the
// calibration tax", section "Speed: from hours to minutes").  This executor
// is that loop for matrices that do not sit on the device: two device slots,
// each holding one matrix, its outputs and its workspace; the copy of matrix
// i+1 into one slot (copy-in stream) overlaps the solver on matrix i in the
// other (the caller's stream) and the copy of matrix i-1's outputs back to the
// host (copy-out stream).  Events order the reuse of a slot: matrix i+2 is
// copied in only after the solver on matrix i has finished reading it, and its
// outputs are written only after those of matrix i have been copied out.
//
// The call blocks until every output has reached host memory.  Host buffers
// should be pinned (cudaHostAlloc / cudaHostRegister) for the copies to
// overlap; pageable buffers work but serialise.  Device memory is the
// caller's buffer; the executor creates two streams and six events per call
// and destroys them before returning.

#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/hqq.h"
#include "hqq_internal.h"

namespace {

constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Largest per-matrix sizes of the list (bytes).
struct SlotSizes {
    size_t W = 0, packed = 0, scale = 0, zero = 0, workspace = 0;
    size_t total() const { return up(W) + up(packed) + up(scale) + up(zero) + up(8) + up(workspace); }
};

int slot_sizes(const hqq_host_matrix* mats, int n, int nbits, int group_size, int axis, int stop_mode,
               int zero_nbits, SlotSizes* out) {
    SlotSizes s;
    for (int i = 0; i < n; ++i) {
        const int64_t rows = mats[i].rows, cols = mats[i].cols;
        const int64_t G = hqq_num_groups(rows, cols, group_size, axis);
        if (G < 0) return HQQ_ERR_SHAPE;
        const size_t ws = hqq_workspace_bytes(rows, cols, group_size, axis, stop_mode, zero_nbits);
        if (ws == 0) return HQQ_ERR_INVALID_ARG;
        s.W = std::max(s.W, static_cast<size_t>(rows * cols) * 2);
        s.packed = std::max(s.packed, hqq_packed_bytes(rows, cols, nbits, group_size, axis));
        s.scale = std::max(s.scale, static_cast<size_t>(G) * 2);
        s.zero = std::max(s.zero, static_cast<size_t>(G) * (zero_nbits == 16 ? 2 : 1));
        s.workspace = std::max(s.workspace, ws);
    }
    *out = s;
    return HQQ_OK;
}

struct Slot {
    uint8_t *W, *packed, *scale, *zero, *meta, *ws;
};

Slot carve(uint8_t* base, const SlotSizes& s) {
    Slot t;
    size_t off = 0;
    t.W = base + off;
    off += up(s.W);
    t.packed = base + off;
    off += up(s.packed);
    t.scale = base + off;
    off += up(s.scale);
    t.zero = base + off;
    off += up(s.zero);
    t.meta = base + off;
    off += up(8);
    t.ws = base + off;
    return t;
}

// Streams and events of one call, released on every exit path.
struct Resources {
    cudaStream_t cin = nullptr, cout = nullptr;
    cudaEvent_t in_done[2] = {}, solved[2] = {}, out_done[2] = {};
    bool ok = true;
    Resources() {
        ok = cudaStreamCreateWithFlags(&cin, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&cout, cudaStreamNonBlocking) == cudaSuccess;
        for (int k = 0; k < 2 && ok; ++k)
            ok = cudaEventCreateWithFlags(&in_done[k], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&solved[k], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&out_done[k], cudaEventDisableTiming) == cudaSuccess;
    }
    ~Resources() {
        if (cin) cudaStreamSynchronize(cin);
        if (cout) cudaStreamSynchronize(cout);
        for (int k = 0; k < 2; ++k) {
            if (in_done[k]) cudaEventDestroy(in_done[k]);
            if (solved[k]) cudaEventDestroy(solved[k]);
            if (out_done[k]) cudaEventDestroy(out_done[k]);
        }
        if (cin) cudaStreamDestroy(cin);
        if (cout) cudaStreamDestroy(cout);
    }
};

}  // namespace

extern "C" {

size_t hqq_stream_device_bytes(const hqq_host_matrix* mats, int n, int nbits, int group_size, int axis,
                               int stop_mode, int zero_nbits) {
    if (mats == nullptr || n < 1) return 0;
    SlotSizes s;
    if (slot_sizes(mats, n, nbits, group_size, axis, stop_mode, zero_nbits, &s) != HQQ_OK) return 0;
    return 2 * s.total();
}

int hqq_quantize_stream(const hqq_host_matrix* mats, int n, int dtype, int nbits, int group_size, int axis, float p,
                        float beta, float kappa, int iters, int stop_mode, int zero_nbits, void* device_buffer,
                        size_t device_bytes, void* stream) {
    if (mats == nullptr || n < 0) return HQQ_ERR_INVALID_ARG;
    if (n == 0) return HQQ_OK;
    SlotSizes s;
    const int rc0 = slot_sizes(mats, n, nbits, group_size, axis, stop_mode, zero_nbits, &s);
    if (rc0 != HQQ_OK) return rc0;
    for (int i = 0; i < n; ++i) {
        const hqq_host_matrix& m = mats[i];
        if (m.rows * m.cols == 0) continue;
        if (!m.W || !m.W_q_packed || !m.scale || !m.zero || (zero_nbits == 8 && !m.zero_meta))
            return HQQ_ERR_INVALID_ARG;
    }
    if (device_buffer == nullptr || device_bytes < 2 * s.total()) return HQQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(device_buffer) & (kAlign - 1)) != 0) return HQQ_ERR_ALIGN;

    Resources r;
    if (!r.ok) {
        cudaGetLastError();
        return HQQ_ERR_CUDA;
    }
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    Slot slot[2] = {carve(static_cast<uint8_t*>(device_buffer), s),
                    carve(static_cast<uint8_t*>(device_buffer) + s.total(), s)};
    int rc = HQQ_OK;
    auto cuda_ok = [&](cudaError_t e) {
        if (e != cudaSuccess && rc == HQQ_OK) rc = HQQ_ERR_CUDA;
        return e == cudaSuccess;
    };
    for (int i = 0; i < n && rc == HQQ_OK; ++i) {
        const hqq_host_matrix& m = mats[i];
        const Slot& t = slot[i & 1];
        const int64_t G = m.rows * m.cols / group_size;
        const size_t wb = static_cast<size_t>(m.rows * m.cols) * 2;
        const size_t pb = hqq_packed_bytes(m.rows, m.cols, nbits, group_size, axis);
        const size_t sb = static_cast<size_t>(G) * 2, zb = static_cast<size_t>(G) * (zero_nbits == 16 ? 2 : 1);
        // copy-in: the solver on matrix i-2 (same slot) must have finished reading W
        if (i >= 2 && !cuda_ok(cudaStreamWaitEvent(r.cin, r.solved[i & 1], 0))) break;
        if (wb && !cuda_ok(cudaMemcpyAsync(t.W, m.W, wb, cudaMemcpyHostToDevice, r.cin))) break;
        if (!cuda_ok(cudaEventRecord(r.in_done[i & 1], r.cin))) break;
        // solve: W has arrived, and matrix i-2's outputs in this slot have been copied out
        if (!cuda_ok(cudaStreamWaitEvent(cs, r.in_done[i & 1], 0))) break;
        if (i >= 2 && !cuda_ok(cudaStreamWaitEvent(cs, r.out_done[i & 1], 0))) break;
        const size_t wsb = hqq_workspace_bytes(m.rows, m.cols, group_size, axis, stop_mode, zero_nbits);
        const int q = hqq::quantize_entry(t.W, m.rows, m.cols, dtype, nbits, group_size, axis, p, beta, kappa, iters,
                                          stop_mode, zero_nbits, t.packed, t.scale, t.zero,
                                          zero_nbits == 8 ? t.meta : nullptr, t.ws, wsb, false, nullptr, nullptr,
                                          nullptr, cs);
        if (q != HQQ_OK) {
            rc = q;
            break;
        }
        if (!cuda_ok(cudaEventRecord(r.solved[i & 1], cs))) break;
        // copy-out
        if (!cuda_ok(cudaStreamWaitEvent(r.cout, r.solved[i & 1], 0))) break;
        if (pb && !cuda_ok(cudaMemcpyAsync(m.W_q_packed, t.packed, pb, cudaMemcpyDeviceToHost, r.cout))) break;
        if (sb && !cuda_ok(cudaMemcpyAsync(m.scale, t.scale, sb, cudaMemcpyDeviceToHost, r.cout))) break;
        if (zb && !cuda_ok(cudaMemcpyAsync(m.zero, t.zero, zb, cudaMemcpyDeviceToHost, r.cout))) break;
        if (zero_nbits == 8 && !cuda_ok(cudaMemcpyAsync(m.zero_meta, t.meta, 8, cudaMemcpyDeviceToHost, r.cout)))
            break;
        if (!cuda_ok(cudaEventRecord(r.out_done[i & 1], r.cout))) break;
    }
    // every output on the host (or the first error) before returning
    const cudaError_t e1 = cudaStreamSynchronize(cs);
    const cudaError_t e2 = cudaStreamSynchronize(r.cout);
    const cudaError_t e3 = cudaStreamSynchronize(r.cin);
    if ((e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess) && rc == HQQ_OK) rc = HQQ_ERR_CUDA;
    if (rc != HQQ_OK) cudaGetLastError();
    return rc;
}

}  // extern "C"
