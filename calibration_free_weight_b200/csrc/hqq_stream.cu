// hqq_stream.cu -- hqq_quantize_stream / hqq_quantize_stream_jobs: quantise
// a list of matrices held in host memory, streaming them through one GPU,
// with settings per matrix (attention and MLP layers at different bit widths,
// "HQQ - Half-Quadratic Quantization" (skill4agent.com), section "Mixed
// precision quantization").
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
// A job whose matrix is the previous job's (the same host buffer and shape,
// e.g. one weight quantised at two settings) reuses the device copy of it:
// the weights cross PCIe once.  The W buffers alternate between the two slots
// on copies only, and a copy into one waits for every solver that read it.
//
// Each job is reported (callback, in order) once its outputs are in host
// memory; the report of job i-2 is taken just before its slot's copy-out event
// is reused for job i, by which time the solver on job i has already waited
// for that copy on the GPU, so reporting costs no overlap.
//
// The call blocks until every output has reached host memory.  Host buffers
// should be pinned (cudaHostAlloc / cudaHostRegister) for the copies to
// overlap; pageable buffers work but serialise.  Device memory is the
// caller's buffer; the executor creates two streams and eight events per call
// and destroys them before returning.

#include <cuda_runtime.h>

#include <algorithm>
#include <vector>

#include "../../include/hqq.h"
#include "hqq_internal.h"

namespace {

constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Buffer sizes of one job (bytes).
struct JobSizes {
    size_t W = 0, packed = 0, scale = 0, zero = 0, workspace = 0;
};

JobSizes job_sizes(const hqq_stream_job& j) {
    const int64_t rows = j.m.rows, cols = j.m.cols;
    const int64_t G = hqq_num_groups(rows, cols, j.group_size, j.axis);
    JobSizes s;
    s.W = static_cast<size_t>(rows * cols) * 2;
    s.packed = hqq_packed_bytes(rows, cols, j.nbits, j.group_size, j.axis);
    s.scale = static_cast<size_t>(G) * 2;
    s.zero = static_cast<size_t>(G) * (j.zero_nbits == 16 ? 2 : 1);
    s.workspace = hqq_workspace_bytes(rows, cols, j.group_size, j.axis, j.stop_mode, j.zero_nbits);
    return s;
}

// One slot: each buffer kind sized for the largest job of the list.
struct SlotSizes {
    JobSizes m;
    size_t total() const { return up(m.W) + up(m.packed) + up(m.scale) + up(m.zero) + up(8) + up(m.workspace); }
};

// Settings and shape of every job (the solver parameters of the call
// included), before anything is copied or launched.
int check_jobs(const hqq_stream_job* jobs, int n, int dtype, float p, float beta, float kappa, int iters,
               SlotSizes* out) {
    SlotSizes s;
    for (int i = 0; i < n; ++i) {
        const hqq_stream_job& j = jobs[i];
        const int ck = hqq::check_args(j.m.rows, j.m.cols, dtype, j.nbits, j.group_size, j.axis, p, beta, kappa, iters,
                                       j.stop_mode, j.zero_nbits);
        if (ck != HQQ_OK) return ck;
        const JobSizes z = job_sizes(j);
        s.m.W = std::max(s.m.W, z.W);
        s.m.packed = std::max(s.m.packed, z.packed);
        s.m.scale = std::max(s.m.scale, z.scale);
        s.m.zero = std::max(s.m.zero, z.zero);
        s.m.workspace = std::max(s.m.workspace, z.workspace);
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
    off += up(s.m.W);
    t.packed = base + off;
    off += up(s.m.packed);
    t.scale = base + off;
    off += up(s.m.scale);
    t.zero = base + off;
    off += up(s.m.zero);
    t.meta = base + off;
    off += up(8);
    t.ws = base + off;
    return t;
}

// Streams and events of one call, released on every exit path.
struct Resources {
    cudaStream_t cin = nullptr, cout = nullptr;
    // in_done / w_read: per W buffer (copied in; last read by a solver),
    // solved / out_done: per output slot (solved; copied out)
    cudaEvent_t in_done[2] = {}, w_read[2] = {}, solved[2] = {}, out_done[2] = {};
    bool ok = true;
    Resources() {
        ok = cudaStreamCreateWithFlags(&cin, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&cout, cudaStreamNonBlocking) == cudaSuccess;
        for (int k = 0; k < 2 && ok; ++k)
            ok = cudaEventCreateWithFlags(&in_done[k], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&w_read[k], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&solved[k], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&out_done[k], cudaEventDisableTiming) == cudaSuccess;
    }
    ~Resources() {
        if (cin) cudaStreamSynchronize(cin);
        if (cout) cudaStreamSynchronize(cout);
        for (int k = 0; k < 2; ++k) {
            if (in_done[k]) cudaEventDestroy(in_done[k]);
            if (w_read[k]) cudaEventDestroy(w_read[k]);
            if (solved[k]) cudaEventDestroy(solved[k]);
            if (out_done[k]) cudaEventDestroy(out_done[k]);
        }
        if (cin) cudaStreamDestroy(cin);
        if (cout) cudaStreamDestroy(cout);
    }
};

std::vector<hqq_stream_job> uniform_jobs(const hqq_host_matrix* mats, int n, int nbits, int group_size, int axis,
                                         int stop_mode, int zero_nbits) {
    std::vector<hqq_stream_job> jobs(static_cast<size_t>(n));
    for (int i = 0; i < n; ++i) jobs[i] = hqq_stream_job{mats[i], nbits, group_size, axis, stop_mode, zero_nbits};
    return jobs;
}

}  // namespace

extern "C" {

size_t hqq_stream_jobs_device_bytes(const hqq_stream_job* jobs, int n) {
    if (jobs == nullptr || n < 1) return 0;
    SlotSizes s;
    // solver parameters that every check accepts: only the jobs' own settings decide
    if (check_jobs(jobs, n, HQQ_F16, 0.7f, 1.0f, 1.0f, 0, &s) != HQQ_OK) return 0;
    return 2 * s.total();
}

size_t hqq_stream_device_bytes(const hqq_host_matrix* mats, int n, int nbits, int group_size, int axis,
                               int stop_mode, int zero_nbits) {
    if (mats == nullptr || n < 1) return 0;
    const std::vector<hqq_stream_job> jobs = uniform_jobs(mats, n, nbits, group_size, axis, stop_mode, zero_nbits);
    return hqq_stream_jobs_device_bytes(jobs.data(), n);
}

int hqq_quantize_stream_jobs(const hqq_stream_job* jobs, int n, int dtype, float p, float beta, float kappa, int iters,
                             void* device_buffer, size_t device_bytes, hqq_stream_done_fn on_done, void* user,
                             int* jobs_done, void* stream) {
    if (jobs_done) *jobs_done = 0;
    if (jobs == nullptr || n < 0) return HQQ_ERR_INVALID_ARG;
    if (n == 0) return HQQ_OK;
    SlotSizes s;
    const int rc0 = check_jobs(jobs, n, dtype, p, beta, kappa, iters, &s);
    if (rc0 != HQQ_OK) return rc0;
    for (int i = 0; i < n; ++i) {
        const hqq_stream_job& j = jobs[i];
        if (j.m.rows * j.m.cols == 0) continue;
        if (!j.m.W || !j.m.W_q_packed || !j.m.scale || !j.m.zero || (j.zero_nbits == 8 && !j.m.zero_meta))
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
    int reported = 0;  // jobs 0 .. reported-1 have been reported done
    auto cuda_ok = [&](cudaError_t e) {
        if (e != cudaSuccess && rc == HQQ_OK) rc = HQQ_ERR_CUDA;
        return e == cudaSuccess;
    };
    // job k is done once its copy-out event (slot k & 1, not yet reused) has completed
    auto report = [&](int k) {
        if (!cuda_ok(cudaEventSynchronize(r.out_done[k & 1]))) return false;
        if (on_done) on_done(k, user);
        reported = k + 1;
        return true;
    };
    int copies = 0, wb = 0;  // W buffers filled so far; the one holding the current job's matrix
    for (int i = 0; i < n && rc == HQQ_OK; ++i) {
        const hqq_stream_job& j = jobs[i];
        const hqq_host_matrix& m = j.m;
        const Slot& t = slot[i & 1];
        const JobSizes z = job_sizes(j);
        const bool reuse = i >= 1 && z.W && m.W == jobs[i - 1].m.W && m.rows == jobs[i - 1].m.rows &&
                           m.cols == jobs[i - 1].m.cols;
        if (!reuse) {
            // copy-in: every solver that read this W buffer must be done with it
            wb = copies & 1;
            ++copies;
            if (copies > 2 && !cuda_ok(cudaStreamWaitEvent(r.cin, r.w_read[wb], 0))) break;
            if (z.W && !cuda_ok(cudaMemcpyAsync(slot[wb].W, m.W, z.W, cudaMemcpyHostToDevice, r.cin))) break;
            if (!cuda_ok(cudaEventRecord(r.in_done[wb], r.cin))) break;
        }
        // solve: W has arrived, and job i-2's outputs in this slot have been copied out
        if (!cuda_ok(cudaStreamWaitEvent(cs, r.in_done[wb], 0))) break;
        if (i >= 2 && !cuda_ok(cudaStreamWaitEvent(cs, r.out_done[i & 1], 0))) break;
        const int q = hqq::quantize_entry(slot[wb].W, m.rows, m.cols, dtype, j.nbits, j.group_size, j.axis, p, beta,
                                          kappa, iters, j.stop_mode, j.zero_nbits, t.packed, t.scale, t.zero,
                                          j.zero_nbits == 8 ? t.meta : nullptr, t.ws, z.workspace, false, nullptr,
                                          nullptr, nullptr, cs);
        if (q != HQQ_OK) {
            rc = q;
            break;
        }
        if (!cuda_ok(cudaEventRecord(r.w_read[wb], cs))) break;
        if (!cuda_ok(cudaEventRecord(r.solved[i & 1], cs))) break;
        // job i-2's copy-out event is about to be reused: report it first
        if (i >= 2 && !report(i - 2)) break;
        // copy-out
        if (!cuda_ok(cudaStreamWaitEvent(r.cout, r.solved[i & 1], 0))) break;
        if (z.packed && !cuda_ok(cudaMemcpyAsync(m.W_q_packed, t.packed, z.packed, cudaMemcpyDeviceToHost, r.cout)))
            break;
        if (z.scale && !cuda_ok(cudaMemcpyAsync(m.scale, t.scale, z.scale, cudaMemcpyDeviceToHost, r.cout))) break;
        if (z.zero && !cuda_ok(cudaMemcpyAsync(m.zero, t.zero, z.zero, cudaMemcpyDeviceToHost, r.cout))) break;
        if (j.zero_nbits == 8 && !cuda_ok(cudaMemcpyAsync(m.zero_meta, t.meta, 8, cudaMemcpyDeviceToHost, r.cout)))
            break;
        if (!cuda_ok(cudaEventRecord(r.out_done[i & 1], r.cout))) break;
    }
    // every output on the host (or the first error) before returning
    const cudaError_t e1 = cudaStreamSynchronize(cs);
    const cudaError_t e2 = cudaStreamSynchronize(r.cout);
    const cudaError_t e3 = cudaStreamSynchronize(r.cin);
    if ((e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess) && rc == HQQ_OK) rc = HQQ_ERR_CUDA;
    if (rc == HQQ_OK)
        for (int k = reported; k < n; ++k)
            if (!report(k)) break;
    if (rc != HQQ_OK) cudaGetLastError();
    if (jobs_done) *jobs_done = rc == HQQ_OK ? n : reported;
    return rc;
}

int hqq_quantize_stream(const hqq_host_matrix* mats, int n, int dtype, int nbits, int group_size, int axis, float p,
                        float beta, float kappa, int iters, int stop_mode, int zero_nbits, void* device_buffer,
                        size_t device_bytes, void* stream) {
    if (mats == nullptr || n < 0) return HQQ_ERR_INVALID_ARG;
    if (n == 0) return HQQ_OK;
    const std::vector<hqq_stream_job> jobs = uniform_jobs(mats, n, nbits, group_size, axis, stop_mode, zero_nbits);
    return hqq_quantize_stream_jobs(jobs.data(), n, dtype, p, beta, kappa, iters, device_buffer, device_bytes, nullptr,
                                    nullptr, nullptr, stream);
}

}  // extern "C"
