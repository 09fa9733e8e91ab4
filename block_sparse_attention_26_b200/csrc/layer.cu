// layer.cu -- one layer from host memory, with the host<->device copies of one
// chunk of heads overlapping the kernels of another (bsa_layer_host).  Host
// code only.
//
// Attention is independent per (batch, head): "minimax-h3-chunk-star7" README,
// "Sol" and "SLA" (block means, routing and the fine pass are all per head).
// So the heads of a layer can be taken in chunks, each chunk a smaller layer
// whose Q, K, V and O are strided views of the whole layer's arrays; the
// chunk's inputs are copied in and its output copied back while the GPU works
// on the neighbouring chunks.
#include <stdio.h>

#include "bsa_internal.h"

using namespace bsa;

namespace {

// Copies heads [h0, h1) of a [B, N, H, d] array between host and device (same
// strides on both sides): for each batch, N rows of (h1 - h0) * d elements.
cudaError_t copy_heads(void *dst, const void *src, const bsa_params &p, int h0, int h1, cudaMemcpyKind kind,
                       cudaStream_t st)
{
    const size_t es = p.dtype == BSA_DT_F32 ? 4 : 2;
    const size_t width = (size_t)(h1 - h0) * p.d * es;
    const size_t pitch = (size_t)p.stride_n * es;
    const size_t off = (size_t)h0 * p.stride_h * es;
    const bool rows_join = p.stride_b == (int64_t)p.N * p.stride_n;   // batches follow each other row-wise
    const int nb = rows_join ? 1 : p.B;
    const size_t height = rows_join ? (size_t)p.B * p.N : (size_t)p.N;
    for (int b = 0; b < nb; ++b) {
        const size_t bo = off + (size_t)b * p.stride_b * es;
        const cudaError_t e = cudaMemcpy2DAsync(static_cast<char *>(dst) + bo, pitch, static_cast<const char *>(src) + bo,
                                                pitch, width, height, kind, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

struct Events {
    cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
    ~Events()
    {
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);   // deferred by the runtime until the event completes
    }
};

}  // namespace

extern "C" {

bsa_status bsa_layer_host(const bsa_params *p, const void *q_host, const void *k_host, const void *v_host,
                          void *out_host, const bsa_layer_device *dev, int32_t heads_per_chunk, void *stream,
                          void *copy_in, void *copy_out)
{
    set_error("%s", "");
    if (p == nullptr || dev == nullptr) {
        set_error("params / device buffers are NULL");
        return BSA_ERR_INVALID_ARG;
    }
    if (q_host == nullptr || k_host == nullptr || v_host == nullptr || out_host == nullptr) {
        set_error("a host array is NULL");
        return BSA_ERR_INVALID_ARG;
    }
    if (p->H < 1 || p->stride_h != p->d) {
        set_error("bsa_layer_host needs the heads of a row side by side (stride_h == d)");
        return BSA_ERR_INVALID_ARG;
    }
    if (heads_per_chunk < 0) {
        set_error("heads_per_chunk < 0");
        return BSA_ERR_INVALID_ARG;
    }
    // default: about 16 chunks (long: 138 ms a layer at 2 heads a chunk, 163 ms at 10,
    // against 116 ms for the inputs' copy alone)
    const int hc = heads_per_chunk > 0 ? std::min<int>(heads_per_chunk, p->H) : std::max(1, (p->H + 15) / 16);
    const cudaStream_t st = (cudaStream_t)stream;
    const cudaStream_t sin = copy_in ? (cudaStream_t)copy_in : st;
    const cudaStream_t sout = copy_out ? (cudaStream_t)copy_out : st;
    const size_t es = p->dtype == BSA_DT_F32 ? 4 : 2;
    const bool E = p->extra_tokens > 0;
    // events: chunk inputs in, chunk output computed, last copy back done (reused
    // per chunk: each wait is enqueued before the event is recorded again)
    Events ev;
    for (auto &e : ev.ev)
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
            set_error("bsa_layer_host: cudaEventCreateWithFlags failed");
            return BSA_ERR_CUDA;
        }
    // Within a call the copies touch only q, k, v and out, which the chunks share
    // head-disjointly; the chunk buffers (means, CSR, workspace) are reused in
    // stream order on `stream`.  Across calls: this call's first copy in must not
    // overwrite q, k, v under work already enqueued on `stream`, so copy_in waits
    // for it; the previous call's copies back are already ahead of `stream`.
    if (sin != st) {
        cudaError_t e = cudaEventRecord(ev.ev[2], st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sin, ev.ev[2], 0);
        if (e != cudaSuccess) {
            set_error("bsa_layer_host: %s", cudaGetErrorString(e));
            return BSA_ERR_CUDA;
        }
    }
    for (int h0 = 0; h0 < p->H; h0 += hc) {
        const int h1 = std::min(p->H, h0 + hc);
        bsa_params c = *p;
        c.H = h1 - h0;
        const size_t off = (size_t)h0 * p->stride_h * es;
        auto at = [&](void *base) { return static_cast<void *>(static_cast<char *>(base) + off); };
        const void *qd = at(dev->q), *kd = at(dev->k), *vd = at(dev->v);
        void *od = at(dev->out);
        cudaError_t e = copy_heads(dev->q, q_host, *p, h0, h1, cudaMemcpyHostToDevice, sin);
        if (e == cudaSuccess) e = copy_heads(dev->k, k_host, *p, h0, h1, cudaMemcpyHostToDevice, sin);
        if (e == cudaSuccess) e = copy_heads(dev->v, v_host, *p, h0, h1, cudaMemcpyHostToDevice, sin);
        if (e == cudaSuccess && sin != st) {
            e = cudaEventRecord(ev.ev[0], sin);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev.ev[0], 0);
        }
        if (e != cudaSuccess) {
            set_error("bsa_layer_host: copy in: %s", cudaGetErrorString(e));
            return BSA_ERR_CUDA;
        }
        bsa_status s = bsa_pool(&c, qd, kd, vd, dev->qbar, dev->kbar, dev->vbar, dev->blk_count, stream);
        if (s == BSA_OK)
            s = bsa_select(&c, dev->qbar, dev->kbar, kd, dev->row_ptr, dev->col_idx, dev->col_capacity,
                           dev->kept_count, E ? dev->extra_idx : nullptr, E ? dev->extra_count : nullptr, dev->ws,
                           dev->ws_bytes, stream);
        if (s == BSA_OK)
            s = bsa_attention(&c, qd, kd, vd, dev->kbar, dev->vbar, dev->blk_count, dev->row_ptr, dev->col_idx,
                              E ? dev->extra_idx : nullptr, E ? dev->extra_count : nullptr, od, nullptr, dev->ws,
                              dev->ws_bytes, stream);
        if (s != BSA_OK) return s;
        if (sout != st) {
            e = cudaEventRecord(ev.ev[1], st);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(sout, ev.ev[1], 0);
        }
        if (e == cudaSuccess) e = copy_heads(out_host, dev->out, *p, h0, h1, cudaMemcpyDeviceToHost, sout);
        if (e != cudaSuccess) {
            set_error("bsa_layer_host: copy out: %s", cudaGetErrorString(e));
            return BSA_ERR_CUDA;
        }
    }
    if (sout != st) {
        cudaError_t e = cudaEventRecord(ev.ev[2], sout);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev.ev[2], 0);
        if (e != cudaSuccess) {
            set_error("bsa_layer_host: %s", cudaGetErrorString(e));
            return BSA_ERR_CUDA;
        }
    }
    return BSA_OK;
}

}  // extern "C"
