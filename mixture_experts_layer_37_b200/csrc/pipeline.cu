// moe_pipeline: layer forwards on host-resident batches, with the copy in of
// one batch, the forward of the previous one and the copy out of the one
// before that running at the same time on three streams.
//
// Step i uses slot s = i % depth (its own device x, out and l_aux buffers).
//   copy-in stream   waits until forward i-depth has read x[s], copies x_host;
//   compute stream   waits for that copy and for copy-out i-depth (out[s] is
//                    free), runs the five-launch forward into out[s];
//   copy-out stream  waits for the forward, copies out[s] and l_aux[s] back.
// The workspace and the routing outputs are shared by all steps: forwards are
// serialised on the compute stream.  Buffers from cudaMalloc, freed by destroy.
#include <string.h>

#include <new>

#include "internal.h"
#include "moe.h"

struct moe_pipeline {
    moe_config_t cfg;
    moe_weights_t weights;
    int depth = 0;
    int dev = 0;
    size_t x_bytes = 0;
    cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
    void* ws = nullptr;
    size_t ws_bytes = 0;
    moe_outputs_t outs[MOE_PIPELINE_MAX_DEPTH];
    void* x_dev[MOE_PIPELINE_MAX_DEPTH] = {};
    cudaEvent_t in_done[MOE_PIPELINE_MAX_DEPTH] = {};
    cudaEvent_t comp_done[MOE_PIPELINE_MAX_DEPTH] = {};
    cudaEvent_t out_done[MOE_PIPELINE_MAX_DEPTH] = {};
    void* shared = nullptr;  // routing outputs, one allocation
    void* slots = nullptr;   // per-slot x, out, l_aux, one allocation
    int64_t submitted = 0;
};

namespace {

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

void release(moe_pipeline* p) {
    if (p == nullptr) return;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(p->dev);
    for (cudaStream_t s : {p->s_in, p->s_comp, p->s_out})
        if (s) cudaStreamSynchronize(s);
    for (int i = 0; i < MOE_PIPELINE_MAX_DEPTH; ++i) {
        if (p->in_done[i]) cudaEventDestroy(p->in_done[i]);
        if (p->comp_done[i]) cudaEventDestroy(p->comp_done[i]);
        if (p->out_done[i]) cudaEventDestroy(p->out_done[i]);
    }
    for (cudaStream_t s : {p->s_in, p->s_comp, p->s_out})
        if (s) cudaStreamDestroy(s);
    if (p->ws) cudaFree(p->ws);
    if (p->shared) cudaFree(p->shared);
    if (p->slots) cudaFree(p->slots);
    cudaSetDevice(prev);
    delete p;
}

}  // namespace

extern "C" {

moe_status_t moe_pipeline_create(const moe_config_t* cfg, const moe_weights_t* weights, int32_t depth,
                                 moe_pipeline_t** pipe) {
    if (pipe == nullptr) return MOE_ERR_INVALID_ARG;
    *pipe = nullptr;
    if (cfg == nullptr || weights == nullptr || depth < 1 || depth > MOE_PIPELINE_MAX_DEPTH)
        return MOE_ERR_INVALID_ARG;
    size_t ws_bytes = 0;
    moe_status_t st = moe_workspace_size(cfg, &ws_bytes);
    if (st != MOE_OK) return st;
    int64_t rows = 0;
    if ((st = moe_max_rows(cfg, &rows)) != MOE_OK) return st;
    if (weights->w_router == nullptr || (cfg->T > 0 && (weights->w_gate_or_w1 == nullptr ||
                                                        weights->w_down_or_w2 == nullptr)))
        return MOE_ERR_INVALID_ARG;

    moe_pipeline* p = new (std::nothrow) moe_pipeline();
    if (p == nullptr) return MOE_ERR_CUDA;
    p->cfg = *cfg;
    p->weights = *weights;
    p->depth = depth;
    p->ws_bytes = ws_bytes;
    cudaGetDevice(&p->dev);
    const int64_t T = cfg->T, E = cfg->E, k = cfg->k;
    const size_t es = cfg->dtype == MOE_DT_BF16 ? 2 : 4;
    p->x_bytes = (size_t)T * cfg->d * es;

    // shared routing outputs
    const size_t n_idx = up256((size_t)T * k * 4), n_w = n_idx, n_cnt = up256(E * 4), n_off = up256((E + 1) * 4);
    const size_t n_slot = n_idx, n_src = up256((size_t)(rows > 0 ? rows : 1) * 4), n_fp = up256(E * 4);
    const size_t shared_bytes = n_idx + n_w + n_cnt + n_off + n_slot + n_src + 2 * n_fp;
    const size_t slot_bytes = 2 * up256(p->x_bytes > 0 ? p->x_bytes : 16) + 256;

    bool ok = cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p->s_comp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaMalloc(&p->ws, ws_bytes) == cudaSuccess && cudaMalloc(&p->shared, shared_bytes) == cudaSuccess &&
              cudaMalloc(&p->slots, slot_bytes * depth) == cudaSuccess;
    for (int i = 0; ok && i < depth; ++i)
        ok = cudaEventCreateWithFlags(&p->in_done[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&p->comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&p->out_done[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        release(p);
        return MOE_ERR_CUDA;
    }
    uint8_t* sh = static_cast<uint8_t*>(p->shared);
    moe_outputs_t base;
    memset(&base, 0, sizeof(base));
    base.topk_idx = reinterpret_cast<int32_t*>(sh);
    sh += n_idx;
    base.topk_w = reinterpret_cast<float*>(sh);
    sh += n_w;
    base.counts = reinterpret_cast<int32_t*>(sh);
    sh += n_cnt;
    base.offsets = reinterpret_cast<int32_t*>(sh);
    sh += n_off;
    base.slot = reinterpret_cast<int32_t*>(sh);
    sh += n_slot;
    base.src_assign = reinterpret_cast<int32_t*>(sh);
    sh += n_src;
    base.f = reinterpret_cast<float*>(sh);
    sh += n_fp;
    base.p = reinterpret_cast<float*>(sh);
    for (int i = 0; i < depth; ++i) {
        uint8_t* b = static_cast<uint8_t*>(p->slots) + slot_bytes * i;
        const size_t xb = up256(p->x_bytes > 0 ? p->x_bytes : 16);
        p->x_dev[i] = b;
        p->outs[i] = base;
        p->outs[i].out = b + xb;
        p->outs[i].l_aux = reinterpret_cast<float*>(b + 2 * xb);
    }
    if ((st = moe_workspace_init(p->ws, ws_bytes, p->s_comp)) != MOE_OK ||
        cudaStreamSynchronize(p->s_comp) != cudaSuccess) {
        release(p);
        return st != MOE_OK ? st : MOE_ERR_CUDA;
    }
    *pipe = p;
    return MOE_OK;
}

moe_status_t moe_pipeline_submit(moe_pipeline_t* p, const void* x_host, void* out_host, float* l_aux_host,
                                 cudaEvent_t start_event, cudaEvent_t end_event, int64_t* ticket) {
    if (p == nullptr || l_aux_host == nullptr) return MOE_ERR_INVALID_ARG;
    if (p->x_bytes > 0 && (x_host == nullptr || out_host == nullptr)) return MOE_ERR_INVALID_ARG;
    const int s = (int)(p->submitted % p->depth);
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != p->dev && cudaSetDevice(p->dev) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status_t st = MOE_OK;
    auto cuda_ok = [&](cudaError_t e) {
        if (e != cudaSuccess && st == MOE_OK) st = MOE_ERR_CUDA;
        return e == cudaSuccess;
    };
    // copy in, once forward i-depth no longer reads x[s]
    if (start_event) cuda_ok(cudaEventRecord(start_event, p->s_in));
    cuda_ok(cudaStreamWaitEvent(p->s_in, p->comp_done[s], 0));
    if (p->x_bytes > 0) cuda_ok(cudaMemcpyAsync(p->x_dev[s], x_host, p->x_bytes, cudaMemcpyHostToDevice, p->s_in));
    cuda_ok(cudaEventRecord(p->in_done[s], p->s_in));
    // forward, once x[s] has arrived and copy-out i-depth has read out[s]
    cuda_ok(cudaStreamWaitEvent(p->s_comp, p->in_done[s], 0));
    cuda_ok(cudaStreamWaitEvent(p->s_comp, p->out_done[s], 0));
    if (st == MOE_OK)
        st = moe_forward(&p->cfg, &p->weights, p->x_dev[s], nullptr, nullptr, &p->outs[s], p->ws, p->ws_bytes,
                         p->s_comp);
    cuda_ok(cudaEventRecord(p->comp_done[s], p->s_comp));
    // copy out
    cuda_ok(cudaStreamWaitEvent(p->s_out, p->comp_done[s], 0));
    if (p->x_bytes > 0) cuda_ok(cudaMemcpyAsync(out_host, p->outs[s].out, p->x_bytes, cudaMemcpyDeviceToHost, p->s_out));
    cuda_ok(cudaMemcpyAsync(l_aux_host, p->outs[s].l_aux, sizeof(float), cudaMemcpyDeviceToHost, p->s_out));
    cuda_ok(cudaEventRecord(p->out_done[s], p->s_out));
    if (end_event) cuda_ok(cudaEventRecord(end_event, p->s_out));
    if (prev != p->dev) cudaSetDevice(prev);
    if (ticket) *ticket = p->submitted;
    ++p->submitted;
    return st;
}

moe_status_t moe_pipeline_wait(moe_pipeline_t* p, int64_t ticket) {
    if (p == nullptr || ticket >= p->submitted) return MOE_ERR_INVALID_ARG;
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != p->dev && cudaSetDevice(p->dev) != cudaSuccess) return MOE_ERR_CUDA;
    // the slot's copy-out event marks the newest step that used the slot, which
    // is `ticket` or a later step on the same in-order stream
    const cudaError_t e = ticket < 0 ? cudaStreamSynchronize(p->s_out)
                                     : cudaEventSynchronize(p->out_done[ticket % p->depth]);
    if (prev != p->dev) cudaSetDevice(prev);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_pipeline_check(moe_pipeline_t* p, uint32_t* site) {
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    int prev = 0;
    cudaGetDevice(&prev);
    if (prev != p->dev && cudaSetDevice(p->dev) != cudaSuccess) return MOE_ERR_CUDA;
    moe_status_t st = moe_check_device_status(p->ws, p->ws_bytes, p->s_comp, site);
    if (prev != p->dev) cudaSetDevice(prev);
    return st;
}

moe_status_t moe_pipeline_destroy(moe_pipeline_t* p) {
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    release(p);
    return MOE_OK;
}

}  // extern "C"
