// End-to-end forward passes from host memory (moe_pipeline_* in moe.h).
//
// A native host loop: per step one host -> device copy on the input stream,
// the layer (a CUDA graph replay, or the eager launch sequence) on the run
// stream, one device -> host copy on the output stream, ordered by events
// per lane.  Lane b's input buffer is rewritten only after the layer that
// read it has finished (run_done[b]); its output buffer only after the
// previous copy out of it has finished (out_done[b]).
//
// Included once, at the end of moe.cu (it calls moe_forward_ex and the
// launch-timing switch there).
#pragma once

struct moe_pipeline {
    int device = 0;
    int depth = 0;
    int flags = 0;
    // the layer
    const void* w_router = nullptr;
    const float* logit_bias = nullptr;
    const void *w1 = nullptr, *b1 = nullptr, *w2 = nullptr, *b2 = nullptr;
    int S = 0;
    const void *w1s = nullptr, *b1s = nullptr, *w2s = nullptr, *b2s = nullptr;
    int F = 0, T = 0, d = 0, ff = 0, E = 0, k = 0, capacity = 0, dtype = 0;
    // lanes (caller-owned device memory)
    std::vector<void*> x_dev, out_dev, ws;
    size_t ws_bytes = 0;
    size_t io_bytes = 0;
    // owned
    cudaStream_t s_in = nullptr, s_run = nullptr, s_out = nullptr;
    std::vector<cudaEvent_t> in_done, run_done, out_done;
    cudaEvent_t in_tail = nullptr, run_tail = nullptr;
    cudaEvent_t t0 = nullptr, t1 = nullptr;
    std::vector<cudaGraphExec_t> graphs;
};

namespace {

int pipeline_layer(moe_pipeline* p, int b, cudaStream_t s) {
    return moe_forward_ex(p->x_dev[b], p->w_router, p->logit_bias, p->w1, p->b1, p->w2, p->b2, p->S, p->w1s,
                          p->b1s, p->w2s, p->b2s, p->F, p->T, p->d, p->ff, p->E, p->k, p->capacity, p->dtype,
                          p->out_dev[b], nullptr, nullptr, nullptr, p->ws[b], p->ws_bytes, s);
}

void pipeline_free(moe_pipeline* p) {
    if (p == nullptr) return;
    for (cudaStream_t s : {p->s_in, p->s_run, p->s_out})
        if (s) cudaStreamSynchronize(s);
    for (cudaGraphExec_t g : p->graphs)
        if (g) cudaGraphExecDestroy(g);
    for (auto* v : {&p->in_done, &p->run_done, &p->out_done})
        for (cudaEvent_t e : *v)
            if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : {p->in_tail, p->run_tail, p->t0, p->t1})
        if (e) cudaEventDestroy(e);
    for (cudaStream_t s : {p->s_in, p->s_run, p->s_out})
        if (s) cudaStreamDestroy(s);
    delete p;
}

// Sets the pipeline's device current for the life of the object.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) {
            ok = false;
            prev = -1;
        } else if (prev != dev && cudaSetDevice(dev) != cudaSuccess) {
            ok = false;
        }
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

// Captures lane b's layer call on the run stream into an executable graph.
// The launch-timing switch is off during the capture (its events must not
// become graph nodes).
int pipeline_capture(moe_pipeline* p, int b, cudaGraphExec_t* exec) {
    bool timing;
    {
        std::lock_guard<std::mutex> lk(g_timing.mu);
        timing = g_timing.enabled;
        g_timing.enabled = false;
    }
    int rc = MOE_OK;
    cudaGraph_t graph = nullptr;
    if (cudaStreamBeginCapture(p->s_run, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        rc = MOE_ERR_CUDA;
    } else {
        rc = pipeline_layer(p, b, p->s_run);
        const cudaError_t end = cudaStreamEndCapture(p->s_run, &graph);
        if (rc == MOE_OK && end != cudaSuccess) rc = MOE_ERR_CUDA;
        if (rc == MOE_OK && cudaGraphInstantiate(exec, graph, 0) != cudaSuccess) rc = MOE_ERR_CUDA;
        if (graph) cudaGraphDestroy(graph);
    }
    {
        std::lock_guard<std::mutex> lk(g_timing.mu);
        g_timing.enabled = timing;
    }
    return rc;
}

}  // namespace

extern "C" {

int moe_pipeline_create(const void* w_router, const float* logit_bias, const void* w1, const void* b1,
                        const void* w2, const void* b2, int S, const void* w1s, const void* b1s, const void* w2s,
                        const void* b2s, int reroute_rounds, int T, int d, int ff, int E, int k, int capacity,
                        int dtype, int depth, void* const* x_dev, void* const* out_dev, void* const* ws,
                        size_t ws_bytes, int flags, moe_pipeline** out) {
    if (out == nullptr) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (depth < 1 || depth > MOE_PIPELINE_MAX_DEPTH || (flags & ~MOE_PIPELINE_GRAPHS) != 0 || T < 1 ||
        x_dev == nullptr || out_dev == nullptr || ws == nullptr)
        return MOE_ERR_INVALID_ARG;
    const size_t need = moe_forward_ex_workspace_size(T, d, ff, E, k, S, reroute_rounds, dtype);
    if (need == 0) return MOE_ERR_INVALID_ARG;
    for (int b = 0; b < depth; ++b) {
        if (x_dev[b] == nullptr || out_dev[b] == nullptr || !aligned16(x_dev[b]) || !aligned16(out_dev[b]))
            return MOE_ERR_INVALID_ARG;
        if (ws[b] == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws[b]) & 255u) != 0)
            return MOE_ERR_WORKSPACE;
    }

    moe_pipeline* p = new moe_pipeline;
    p->depth = depth;
    p->flags = flags;
    p->w_router = w_router;
    p->logit_bias = logit_bias;
    p->w1 = w1;
    p->b1 = b1;
    p->w2 = w2;
    p->b2 = b2;
    p->S = S;
    p->w1s = w1s;
    p->b1s = b1s;
    p->w2s = w2s;
    p->b2s = b2s;
    p->F = reroute_rounds;
    p->T = T;
    p->d = d;
    p->ff = ff;
    p->E = E;
    p->k = k;
    p->capacity = capacity;
    p->dtype = dtype;
    p->x_dev.assign(x_dev, x_dev + depth);
    p->out_dev.assign(out_dev, out_dev + depth);
    p->ws.assign(ws, ws + depth);
    p->ws_bytes = ws_bytes;
    p->io_bytes = size_t(T) * d * elem_bytes(dtype);

    auto fail = [&](int rc) {
        pipeline_free(p);
        return rc;
    };
    if (cudaGetDevice(&p->device) != cudaSuccess) return fail(MOE_ERR_CUDA);
    for (cudaStream_t* s : {&p->s_in, &p->s_run, &p->s_out})
        if (cudaStreamCreateWithFlags(s, cudaStreamNonBlocking) != cudaSuccess) return fail(MOE_ERR_CUDA);
    for (auto* v : {&p->in_done, &p->run_done, &p->out_done}) {
        v->assign(depth, nullptr);
        for (cudaEvent_t& e : *v)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return fail(MOE_ERR_CUDA);
    }
    for (cudaEvent_t* e : {&p->in_tail, &p->run_tail})
        if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return fail(MOE_ERR_CUDA);
    for (cudaEvent_t* e : {&p->t0, &p->t1})
        if (cudaEventCreate(e) != cudaSuccess) return fail(MOE_ERR_CUDA);

    // warm-up: one eager pass per lane on zeroed inputs (validates the
    // layer's arguments and sets the kernels' attributes before any capture)
    for (int b = 0; b < depth; ++b) {
        if (cudaMemsetAsync(p->x_dev[b], 0, p->io_bytes, p->s_run) != cudaSuccess) return fail(MOE_ERR_CUDA);
        const int rc = pipeline_layer(p, b, p->s_run);
        if (rc != MOE_OK) return fail(rc);
    }
    if (cudaStreamSynchronize(p->s_run) != cudaSuccess) return fail(MOE_ERR_CUDA);
    if (flags & MOE_PIPELINE_GRAPHS) {
        p->graphs.assign(depth, nullptr);
        for (int b = 0; b < depth; ++b) {
            const int rc = pipeline_capture(p, b, &p->graphs[b]);
            if (rc != MOE_OK) return fail(rc);
        }
    }
    *out = p;
    return MOE_OK;
}

int moe_pipeline_run(moe_pipeline* p, const void* const* x_host, void* const* out_host, int n,
                     float* elapsed_ms) {
    if (p == nullptr || n < 0 || (n > 0 && (x_host == nullptr || out_host == nullptr))) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (x_host[i] == nullptr || out_host[i] == nullptr) return MOE_ERR_INVALID_ARG;
    TraceRange trace_("moe_pipeline_run");
    DeviceGuard guard(p->device);
    if (!guard.ok) return MOE_ERR_CUDA;
    bool ok = cudaEventRecord(p->t0, p->s_in) == cudaSuccess && cudaStreamWaitEvent(p->s_run, p->t0, 0) == cudaSuccess &&
              cudaStreamWaitEvent(p->s_out, p->t0, 0) == cudaSuccess;
    int rc = MOE_OK;
    for (int i = 0; ok && i < n; ++i) {
        const int b = i % p->depth;
        // input copy once the lane's previous layer has read its input
        ok = cudaStreamWaitEvent(p->s_in, p->run_done[b], 0) == cudaSuccess &&
             cudaMemcpyAsync(p->x_dev[b], x_host[i], p->io_bytes, cudaMemcpyHostToDevice, p->s_in) == cudaSuccess &&
             cudaEventRecord(p->in_done[b], p->s_in) == cudaSuccess &&
             // the layer once the input is in and the lane's previous output is out
             cudaStreamWaitEvent(p->s_run, p->in_done[b], 0) == cudaSuccess &&
             cudaStreamWaitEvent(p->s_run, p->out_done[b], 0) == cudaSuccess;
        if (!ok) break;
        if (!p->graphs.empty()) {
            ok = cudaGraphLaunch(p->graphs[b], p->s_run) == cudaSuccess;
        } else if ((rc = pipeline_layer(p, b, p->s_run)) != MOE_OK) {
            break;
        }
        ok = ok && cudaEventRecord(p->run_done[b], p->s_run) == cudaSuccess &&
             // the output copy once the layer is done
             cudaStreamWaitEvent(p->s_out, p->run_done[b], 0) == cudaSuccess &&
             cudaMemcpyAsync(out_host[i], p->out_dev[b], p->io_bytes, cudaMemcpyDeviceToHost, p->s_out) ==
                 cudaSuccess &&
             cudaEventRecord(p->out_done[b], p->s_out) == cudaSuccess;
    }
    // the end of all three streams, on the output stream
    ok = ok && rc == MOE_OK && cudaEventRecord(p->in_tail, p->s_in) == cudaSuccess &&
         cudaEventRecord(p->run_tail, p->s_run) == cudaSuccess &&
         cudaStreamWaitEvent(p->s_out, p->in_tail, 0) == cudaSuccess &&
         cudaStreamWaitEvent(p->s_out, p->run_tail, 0) == cudaSuccess &&
         cudaEventRecord(p->t1, p->s_out) == cudaSuccess;
    // every issued step completes before returning, also on an error
    for (cudaStream_t s : {p->s_in, p->s_run, p->s_out})
        if (cudaStreamSynchronize(s) != cudaSuccess) ok = false;
    if (rc != MOE_OK) return rc;
    if (!ok) return MOE_ERR_CUDA;
    if (elapsed_ms != nullptr && cudaEventElapsedTime(elapsed_ms, p->t0, p->t1) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_pipeline_destroy(moe_pipeline* p) {
    if (p == nullptr) return MOE_OK;
    DeviceGuard guard(p->device);
    pipeline_free(p);
    return guard.ok ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
