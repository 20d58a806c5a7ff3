// Streaming session: one Gated DeltaNet layer step (pre-processing ->
// recurrence with a carried state -> output gate) over a constant-size
// memory, replayed as a CUDA graph.
//
// The InfiniteVL project page ("Advanced Usage: CUDA Graph Acceleration",
// "Accelerated Streaming Inference", "Accelerated Decode") streams a video
// frame by frame: because the linear layers keep a fixed-size state instead
// of a growing cache, the per-frame computation (and the per-token decode
// step) has fixed shapes and fixed buffers, so it can be captured once and
// replayed without launch overhead.  The caller owns every buffer (states,
// staging, intermediates, workspace) and keeps them in place for the
// session's lifetime; the session holds their addresses, a capture stream and
// the instantiated graphs.  A step is captured on first use for its token
// count (full segments, partial segments and the decode step each get a
// graph) and replayed on the caller's stream afterwards.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <new>

#include "gdn.h"
#include "gdn_internal.h"

namespace {

constexpr int kMaxGraphs = 8;   // distinct per-stream token counts kept instantiated

struct Graph {
    int tokens = -1;            // tokens per stream; 0 = the decode step
    cudaGraphExec_t exec = nullptr;
};

}  // namespace

struct gdn_session {
    int B, H, d, seg, dtype, activation, gate;
    float eps;
    gdn_session_buffers_t buf;
    cudaStream_t cap = nullptr;            // capture stream (owned)
    Graph graphs[kMaxGraphs];
    std::mutex mu;
};

namespace {

int cuda_status(cudaError_t e) { return e == cudaSuccess ? GDN_OK : gdn::note_cuda_error(e); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The layer step for `tokens` tokens per stream (0: one decode token per
// stream), enqueued on `st` through the public entry points: a segment is one
// gdn_layer_prefill call (pre-processing and output gate fused into the
// prefill kernels on the tensor-core path), a decode token is
// gdn_preprocess -> gdn_decode_step -> gdn_output_gate.
int enqueue_step(gdn_session *s, int tokens, cudaStream_t st) {
    const gdn_session_buffers_t &b = s->buf;
    const int B = s->B, H = s->H, d = s->d;
    if (tokens > 0) {
        const int64_t T = (int64_t)B * tokens;
        return gdn_layer_prefill(b.xq, b.xk, b.xv, b.conv_w, b.a, b.b, b.conv_state, b.conv_state, b.state, b.state,
                                 b.z, b.norm_w, b.y, nullptr, B, T, H, d, s->activation, s->gate, s->eps, s->dtype,
                                 b.workspace, b.workspace_bytes, st);
    }
    int rc = gdn_preprocess(b.xq, b.xk, b.xv, b.conv_w, b.a, b.b, b.conv_state, b.q, b.k, b.v, b.g, b.beta,
                            b.conv_state, nullptr, B, B, H, d, s->activation, s->eps, s->dtype, st);
    if (rc != GDN_OK) return rc;
    rc = gdn_decode_step(b.q, b.k, b.v, b.g, b.beta, b.state, b.state, b.o, B, H, d, d, s->dtype, st);
    if (rc != GDN_OK) return rc;
    return gdn_output_gate(b.o, b.z, b.norm_w, b.y, (int64_t)B * H, d, s->gate, s->eps, s->dtype, st);
}

// Instantiated graph of the step for `tokens`, captured on first use.
int graph_for(gdn_session *s, int tokens, cudaGraphExec_t *out) {
    for (Graph &g : s->graphs)
        if (g.exec && g.tokens == tokens) {
            *out = g.exec;
            return GDN_OK;
        }
    cudaError_t e = cudaStreamBeginCapture(s->cap, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return cuda_status(e);
    const int rc = enqueue_step(s, tokens, s->cap);
    cudaGraph_t graph = nullptr;
    e = cudaStreamEndCapture(s->cap, &graph);
    if (rc != GDN_OK) {
        if (graph) cudaGraphDestroy(graph);
        return rc;
    }
    if (e != cudaSuccess) return cuda_status(e);
    cudaGraphExec_t exec = nullptr;
    e = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) return cuda_status(e);
    Graph *slot = &s->graphs[0];
    for (Graph &g : s->graphs)
        if (!g.exec) {
            slot = &g;
            break;
        }
    if (slot->exec) cudaGraphExecDestroy(slot->exec);   // all slots used: replace the first
    slot->exec = exec;
    slot->tokens = tokens;
    *out = exec;
    return GDN_OK;
}

int launch_graph(gdn_session *s, int tokens, void *stream) {
    std::lock_guard<std::mutex> lock(s->mu);
    cudaGraphExec_t exec = nullptr;
    const int rc = graph_for(s, tokens, &exec);
    if (rc != GDN_OK) return rc;
    return cuda_status(cudaGraphLaunch(exec, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

size_t gdn_session_workspace_size(int num_streams, int H, int d, int seg_tokens, int dtype) {
    if (num_streams < 1 || seg_tokens < 1) return 0;
    return gdn_layer_prefill_workspace_size(num_streams, (int64_t)num_streams * seg_tokens, H, d, dtype);
}

int gdn_session_create(int num_streams, int H, int d, int seg_tokens, int dtype, int activation, int gate,
                       float eps, const gdn_session_buffers_t *buffers, gdn_session **out) {
    if (!out) return GDN_ERR_INVALID_ARG;
    *out = nullptr;
    if (!buffers || num_streams < 1 || H < 1 || seg_tokens < 1) return GDN_ERR_INVALID_ARG;
    if ((int64_t)num_streams * seg_tokens * H > ((int64_t)1 << 31)) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (activation != GDN_ACT_NONE && activation != GDN_ACT_SILU) return GDN_ERR_INVALID_ARG;
    if (gate != GDN_GATE_SIGMOID && gate != GDN_GATE_SILU) return GDN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1.f) return GDN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return GDN_ERR_UNSUPPORTED;
    const gdn_session_buffers_t &b = *buffers;
    const void *need[] = {b.xq, b.xk, b.xv, b.a, b.b, b.z, b.y, b.q, b.k, b.v, b.o, b.g, b.beta, b.state,
                          b.conv_state, b.conv_w};
    for (const void *p : need)
        if (!p || !aligned16(p)) return GDN_ERR_INVALID_ARG;
    if ((b.norm_w && !aligned16(b.norm_w)) || (b.workspace && !aligned16(b.workspace))) return GDN_ERR_INVALID_ARG;
    const size_t ws = gdn_session_workspace_size(num_streams, H, d, seg_tokens, dtype);
    if (b.workspace_bytes < ws || (ws > 0 && !b.workspace)) return GDN_ERR_WORKSPACE;
    // the kernels' one-time per-device set-up, here and not inside a later capture
    cudaError_t e = gdn::prefill_tc_setup();
    if (e == cudaSuccess) e = gdn::layer_ops_setup(dtype, d);
    if (e != cudaSuccess) return cuda_status(e);
    gdn_session *s = new (std::nothrow) gdn_session();
    if (!s) return GDN_ERR_INVALID_ARG;
    s->B = num_streams;
    s->H = H;
    s->d = d;
    s->seg = seg_tokens;
    s->dtype = dtype;
    s->activation = activation;
    s->gate = gate;
    s->eps = eps;
    s->buf = b;
    e = cudaStreamCreateWithFlags(&s->cap, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
        delete s;
        return cuda_status(e);
    }
    *out = s;
    return GDN_OK;
}

int gdn_session_prefill(gdn_session *s, int tokens, void *stream) {
    if (!s || tokens < 1 || tokens > s->seg) return GDN_ERR_INVALID_ARG;
    return launch_graph(s, tokens, stream);
}

int gdn_session_decode(gdn_session *s, void *stream) {
    if (!s) return GDN_ERR_INVALID_ARG;
    return launch_graph(s, 0, stream);
}

int gdn_session_step_eager(gdn_session *s, int tokens, void *stream) {
    if (!s || tokens < 0 || tokens > s->seg) return GDN_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(s->mu);
    return enqueue_step(s, tokens, static_cast<cudaStream_t>(stream));
}

int gdn_session_graph_count(const gdn_session *s) {
    if (!s) return 0;
    int n = 0;
    for (const Graph &g : s->graphs) n += g.exec != nullptr;
    return n;
}

void gdn_session_destroy(gdn_session *s) {
    if (!s) return;
    for (Graph &g : s->graphs)
        if (g.exec) cudaGraphExecDestroy(g.exec);
    if (s->cap) cudaStreamDestroy(s->cap);
    delete s;
}

}  // extern "C"
