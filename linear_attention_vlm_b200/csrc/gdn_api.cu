// Host side of the C ABI declared in include/gdn.h: argument validation,
// workspace sizing and dispatch to the kernels.  No allocation, no device
// synchronisation.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "gdn.h"
#include "gdn_internal.h"
#include "prefill_tc.h"

namespace {

thread_local char g_last_cuda_error[256] = "";

int cuda_fail(cudaError_t e) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return GDN_ERR_CUDA;
}

bool misaligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

bool shape_supported(int dk, int dv) { return dk == dv && (dk == 64 || dk == 128); }

// The fused tensor-core kernel covers bf16 with d_k = d_v = 128; everything
// else (fp32, d = 64, an empty batch) takes the SIMT kernel.
bool use_tc(int64_t total_tokens, int dk, int dtype) {
    return dtype == GDN_BF16 && dk == 128 && total_tokens > 0;
}

constexpr uint64_t kWaitLimitNs = GDN_WAIT_LIMIT_DEFAULT;   // 2 s bound on any in-kernel wait

// Bound on the work-loop waits of the kernels this host thread launches
// (gdn_set_wait_limit); the drains before a kernel exits always keep 2 s.
thread_local uint64_t g_wait_limit_ns = kWaitLimitNs;

// Common validation of gdn_prefill's arguments (without workspace).
int check_prefill(const void *q, const void *k, const void *v, const float *g,
                  const float *beta, const float *state_in, const void *out,
                  const float *state_out, const int32_t *cu_seqlens, int num_seqs,
                  int64_t total_tokens, int H, int dk, int dv, int chunk, int dtype) {
    if (num_seqs < 1 || H < 1 || total_tokens < 0 || dk < 1 || dv < 1) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (chunk != gdn::kChunk || !shape_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)num_seqs * H > (int64_t)INT32_MAX / 2) return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, state_in, out, state_out, cu_seqlens};
    for (const void *p : ptrs)
        if (p && misaligned(p)) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && total_tokens % num_seqs != 0) return GDN_ERR_INVALID_ARG;
    if (state_out && state_in && state_out != state_in) {
        const size_t bytes = (size_t)num_seqs * H * dv * dk * sizeof(float);
        const char *a = reinterpret_cast<const char *>(state_in);
        const char *b = reinterpret_cast<const char *>(state_out);
        if (a < b + bytes && b < a + bytes) return GDN_ERR_INVALID_ARG;   // partial overlap
    }
    return GDN_OK;
}

// true if [a, a + na) and [b, b + nb) share a byte
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const char *x = static_cast<const char *>(a), *y = static_cast<const char *>(b);
    return x < y + nb && y < x + na;
}

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// Workspace of gdn_layer_prefill.  Tensor-core path: [prefill workspace]
// [q][k][v] (processed, dtype) [g][beta] (fp32); otherwise [q][k][v][o][g][beta].
struct LayerWs {
    size_t prefill, tens, gates, total;
};

LayerWs layer_ws(int num_seqs, int64_t total_tokens, int H, int d, int dtype) {
    LayerWs w{0, 0, 0, 0};
    const size_t es = dtype == GDN_BF16 ? 2 : 4;
    w.tens = align256((size_t)total_tokens * H * d * es);
    w.gates = align256((size_t)total_tokens * H * 4);
    if (use_tc(total_tokens, d, dtype)) {
        w.prefill = align256(gdn::tc_workspace_bytes(num_seqs, total_tokens, H, /*varlen=*/true));
        w.total = w.prefill + 3 * w.tens + 2 * w.gates;
    } else {
        w.total = 4 * w.tens + 2 * w.gates;
    }
    return w;
}

}  // namespace

int gdn::note_cuda_error(cudaError_t e) { return cuda_fail(e); }

extern "C" {

const char *gdn_status_string(int status) {
    switch (status) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: invalid argument";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: shape, chunk or dtype not implemented";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA: CUDA runtime error";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: a wait inside a kernel gave up";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing or too small";
        default: return "unknown gdn_status";
    }
}

const char *gdn_last_cuda_error(void) { return g_last_cuda_error; }

void gdn_set_wait_limit(uint64_t ns) { g_wait_limit_ns = ns; }

int gdn_read_status(const int32_t *word, void *stream, int32_t *code) {
    if (code) *code = 0;
    if (!word || (reinterpret_cast<uintptr_t>(word) & 3u)) return GDN_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, word, sizeof(h), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (code) *code = h;
    return h == 0 ? GDN_OK : GDN_ERR_TIMEOUT;
}

size_t gdn_prefill_workspace_size(int num_seqs, int64_t total_tokens, int H, int dk, int dv,
                                  int chunk, int dtype) {
    if (num_seqs < 1 || H < 1 || total_tokens < 0) return 0;
    if (chunk != gdn::kChunk || !shape_supported(dk, dv)) return 0;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return 0;
    return use_tc(total_tokens, dk, dtype)
               ? gdn::tc_workspace_bytes(num_seqs, total_tokens, H, /*varlen=*/true)
               : 0;
}

int gdn_prefill_kernel_count(int num_seqs, int64_t total_tokens, int H, int dk, int dv,
                             int chunk, int dtype, int packed) {
    if (num_seqs < 1 || H < 1 || total_tokens < 0) return 0;
    if (chunk != gdn::kChunk || !shape_supported(dk, dv)) return 0;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return 0;
    return use_tc(total_tokens, dk, dtype)
               ? gdn::tc_kernel_count(num_seqs, total_tokens, H, packed != 0)
               : 1;
}

int gdn_prefill(const void *q, const void *k, const void *v, const float *g, const float *beta,
                const float *state_in, void *out, float *state_out, const int32_t *cu_seqlens,
                int num_seqs, int64_t total_tokens, int H, int dk, int dv, int chunk, int dtype,
                void *workspace, size_t workspace_bytes, void *stream) {
    int st = check_prefill(q, k, v, g, beta, state_in, out, state_out, cu_seqlens, num_seqs,
                           total_tokens, H, dk, dv, chunk, dtype);
    if (st != GDN_OK) return st;
    const size_t need = gdn_prefill_workspace_size(num_seqs, total_tokens, H, dk, dv, chunk, dtype);
    if (need > 0 && (!workspace || workspace_bytes < need)) return GDN_ERR_WORKSPACE;
    if (workspace && misaligned(workspace)) return GDN_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t uniform_len = cu_seqlens ? 0 : total_tokens / num_seqs;
    if (use_tc(total_tokens, dk, dtype)) {
        int *err = static_cast<int *>(workspace);
        cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
        if (e != cudaSuccess) return cuda_fail(e);
        gdn::TcLaunch L{q, k, v, g, beta, state_in, out, state_out, cu_seqlens, uniform_len,
                        total_tokens, num_seqs, H, workspace, err, g_wait_limit_ns, kWaitLimitNs, nullptr};
        e = gdn::launch_prefill_tc(L, s);
        return e == cudaSuccess ? GDN_OK : cuda_fail(e);
    }
    cudaError_t e = gdn::launch_prefill_simt(dtype, dk, q, k, v, g, beta, state_in, out,
                                             state_out, cu_seqlens, uniform_len, num_seqs, H, s);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

int gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                    const float *beta, const float *state_in, float *state_out, void *out,
                    int B, int H, int dk, int dv, int dtype, void *stream) {
    if (B < 0 || H < 1) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!shape_supported(dk, dv)) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if ((int64_t)B * H > (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, state_in, state_out, out};
    for (const void *p : ptrs)
        if (!p || misaligned(p)) return GDN_ERR_INVALID_ARG;
    if (state_out != state_in) {
        const size_t bytes = (size_t)B * H * dv * dk * sizeof(float);
        const char *a = reinterpret_cast<const char *>(state_in);
        const char *b = reinterpret_cast<const char *>(state_out);
        if (a < b + bytes && b < a + bytes) return GDN_ERR_INVALID_ARG;
    }
    cudaError_t e = gdn::launch_decode(dtype, dk, q, k, v, g, beta, state_in, state_out, out, B,
                                       H, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

int gdn_preprocess(const void *xq, const void *xk, const void *xv, const float *conv_w,
                   const float *a_logit, const float *b_logit, const void *conv_state_in, void *q,
                   void *k, void *v, float *g, float *beta, void *conv_state_out,
                   const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens, int H, int d,
                   int activation, float eps, int dtype, void *stream) {
    if (num_seqs < 1 || H < 1 || total_tokens < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (activation != GDN_ACT_NONE && activation != GDN_ACT_SILU) return GDN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1.f) return GDN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)num_seqs * 3 * 3 * H * d > (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (total_tokens > (int64_t)INT32_MAX * 32) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && total_tokens % num_seqs != 0) return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!xq || !xk || !xv || !conv_w || !a_logit || !b_logit || !q || !k || !v || !g || !beta))
        return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {xq, xk, xv, conv_w, a_logit, b_logit, conv_state_in, q, k, v, g, beta, conv_state_out,
                          cu_seqlens};
    for (const void *p : ptrs)
        if (p && misaligned(p)) return GDN_ERR_INVALID_ARG;
    const size_t es = dtype == GDN_BF16 ? 2 : 4;
    const size_t tens = (size_t)total_tokens * H * d * es, gates = (size_t)total_tokens * H * 4;
    const size_t st = (size_t)num_seqs * 9 * H * d * es;
    // no output may overlap an input; the convolution state may be updated in place
    const void *outs[] = {q, k, v, g, beta};
    const size_t out_n[] = {tens, tens, tens, gates, gates};
    const void *ins[] = {xq, xk, xv, a_logit, b_logit, conv_state_in, conv_w};
    const size_t in_n[] = {tens, tens, tens, gates, gates, st, (size_t)3 * H * d * 16};
    for (int i = 0; i < 5; ++i) {
        for (int j = 0; j < 7; ++j)
            if (overlaps(outs[i], out_n[i], ins[j], in_n[j])) return GDN_ERR_INVALID_ARG;
        if (overlaps(outs[i], out_n[i], conv_state_out, st)) return GDN_ERR_INVALID_ARG;
        for (int j = i + 1; j < 5; ++j)
            if (overlaps(outs[i], out_n[i], outs[j], out_n[j])) return GDN_ERR_INVALID_ARG;
    }
    for (int j = 0; j < 7; ++j)
        if (j != 5 && overlaps(conv_state_out, st, ins[j], in_n[j])) return GDN_ERR_INVALID_ARG;
    if (conv_state_out && conv_state_in && conv_state_out != conv_state_in && overlaps(conv_state_out, st, conv_state_in, st))
        return GDN_ERR_INVALID_ARG;
    if (total_tokens == 0 && !conv_state_out) return GDN_OK;
    gdn::PreprocessArgs A;
    A.xq = xq; A.xk = xk; A.xv = xv;
    A.conv_w = conv_w; A.a_logit = a_logit; A.b_logit = b_logit;
    A.cs_in = conv_state_in;
    A.q = q; A.k = k; A.v = v; A.g = g; A.beta = beta;
    A.cs_out = conv_state_out;
    A.cu_seqlens = cu_seqlens;
    A.num_seqs = num_seqs;
    A.total_tokens = total_tokens;
    A.H = H; A.d = d; A.activation = activation; A.dtype = dtype;
    A.eps = eps;
    const cudaError_t e = gdn::launch_preprocess(A, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

int gdn_output_gate(const void *o, const void *z, const float *norm_w, void *y, int64_t rows, int dv,
                    int gate, float eps, int dtype, void *stream) {
    if (rows < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (gate != GDN_GATE_SIGMOID && gate != GDN_GATE_SILU) return GDN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1.f) return GDN_ERR_INVALID_ARG;
    if (dv != 64 && dv != 128) return GDN_ERR_UNSUPPORTED;
    if (rows == 0) return GDN_OK;
    if (rows > (int64_t)INT32_MAX * 8) return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {o, z, y};
    for (const void *p : ptrs)
        if (!p || misaligned(p)) return GDN_ERR_INVALID_ARG;
    if (norm_w && misaligned(norm_w)) return GDN_ERR_INVALID_ARG;
    const size_t n = (size_t)rows * dv * (dtype == GDN_BF16 ? 2 : 4);
    // y may equal o (in place); no other overlap
    if (y != o && overlaps(y, n, o, n)) return GDN_ERR_INVALID_ARG;
    if (overlaps(y, n, z, n) || overlaps(y, n, norm_w, (size_t)dv * 4)) return GDN_ERR_INVALID_ARG;
    const cudaError_t e = gdn::launch_output_gate(dtype, dv, o, z, norm_w, y, rows, gate, eps,
                                                  static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

size_t gdn_layer_prefill_workspace_size(int num_seqs, int64_t total_tokens, int H, int d, int dtype) {
    if (num_seqs < 1 || H < 1 || total_tokens < 0) return 0;
    if ((d != 64 && d != 128) || (dtype != GDN_F32 && dtype != GDN_BF16)) return 0;
    return layer_ws(num_seqs, total_tokens, H, d, dtype).total;
}

int gdn_layer_prefill(const void *xq, const void *xk, const void *xv, const float *conv_w, const float *a_logit,
                      const float *b_logit, const void *conv_state_in, void *conv_state_out, const float *state_in,
                      float *state_out, const void *z, const float *norm_w, void *y, const int32_t *cu_seqlens,
                      int num_seqs, int64_t total_tokens, int H, int d, int activation, int gate, float eps,
                      int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (num_seqs < 1 || H < 1 || total_tokens < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (activation != GDN_ACT_NONE && activation != GDN_ACT_SILU) return GDN_ERR_INVALID_ARG;
    if (gate != GDN_GATE_SIGMOID && gate != GDN_GATE_SILU) return GDN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1.f) return GDN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)num_seqs * H > (int64_t)INT32_MAX / 2) return GDN_ERR_INVALID_ARG;
    if ((int64_t)num_seqs * 3 * 3 * H * d > (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;
    if (total_tokens > (int64_t)INT32_MAX * 8) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && total_tokens % num_seqs != 0) return GDN_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!xq || !xk || !xv || !conv_w || !a_logit || !b_logit || !z || !y))
        return GDN_ERR_INVALID_ARG;
    const void *ptrs[] = {xq, xk, xv, conv_w, a_logit, b_logit, conv_state_in, conv_state_out, state_in, state_out,
                          z, norm_w, y, cu_seqlens, workspace};
    for (const void *p : ptrs)
        if (p && misaligned(p)) return GDN_ERR_INVALID_ARG;
    const LayerWs W = layer_ws(num_seqs, total_tokens, H, d, dtype);
    if (!workspace || workspace_bytes < W.total) return GDN_ERR_WORKSPACE;
    const size_t es = dtype == GDN_BF16 ? 2 : 4;
    const size_t tens = (size_t)total_tokens * H * d * es, gates = (size_t)total_tokens * H * 4;
    const size_t cst = (size_t)num_seqs * 9 * H * d * es, st = (size_t)num_seqs * H * d * d * 4;
    // y, the workspace and the states may not overlap the inputs or each other;
    // the convolution and recurrent states may each be updated in place
    const void *ins[] = {xq, xk, xv, conv_w, a_logit, b_logit, z, norm_w, cu_seqlens};
    const size_t in_n[] = {tens, tens, tens, (size_t)3 * H * d * 16, gates, gates, tens, (size_t)d * 4,
                           (size_t)(num_seqs + 1) * 4};
    const void *outs[] = {y, workspace, conv_state_out, state_out};
    const size_t out_n[] = {tens, W.total, cst, st};
    for (int i = 0; i < 4; ++i) {
        for (int j = 0; j < 9; ++j)
            if (overlaps(outs[i], out_n[i], ins[j], in_n[j])) return GDN_ERR_INVALID_ARG;
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(outs[i], out_n[i], outs[j], out_n[j])) return GDN_ERR_INVALID_ARG;
    }
    const void *states_in[] = {conv_state_in, state_in};
    const size_t states_n[] = {cst, st};
    for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 2; ++j) {
            if (overlaps(outs[j], out_n[j], states_in[i], states_n[i])) return GDN_ERR_INVALID_ARG;
            if (overlaps(outs[2 + j], out_n[2 + j], states_in[i], states_n[i]) &&
                !(i == j && outs[2 + j] == states_in[i]))
                return GDN_ERR_INVALID_ARG;   // each state in place (the same buffer) or apart
        }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int64_t uniform_len = cu_seqlens ? 0 : total_tokens / num_seqs;
    cudaError_t e = cudaSuccess;
    if (use_tc(total_tokens, d, dtype)) {
        // one pass of prep + chain kernels; the convolution state is written
        // after them (it may be the state they read)
        int *err = reinterpret_cast<int *>(ws);
        e = cudaMemsetAsync(err, 0, sizeof(int), s);
        if (e != cudaSuccess) return cuda_fail(e);
        gdn::TcLayer Ly;
        Ly.xq = xq; Ly.xk = xk; Ly.xv = xv;
        Ly.conv_w = conv_w; Ly.a_logit = a_logit; Ly.b_logit = b_logit;
        Ly.cs_in = conv_state_in;
        Ly.q = ws + W.prefill;
        Ly.k = ws + W.prefill + W.tens;
        Ly.v = ws + W.prefill + 2 * W.tens;
        Ly.g = reinterpret_cast<float *>(ws + W.prefill + 3 * W.tens);
        Ly.beta = reinterpret_cast<float *>(ws + W.prefill + 3 * W.tens + W.gates);
        Ly.activation = activation;
        Ly.eps = eps;
        Ly.z = z;
        Ly.norm_w = norm_w;
        Ly.gate = gate;
        gdn::TcLaunch L{nullptr, nullptr, nullptr, nullptr, nullptr, state_in, y, state_out, cu_seqlens, uniform_len,
                        total_tokens, num_seqs, H, workspace, err, g_wait_limit_ns, kWaitLimitNs, &Ly};
        e = gdn::launch_prefill_tc(L, s);
    } else {
        // the three steps one after another through the workspace
        void *q = ws, *k = ws + W.tens, *v = ws + 2 * W.tens, *o = ws + 3 * W.tens;
        float *g = reinterpret_cast<float *>(ws + 4 * W.tens);
        float *beta = reinterpret_cast<float *>(ws + 4 * W.tens + W.gates);
        if (total_tokens > 0) {
            gdn::PreprocessArgs A;
            A.xq = xq; A.xk = xk; A.xv = xv;
            A.conv_w = conv_w; A.a_logit = a_logit; A.b_logit = b_logit;
            A.cs_in = conv_state_in;
            A.q = q; A.k = k; A.v = v; A.g = g; A.beta = beta;
            A.cs_out = nullptr;
            A.cu_seqlens = cu_seqlens;
            A.num_seqs = num_seqs;
            A.total_tokens = total_tokens;
            A.H = H; A.d = d; A.activation = activation; A.dtype = dtype;
            A.eps = eps;
            e = gdn::launch_preprocess(A, s);
        }
        if (e == cudaSuccess)
            e = gdn::launch_prefill_simt(dtype, d, q, k, v, g, beta, state_in, o, state_out, cu_seqlens, uniform_len,
                                         num_seqs, H, s);
        if (e == cudaSuccess && total_tokens > 0)
            e = gdn::launch_output_gate(dtype, d, o, z, norm_w, y, total_tokens * H, gate, eps, s);
    }
    if (e == cudaSuccess && conv_state_out)
        e = gdn::launch_conv_state(dtype, d, xq, xk, xv, conv_state_in, conv_state_out, cu_seqlens, num_seqs,
                                   total_tokens, H, s);
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

int gdn_rope(const void *x, void *out, const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens, int H, int d,
             int pos_offset, float base, int dtype, void *stream) {
    if (num_seqs < 1 || H < 1 || total_tokens < 0 || pos_offset < 0) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (!(base > 1.f) || !(base < 3.0e38f)) return GDN_ERR_INVALID_ARG;
    if (d < 8 || d > 256 || d % 8 != 0) return GDN_ERR_UNSUPPORTED;
    if (total_tokens > (int64_t)INT32_MAX || total_tokens + pos_offset > (int64_t)INT32_MAX)
        return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && total_tokens % num_seqs != 0) return GDN_ERR_INVALID_ARG;
    if (total_tokens == 0) return GDN_OK;
    if (!x || !out || misaligned(x) || misaligned(out) || (cu_seqlens && misaligned(cu_seqlens)))
        return GDN_ERR_INVALID_ARG;
    const size_t n = (size_t)total_tokens * H * d * (dtype == GDN_BF16 ? 2 : 4);
    if (out != x && overlaps(out, n, x, n)) return GDN_ERR_INVALID_ARG;   // in place, or apart
    const cudaError_t e = gdn::launch_rope(dtype, x, out, cu_seqlens, num_seqs, total_tokens, H, d, pos_offset,
                                           (double)base, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

int gdn_swa_attention(const void *q, const void *k, const void *v, void *o, const int32_t *cu_seqlens,
                      int num_seqs, int64_t total_tokens, int Hq, int Hkv, int d, int window, float scale,
                      int dtype, int32_t *status, void *stream) {
    if (num_seqs < 1 || Hq < 1 || Hkv < 1 || total_tokens < 0 || window < 1) return GDN_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || Hq > 65535) return GDN_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || !(scale < 3.0e38f)) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 || d != 128) return GDN_ERR_UNSUPPORTED;
    if (total_tokens > (int64_t)INT32_MAX - 256) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && total_tokens % num_seqs != 0) return GDN_ERR_INVALID_ARG;
    if (total_tokens == 0) return GDN_OK;
    const void *ptrs[] = {q, k, v, o};
    for (const void *p : ptrs)
        if (!p || misaligned(p)) return GDN_ERR_INVALID_ARG;
    if ((cu_seqlens && misaligned(cu_seqlens)) || (reinterpret_cast<uintptr_t>(status) & 3u))
        return GDN_ERR_INVALID_ARG;
    const size_t nq = (size_t)total_tokens * Hq * d * 2, nkv = (size_t)total_tokens * Hkv * d * 2;
    if (overlaps(o, nq, q, nq) || overlaps(o, nq, k, nkv) || overlaps(o, nq, v, nkv)) return GDN_ERR_INVALID_ARG;
    gdn::SwaLaunch L;
    L.q = q; L.k = k; L.v = v; L.o = o;
    L.cu_seqlens = cu_seqlens;
    L.num_seqs = num_seqs;
    L.total_tokens = total_tokens;
    L.Hq = Hq; L.Hkv = Hkv; L.window = window;
    L.scale = scale > 0.f ? scale : 1.f / sqrtf((float)d);
    L.err = status;
    L.timeout_ns = g_wait_limit_ns;
    L.drain_ns = kWaitLimitNs;
    const cudaError_t e = gdn::launch_swa(L, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : cuda_fail(e);
}

}  // extern "C"
