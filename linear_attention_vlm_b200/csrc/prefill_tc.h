// Launch interface of the tensor-core prefill (prefill_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

// Bytes of per-chunk factors the prep kernel hands to the chain kernel for
// one (chunk, head): -W (64 x 128 bf16), T'' (64 x 64 bf16) and the scaled
// QK^T triangle Pt (64 x 64 bf16), already in the 128-byte-swizzled
// shared-memory layout of the MMAs.
constexpr size_t kTileBytes = 32768;

// The layer steps fused into the prefill (gdn_layer_prefill): the prep kernel
// forms q, k, v, g and beta from the raw projections (causal depthwise
// convolution of window 4, optional SiLU, q/k L2 norm, beta = sigmoid(b),
// g = log sigmoid(a)); q, k, v, g and beta go to the buffers below for the
// chain kernels; the output pass writes y = n(o) * act(z) instead of o.
struct TcLayer {
    const void *xq, *xk, *xv;          // raw projections [T, H, 128] bf16
    const float *conv_w;               // [3, H, 128, 4]
    const float *a_logit, *b_logit;    // [T, H]
    const void *cs_in;                 // [N, 3, 3, H, 128] bf16, or null (zeros)
    void *q, *k, *v;                   // processed q (rows scaled by exp(G_t) of their chunk), k, v
                                       // [T, H, 128] bf16 (written)
    float *g, *beta;                   // [T, H] (written)
    int activation;                    // GDN_ACT_NONE / GDN_ACT_SILU
    float eps;                         // of the q/k L2 norm and of the RMS norm
    const void *z;                     // output-gate input [T, H, 128] bf16
    const float *norm_w;               // [128] or null (no RMS norm)
    int gate;                          // GDN_GATE_SIGMOID / GDN_GATE_SILU
};

struct TcLaunch {
    const void *q, *k, *v;
    const float *g, *beta, *state_in;
    void *out;
    float *state_out;
    const int32_t *cu_seqlens;   // null: num_seqs sequences of uniform_len tokens
    int64_t uniform_len, total_tokens;
    int num_seqs, H;
    void *workspace;             // tc_workspace_bytes(...) bytes, 16-byte aligned
    int *err;                    // device status word (0 = ok)
    uint64_t timeout_ns;         // bound on the waits of the kernels' work loops
    uint64_t drain_ns;           // bound on the waits that drain copies and MMAs before exit
    const TcLayer *layer;        // null: plain prefill of q, k, v, g, beta into out
};

// Upper bound on the number of 64-token chunks of a packed batch.
inline int64_t tc_chunk_bound(int num_seqs, int64_t total_tokens, bool varlen) {
    return varlen ? (total_tokens + 63) / 64 + num_seqs : num_seqs * ((total_tokens / num_seqs + 63) / 64);
}

// Sequence-parallel ranges: a batch of few long unpacked sequences is split
// into nseg ranges of chunks per sequence so that about one CTA per SM works
// on it (see the chain kernel); 1 means one range per sequence.
constexpr int kScanMaxSegs = 16;     // ranges per sequence at most
constexpr int kScanMinChunks = 8;    // chunks per range at least
constexpr int kScanRefSMs = 148;     // SM count the workspace is sized for (B200)

inline int tc_scan_segments(int num_seqs, int64_t total_tokens, int H, bool varlen, int sm_count) {
    if (varlen || num_seqs < 1 || H < 1 || total_tokens <= 0) return 1;
    const int64_t units = (int64_t)num_seqs * H;
    if (2 * units > sm_count) return 1;
    const int64_t cps = (total_tokens / num_seqs + 63) / 64;
    int64_t nseg = sm_count / units;
    if (nseg > kScanMaxSegs) nseg = kScanMaxSegs;
    if (nseg > cps / kScanMinChunks) nseg = cps / kScanMinChunks;
    if (nseg < 2) return 1;
    const int64_t len = (cps + nseg - 1) / nseg;
    return (int)((cps + len - 1) / len);    // no empty trailing range
}

// Workspace layout: [status 1 KiB][chunk offsets, 4 (N+1) B, padded to 1 KiB]
// [tiles: chunk_bound * H * kTileBytes][range transitions R, M and range start
// states: 3 x N * H * (nseg - 1) * 64 KiB].
size_t tc_workspace_bytes(int num_seqs, int64_t total_tokens, int H, bool varlen);
int tc_kernel_count(int num_seqs, int64_t total_tokens, int H, bool varlen);
cudaError_t launch_prefill_tc(const TcLaunch &L, cudaStream_t stream);

}  // namespace gdn
