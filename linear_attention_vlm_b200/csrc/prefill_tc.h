// Launch interface of the tensor-core prefill (prefill_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

// Bytes of per-chunk factors the prep kernel hands to the chain kernel for
// one (chunk, head): W (64 x 128 bf16), diag(gamma) Q (64 x 128 bf16),
// T'' (64 x 64 bf16) and the scaled QK^T triangle (64 x 64 bf16), each already
// in the 128-byte-swizzled shared-memory layout of the MMAs.
constexpr size_t kTileBytes = 49152;

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
    uint64_t timeout_ns;         // bound on every wait inside the kernels
};

// Upper bound on the number of 64-token chunks of a packed batch.
inline int64_t tc_chunk_bound(int num_seqs, int64_t total_tokens, bool varlen) {
    return varlen ? (total_tokens + 63) / 64 + num_seqs : num_seqs * ((total_tokens / num_seqs + 63) / 64);
}

// Workspace layout: [status 256 B][chunk offsets, 4 (N+1) B, padded to 1 KiB]
// [tiles: chunk_bound * H * kTileBytes].
size_t tc_workspace_bytes(int num_seqs, int64_t total_tokens, int H, bool varlen);
int tc_kernel_count(bool varlen);
cudaError_t launch_prefill_tc(const TcLaunch &L, cudaStream_t stream);

}  // namespace gdn
