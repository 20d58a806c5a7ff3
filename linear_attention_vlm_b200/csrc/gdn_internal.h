// Internal declarations shared by the libgdn.so translation units.
// Not part of the public ABI (that is include/gdn.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

constexpr int kChunk = 64;   // chunk length of the chunkwise prefill

// Sequence bounds of sequence n: from cu_seqlens if given, else uniform.
struct SeqBounds {
    const int32_t *cu;   // device, may be null
    int64_t uniform_len; // used when cu == null
    __device__ __forceinline__ void get(int n, int64_t &bos, int64_t &eos) const {
        if (cu) {
            bos = cu[n];
            eos = cu[n + 1];
        } else {
            bos = (int64_t)n * uniform_len;
            eos = bos + uniform_len;
        }
    }
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// sigmoid and SiLU with the fast exponential and division intrinsics
// (relative error ~1e-6, far below the bf16 storage step; a huge exp(-x)
// gives 0, the correct limit)
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// The bf16 path's sigmoid and SiLU: sigmoid(x) = (1 + tanh(x / 2)) / 2 with
// tanh on the special-function unit (tanh.approx.f32, relative error about
// 2^-11): one SFU op instead of an exponential and a reciprocal, and an
// absolute error near 2^-12 that the bf16 rounding of the results (2^-9)
// swamps.  The fp32 path keeps sigmoid_f and silu_f.
__device__ __forceinline__ float tanh_sfu(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
    return t;
}
__device__ __forceinline__ float sigmoid_t(float x) { return fmaf(0.5f, tanh_sfu(0.5f * x), 0.5f); }
__device__ __forceinline__ float silu_t(float x) {
    const float h = 0.5f * x;
    return fmaf(h, tanh_sfu(h), h);
}
// the forms for storage type T
template <typename T> __device__ __forceinline__ float sigmoid_io(float x) { return sigmoid_f(x); }
template <> __device__ __forceinline__ float sigmoid_io<__nv_bfloat16>(float x) { return sigmoid_t(x); }
template <typename T> __device__ __forceinline__ float silu_io(float x) { return silu_f(x); }
template <> __device__ __forceinline__ float silu_io<__nv_bfloat16>(float x) { return silu_t(x); }

// log(sigmoid(x)) = min(x, 0) - log1p(exp(-|x|)), without overflow
__device__ __forceinline__ float log_sigmoid_f(float x) { return fminf(x, 0.f) - log1pf(expf(-fabsf(x))); }

// Records e as this host thread's last CUDA error (gdn_last_cuda_error) and
// returns GDN_ERR_CUDA.
int note_cuda_error(cudaError_t e);

// Launchers (return cudaError_t of the launch).
cudaError_t launch_decode(int dtype, int dk, const void *q, const void *k, const void *v,
                          const float *g, const float *beta, const float *state_in,
                          float *state_out, void *out, int B, int H, cudaStream_t stream);

cudaError_t launch_prefill_simt(int dtype, int dk, const void *q, const void *k,
                                const void *v, const float *g, const float *beta,
                                const float *state_in, void *out, float *state_out,
                                const int32_t *cu_seqlens, int64_t uniform_len,
                                int num_seqs, int H, cudaStream_t stream);

// Layer steps around the recurrence (layer_ops.cu).
struct PreprocessArgs {
    const void *xq, *xk, *xv;          // raw projections [T, H, d], dtype
    const float *conv_w;               // [3, H, d, 4]
    const float *a_logit, *b_logit;    // [T, H]
    const void *cs_in;                 // [N, 3, 3, H, d] dtype, or null (zeros)
    void *q, *k, *v;                   // [T, H, d] dtype (written)
    float *g, *beta;                   // [T, H] (written)
    void *cs_out;                      // [N, 3, 3, H, d] dtype, or null
    const int32_t *cu_seqlens;         // [N+1] or null (N equal sequences)
    int num_seqs;
    int64_t total_tokens;
    int H, d, activation, dtype;
    float eps;
};
cudaError_t launch_preprocess(const PreprocessArgs &A, cudaStream_t stream);
// The convolution state after each sequence (the raw inputs at its last three
// positions, older ones from cs_in); reads every value before writing, so
// cs_out may equal cs_in.
cudaError_t launch_conv_state(int dtype, int d, const void *xq, const void *xk, const void *xv, const void *cs_in,
                              void *cs_out, const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens, int H,
                              cudaStream_t stream);
cudaError_t launch_output_gate(int dtype, int dv, const void *o, const void *z, const float *norm_w, void *y,
                               int64_t rows, int gate, float eps, cudaStream_t stream);

// One-time per-device kernel attribute set-up (shared-memory limits), so that
// later launches can be captured into CUDA graphs without it.
cudaError_t prefill_tc_setup();
cudaError_t layer_ops_setup(int dtype, int d);

// Sliding-window attention and RoPE (swa.cu).
struct SwaLaunch {
    const void *q, *k, *v;             // [T, Hq | Hkv | Hkv, 128] bf16
    void *o;                           // [T, Hq, 128] bf16
    const int32_t *cu_seqlens;         // [N+1] or null (N equal sequences)
    int num_seqs;
    int64_t total_tokens;
    int Hq, Hkv, window;
    float scale;
    int *err;                          // device status word, or null
    uint64_t timeout_ns;               // bound on the waits of the kernel's work loops
    uint64_t drain_ns;                 // bound on the waits that drain copies and MMAs before exit
};
cudaError_t launch_swa(const SwaLaunch &L, cudaStream_t stream);
cudaError_t swa_setup();
cudaError_t launch_rope(int dtype, const void *x, void *out, const int32_t *cu_seqlens, int num_seqs,
                        int64_t total_tokens, int H, int d, int offset, double base, cudaStream_t stream);

}  // namespace gdn
