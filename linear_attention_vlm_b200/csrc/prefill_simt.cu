// Chunkwise Gated DeltaNet prefill in plain fp32 SIMT arithmetic.
//
// This is the fp32 path (fp32 inputs and outputs, accurate to ~1e-6 relative)
// and the path for shapes the tensor-core kernels do not cover.  One CTA owns
// a slice of DVS rows of one head's d_v x d_k state and walks its sequence
// chunk by chunk; the chunk-local factors are recomputed by every slice.
//
// Chunk algebra (chunk of C tokens, start state S0, G = cumsum(g) inside the
// chunk, gamma_r = exp(G_r), Gam_ri = exp(G_r - G_i) for i <= r):
//   A  = strict_lower(diag(beta) (K K^T o Gam))
//   (I + A) W  = diag(beta gamma) K       -> W   (forward substitution)
//   (I + A) Ut = diag(beta) V             -> Ut
//   U  = Ut - W S0^T
//   O  = diag(gamma) Q S0^T + tril(Q K^T o Gam) U
//   S  = gamma_C S0 + U^T diag(exp(G_C - G)) K
// which is the token recurrence S_t = a_t S_{t-1} (I - b_t k_t k_t^T) +
// b_t v_t k_t^T, o_t = S_t q_t unrolled over the chunk.  Tokens past the end
// of a sequence are given k = q = v = 0, g = 0 and beta = 0, which leaves the
// state untouched, so a partial last chunk needs no other special case.
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;

template <int DK, int DVS>
struct SimtSmem {
    static constexpr int C = kChunk;
    static constexpr int KP = DK + 1;   // padded rows: conflict-free column walks
    static constexpr int CP = C + 1;
    static constexpr int kFloats = 3 * C * KP + DVS * KP + C * DVS + 2 * C * CP + 4 * C;
    static constexpr size_t kBytes = sizeof(float) * (size_t)kFloats;
};

template <typename T, int DK, int DV, int DVS>
__global__ void __launch_bounds__(kThreads)
gdn_prefill_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                        const float *__restrict__ g, const float *__restrict__ beta,
                        const float *state_in, T *__restrict__ out, float *state_out,
                        SeqBounds seqs, int H) {
    using L = SimtSmem<DK, DVS>;
    constexpr int C = L::C, KP = L::KP, CP = L::CP;
    extern __shared__ float sm[];
    float *Ks = sm;                 // [C][KP]
    float *Qs = Ks + C * KP;        // [C][KP]
    float *Ws = Qs + C * KP;        // [C][KP]
    float *Ss = Ws + C * KP;        // [DVS][KP]   state slice, rows v0..v0+DVS
    float *Vs = Ss + DVS * KP;      // [C][DVS]    V slice -> Ut -> U (in place)
    float *As = Vs + C * DVS;       // [C][CP]
    float *Ps = As + C * CP;        // [C][CP]
    float *Gs = Ps + C * CP;        // [C] cumulative log gate
    float *Bs = Gs + C;             // [C] beta
    float *gam = Bs + C;            // [C] exp(G_r)
    float *dec = gam + C;           // [C] exp(G_last - G_r)

    const int tid = threadIdx.x;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int v0 = blockIdx.y * DVS;
    int64_t bos, eos;
    seqs.get(n, bos, eos);
    const size_t sbase = (((size_t)n * H + h) * DV + v0) * DK;

    for (int idx = tid; idx < DVS * DK; idx += kThreads) {
        const int c = idx / DK, j = idx % DK;
        Ss[c * KP + j] = state_in ? state_in[sbase + (size_t)c * DK + j] : 0.f;
    }

    for (int64_t t0 = bos; t0 < eos; t0 += C) {
        const int len = (eos - t0 < C) ? (int)(eos - t0) : C;
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int r = idx / DK, j = idx % DK;
            float kv = 0.f, qv = 0.f;
            if (r < len) {
                const size_t off = ((size_t)(t0 + r) * H + h) * DK + j;
                kv = to_f32(k[off]);
                qv = to_f32(q[off]);
            }
            Ks[r * KP + j] = kv;
            Qs[r * KP + j] = qv;
        }
        for (int idx = tid; idx < C * DVS; idx += kThreads) {
            const int r = idx / DVS, c = idx % DVS;
            Vs[idx] = r < len ? to_f32(v[((size_t)(t0 + r) * H + h) * DV + v0 + c]) : 0.f;
        }
        if (tid < C) {
            const bool ok = tid < len;
            Gs[tid] = ok ? g[(size_t)(t0 + tid) * H + h] : 0.f;
            Bs[tid] = ok ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
        }
        __syncthreads();
        if (tid == 0) {
            float acc = 0.f;
            for (int r = 0; r < C; ++r) { acc += Gs[r]; Gs[r] = acc; }
        }
        __syncthreads();
        if (tid < C) {
            gam[tid] = expf(Gs[tid]);
            dec[tid] = expf(Gs[C - 1] - Gs[tid]);
        }
        // A (strictly lower) and P (lower incl. diagonal)
        for (int idx = tid; idx < C * C; idx += kThreads) {
            const int r = idx / C, i = idx % C;
            float a = 0.f, p = 0.f;
            if (i <= r) {
                float kk = 0.f, qk = 0.f;
#pragma unroll 8
                for (int j = 0; j < DK; ++j) {
                    const float ki = Ks[i * KP + j];
                    kk = fmaf(Ks[r * KP + j], ki, kk);
                    qk = fmaf(Qs[r * KP + j], ki, qk);
                }
                const float d = expf(Gs[r] - Gs[i]);
                if (i < r) a = Bs[r] * d * kk;
                p = d * qk;
            }
            As[r * CP + i] = a;
            Ps[r * CP + i] = p;
        }
        __syncthreads();
        // Forward substitution, one column per thread: W (DK columns), Ut (DVS columns).
        for (int col = tid; col < DK + DVS; col += kThreads) {
            if (col < DK) {
                for (int r = 0; r < C; ++r) {
                    float acc = Bs[r] * gam[r] * Ks[r * KP + col];
                    for (int i = 0; i < r; ++i) acc = fmaf(-As[r * CP + i], Ws[i * KP + col], acc);
                    Ws[r * KP + col] = acc;
                }
            } else {
                const int c = col - DK;
                for (int r = 0; r < C; ++r) {
                    float acc = Bs[r] * Vs[r * DVS + c];
                    for (int i = 0; i < r; ++i) acc = fmaf(-As[r * CP + i], Vs[i * DVS + c], acc);
                    Vs[r * DVS + c] = acc;
                }
            }
        }
        __syncthreads();
        // U = Ut - W S0^T
        for (int idx = tid; idx < C * DVS; idx += kThreads) {
            const int r = idx / DVS, c = idx % DVS;
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < DK; ++j) acc = fmaf(Ws[r * KP + j], Ss[c * KP + j], acc);
            Vs[idx] -= acc;
        }
        __syncthreads();
        // O = diag(gamma) Q S0^T + P U
        for (int idx = tid; idx < C * DVS; idx += kThreads) {
            const int r = idx / DVS, c = idx % DVS;
            if (r < len) {
                float acc = 0.f;
#pragma unroll 8
                for (int j = 0; j < DK; ++j) acc = fmaf(Qs[r * KP + j], Ss[c * KP + j], acc);
                acc *= gam[r];
                for (int i = 0; i <= r; ++i) acc = fmaf(Ps[r * CP + i], Vs[i * DVS + c], acc);
                out[((size_t)(t0 + r) * H + h) * DV + v0 + c] = from_f32<T>(acc);
            }
        }
        __syncthreads();
        // S = gamma_C S0 + U^T diag(dec) K
        const float gC = gam[C - 1];
        for (int idx = tid; idx < DVS * DK; idx += kThreads) {
            const int c = idx / DK, j = idx % DK;
            float acc = 0.f;
#pragma unroll 8
            for (int r = 0; r < C; ++r) acc = fmaf(dec[r] * Vs[r * DVS + c], Ks[r * KP + j], acc);
            Ss[c * KP + j] = fmaf(gC, Ss[c * KP + j], acc);
        }
    }
    __syncthreads();
    if (state_out) {
        for (int idx = tid; idx < DVS * DK; idx += kThreads) {
            const int c = idx / DK, j = idx % DK;
            state_out[sbase + (size_t)c * DK + j] = Ss[c * KP + j];
        }
    }
}

template <typename T, int D>
cudaError_t launch_t(const void *q, const void *k, const void *v, const float *g,
                     const float *beta, const float *state_in, void *out, float *state_out,
                     const int32_t *cu, int64_t uniform_len, int num_seqs, int H,
                     cudaStream_t stream) {
    constexpr int DVS = 32;
    auto kern = gdn_prefill_simt_kernel<T, D, D, DVS>;
    const size_t smem = SimtSmem<D, DVS>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)num_seqs * (unsigned)H, D / DVS);
    kern<<<grid, kThreads, smem, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), g, beta,
        state_in, static_cast<T *>(out), state_out, SeqBounds{cu, uniform_len}, H);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(int dtype, int dk, const void *q, const void *k,
                                const void *v, const float *g, const float *beta,
                                const float *state_in, void *out, float *state_out,
                                const int32_t *cu_seqlens, int64_t uniform_len,
                                int num_seqs, int H, cudaStream_t stream) {
    if (dtype == 0)
        return dk == 128 ? launch_t<float, 128>(q, k, v, g, beta, state_in, out, state_out, cu_seqlens, uniform_len, num_seqs, H, stream)
                         : launch_t<float, 64>(q, k, v, g, beta, state_in, out, state_out, cu_seqlens, uniform_len, num_seqs, H, stream);
    return dk == 128
               ? launch_t<__nv_bfloat16, 128>(q, k, v, g, beta, state_in, out, state_out, cu_seqlens, uniform_len, num_seqs, H, stream)
               : launch_t<__nv_bfloat16, 64>(q, k, v, g, beta, state_in, out, state_out, cu_seqlens, uniform_len, num_seqs, H, stream);
}

}  // namespace gdn
