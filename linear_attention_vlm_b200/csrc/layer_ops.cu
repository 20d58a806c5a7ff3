// The layer steps around the Gated DeltaNet recurrence (explainer page,
// "Step 2: Process tokens with Hybrid Blocks": every Gated DeltaNet layer
// has a 1-D convolution of window 4 and an output gate).
//
// gdn_preprocess_kernel: per (token, head), from the raw projections
//   y_X = act( sum_{i=0..3} w_X[c][i] x_X[t - 3 + i] )     X in {q, k, v},
//         causal, depthwise, restarted at each sequence start (earlier
//         positions come from the carried convolution state, else zero)
//   q = y_q / sqrt(|y_q|^2 + eps),  k likewise,  v = y_v
//   g = log(sigmoid(a)),  beta = sigmoid(b)
// A CTA stages the raw inputs of 64 tokens (+3 before them) of one head in
// shared memory, so every input is read from HBM once with all loads in
// flight together; lanes own d/32 consecutive channels, and the L2 norms are
// warp reductions.
// gdn_conv_state_kernel writes the convolution state after each sequence
// (the raw inputs at its last three positions); it runs after the main
// kernel, so the state may be updated in place.
// gdn_output_gate_kernel: y = n(o) * act(z) per (token, head), n the identity
// or an RMS norm over d_v with per-channel weights, act sigmoid or SiLU; one
// warp per (token, head).
// All three are HBM-bound streaming kernels.
#include "gdn_internal.h"

namespace gdn {
namespace {

template <typename T, int CPL>
__device__ __forceinline__ void load_ch(const T *p, float (&x)[CPL]) {
#pragma unroll
    for (int j = 0; j < CPL; ++j) x[j] = to_f32(p[j]);
}

template <>
__device__ __forceinline__ void load_ch<__nv_bfloat16, 4>(const __nv_bfloat16 *p, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}

template <>
__device__ __forceinline__ void load_ch<float, 4>(const float *p, float (&x)[4]) {
    const float4 u = *reinterpret_cast<const float4 *>(p);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
}

template <typename T, int CPL>
__device__ __forceinline__ void store_ch(T *p, const float (&x)[CPL]) {
#pragma unroll
    for (int j = 0; j < CPL; ++j) p[j] = from_f32<T>(x[j]);
}

template <>
__device__ __forceinline__ void store_ch<__nv_bfloat16, 4>(__nv_bfloat16 *p, const float (&x)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t *>(&a);
    u.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}

template <>
__device__ __forceinline__ void store_ch<float, 4>(float *p, const float (&x)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}

__device__ __forceinline__ float warp_sum(float s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Sequence n containing token t: the last n with bos(n) <= t (empty sequences
// share their start with the next one and are skipped that way).
__device__ __forceinline__ int seq_of(const SeqBounds &sb, int N, int64_t t) {
    if (!sb.cu) return (int)(t / sb.uniform_len);
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sb.cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

constexpr int kPreTokensPerWarp = 8;
constexpr int kPreWarps = 8;
constexpr int kPreTokens = kPreTokensPerWarp * kPreWarps;   // tokens per CTA
constexpr int kPreWin = kPreTokens + 3;                      // staged positions

template <typename T, int D>
constexpr size_t preprocess_smem() {
    return (size_t)3 * kPreWin * D * sizeof(T) + (size_t)3 * D * 4 * sizeof(float);
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(reinterpret_cast<uint64_t>(src))
                 : "memory");
}

template <typename T>
__device__ __forceinline__ const T *pick3(int X, const T *a, const T *b, const T *c) {
    return X == 0 ? a : (X == 1 ? b : c);
}

// One CTA per (64 tokens, head).  The raw inputs of positions t0-3 .. t0+63
// and the head's convolution weights are staged in shared memory with 16-byte
// loads (all in flight at once); then warp w computes tokens t0+8w .. +7, each
// lane d/32 consecutive channels.
template <typename T, int D>
__global__ void __launch_bounds__(kPreWarps * 32)
gdn_preprocess_kernel(const T *__restrict__ xq, const T *__restrict__ xk, const T *__restrict__ xv,
                      const float *__restrict__ conv_w, const float *__restrict__ a_logit,
                      const float *__restrict__ b_logit, const T *__restrict__ cs_in,
                      T *__restrict__ q, T *__restrict__ k, T *__restrict__ v, float *__restrict__ g,
                      float *__restrict__ beta, SeqBounds sb, int N, int64_t T_total, int H, int act,
                      float eps) {
    constexpr int CPL = D / 32;
    constexpr int VEC = 16 / (int)sizeof(T), PIECES = D / VEC;
    extern __shared__ __align__(16) uint8_t smraw[];
    T *xs = reinterpret_cast<T *>(smraw);                                   // [3][kPreWin][D]
    float *ws = reinterpret_cast<float *>(smraw + (size_t)3 * kPreWin * D * sizeof(T));   // [3][D][4]
    const int h = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * kPreTokens;
    const size_t row = (size_t)H * D;   // elements per token of one tensor

    // asynchronous 16-byte copies: every piece of the tile is in flight at once
    for (int i = threadIdx.x; i < 3 * kPreWin * PIECES; i += blockDim.x) {
        const int X = i / (kPreWin * PIECES), rem = i % (kPreWin * PIECES), r = rem / PIECES, pc = rem % PIECES;
        const int64_t p = t0 - 3 + r;
        if (p >= 0 && p < T_total)   // other rows are never read
            cp_async16(xs + ((size_t)X * kPreWin + r) * D + pc * VEC,
                       pick3(X, xq, xk, xv) + (size_t)p * row + (size_t)h * D + pc * VEC);
    }
    for (int i = threadIdx.x; i < 3 * D; i += blockDim.x) {
        const int X = i / D, c = i % D;
        cp_async16(ws + 4 * i, conv_w + (((size_t)X * H + h) * D + c) * 4);
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    const int64_t tb = t0 + warp * kPreTokensPerWarp;
    if (tb >= T_total) return;
    const int nt = (int)(tb + kPreTokensPerWarp < T_total ? kPreTokensPerWarp : T_total - tb);
    const int c0 = lane * CPL;
    float w[3][CPL][4];   // this lane's taps, held for all of its tokens
#pragma unroll
    for (int X = 0; X < 3; ++X)
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const float4 t4 = *reinterpret_cast<const float4 *>(ws + (X * D + c0 + j) * 4);
            w[X][j][0] = t4.x; w[X][j][1] = t4.y; w[X][j][2] = t4.z; w[X][j][3] = t4.w;
        }
    int n = seq_of(sb, N, tb);
    int64_t bos, eos;
    sb.get(n, bos, eos);
    if (nt == kPreTokensPerWarp && tb - 3 >= bos && tb + kPreTokensPerWarp <= eos) {
        // Fast path: all 8 tokens and their 3 predecessors lie in one sequence.
        // One tensor at a time, the lane holds the 11 staged rows of its
        // channels and forms the 8 outputs from them (each row read once).
        const int lr0 = (int)(tb - t0);   // staged row of position tb - 3
#pragma unroll
        for (int X = 0; X < 3; ++X) {
            float xr[kPreTokensPerWarp + 3][CPL];
#pragma unroll
            for (int r = 0; r < kPreTokensPerWarp + 3; ++r)
                load_ch<T, CPL>(xs + (X * kPreWin + lr0 + r) * D + c0, xr[r]);
            float yv[kPreTokensPerWarp][CPL];
#pragma unroll
            for (int u = 0; u < kPreTokensPerWarp; ++u)
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    float a = w[X][j][0] * xr[u][j];
                    a = fmaf(w[X][j][1], xr[u + 1][j], a);
                    a = fmaf(w[X][j][2], xr[u + 2][j], a);
                    a = fmaf(w[X][j][3], xr[u + 3][j], a);
                    yv[u][j] = act ? silu_io<T>(a) : a;
                }
            if (X < 2) {   // L2 norm per token: 8 independent warp reductions
                float ss[kPreTokensPerWarp];
#pragma unroll
                for (int u = 0; u < kPreTokensPerWarp; ++u) {
                    ss[u] = 0.f;
#pragma unroll
                    for (int j = 0; j < CPL; ++j) ss[u] = fmaf(yv[u][j], yv[u][j], ss[u]);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                    for (int u = 0; u < kPreTokensPerWarp; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
#pragma unroll
                for (int u = 0; u < kPreTokensPerWarp; ++u) {
                    const float rn = rsqrtf(ss[u] + eps);
#pragma unroll
                    for (int j = 0; j < CPL; ++j) yv[u][j] *= rn;
                }
            }
            T *dst = (X == 0 ? q : (X == 1 ? k : v)) + (size_t)tb * row + (size_t)h * D + c0;
#pragma unroll
            for (int u = 0; u < kPreTokensPerWarp; ++u) store_ch<T, CPL>(dst + (size_t)u * row, yv[u]);
        }
    } else
    for (int it = 0; it < nt; ++it) {
        const int64_t t = tb + it;
        while (t >= eos) {   // the next non-empty sequence starts at t
            ++n;
            sb.get(n, bos, eos);
        }
        const int lr = (int)(t - t0);                                   // staged row of t is lr + 3
        const int inseq = (int)(t - bos < 3 ? t - bos : 3);             // taps 3 - inseq .. 3 are in the sequence
        float y[3][CPL];
#pragma unroll
        for (int X = 0; X < 3; ++X) {
#pragma unroll
            for (int j = 0; j < CPL; ++j) y[X][j] = 0.f;
            if (inseq == 3) {   // warp-uniform: every tap from the staged tile
                const T *src = xs + (X * kPreWin + lr) * D + c0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float xv4[CPL];
                    load_ch<T, CPL>(src + i * D, xv4);
#pragma unroll
                    for (int j = 0; j < CPL; ++j) y[X][j] = fmaf(w[X][j][i], xv4[j], y[X][j]);
                }
            } else {            // the first three tokens of a sequence
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float xv4[CPL];
                    if (i + inseq >= 3) {
                        load_ch<T, CPL>(xs + (X * kPreWin + lr + i) * D + c0, xv4);
                    } else if (cs_in) {
                        load_ch<T, CPL>(cs_in + (((size_t)n * 3 + (i + inseq)) * 3 + X) * row + (size_t)h * D + c0,
                                        xv4);
                    } else {
#pragma unroll
                        for (int j = 0; j < CPL; ++j) xv4[j] = 0.f;
                    }
#pragma unroll
                    for (int j = 0; j < CPL; ++j) y[X][j] = fmaf(w[X][j][i], xv4[j], y[X][j]);
                }
            }
            if (act) {
#pragma unroll
                for (int j = 0; j < CPL; ++j) y[X][j] = silu_io<T>(y[X][j]);
            }
        }
        float ss[2] = {0.f, 0.f};
#pragma unroll
        for (int X = 0; X < 2; ++X)
#pragma unroll
            for (int j = 0; j < CPL; ++j) ss[X] = fmaf(y[X][j], y[X][j], ss[X]);
#pragma unroll
        for (int X = 0; X < 2; ++X) {
            const float r = rsqrtf(warp_sum(ss[X]) + eps);
#pragma unroll
            for (int j = 0; j < CPL; ++j) y[X][j] *= r;
        }
        const size_t o = (size_t)t * row + (size_t)h * D + c0;
        store_ch<T, CPL>(q + o, y[0]);
        store_ch<T, CPL>(k + o, y[1]);
        store_ch<T, CPL>(v + o, y[2]);
    }
    if (lane < nt) {   // gates: one token per lane
        const size_t i = (size_t)(tb + lane) * H + h;
        g[i] = log_sigmoid_f(a_logit[i]);
        beta[i] = sigmoid_f(b_logit[i]);
    }
}

// state_out[n][s] = raw inputs at position eos - 3 + s (from the carried state
// when that position precedes the sequence).  Each thread owns one
// (tensor, head, channel) and reads all three values before writing any.
template <typename T>
__global__ void __launch_bounds__(256)
gdn_conv_state_kernel(const T *__restrict__ xq, const T *__restrict__ xk, const T *__restrict__ xv,
                      const T *cs_in, T *cs_out, SeqBounds sb, int H, int D) {
    const int n = blockIdx.x;
    int64_t bos, eos;
    sb.get(n, bos, eos);
    const int hd = H * D;
    for (int i = blockIdx.y * blockDim.x + threadIdx.x; i < 3 * hd; i += gridDim.y * blockDim.x) {
        const int X = i / hd, c = i % hd;
        const T *x = pick3(X, xq, xk, xv);
        T val[3];
#pragma unroll
        for (int s = 0; s < 3; ++s) {
            const int64_t p = eos - 3 + s;
            if (p >= bos) val[s] = x[(size_t)p * hd + c];
            else if (cs_in) val[s] = cs_in[(((size_t)n * 3 + (p - bos + 3)) * 3 + X) * hd + c];
            else val[s] = from_f32<T>(0.f);
        }
#pragma unroll
        for (int s = 0; s < 3; ++s) cs_out[(((size_t)n * 3 + s) * 3 + X) * hd + c] = val[s];
    }
}

constexpr int kGateWarps = 8;
constexpr int kGateRowsPerWarp = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kGateWarps * 32)
gdn_output_gate_kernel(const T *__restrict__ o, const T *__restrict__ z, const float *__restrict__ norm_w,
                       T *__restrict__ y, int64_t rows, int gate, float eps) {
    constexpr int CPL = D / 32;
    const int64_t r0 = ((int64_t)blockIdx.x * kGateWarps + (threadIdx.x >> 5)) * kGateRowsPerWarp;
    if (r0 >= rows) return;
    const int lane = threadIdx.x & 31, c0 = lane * CPL;
    float wn[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) wn[j] = norm_w ? norm_w[c0 + j] : 1.f;
    // all rows' loads first, so that they are in flight together
    float ov[kGateRowsPerWarp][CPL], zv[kGateRowsPerWarp][CPL];
#pragma unroll
    for (int rr = 0; rr < kGateRowsPerWarp; ++rr) {
        const int64_t r = r0 + rr;
        if (r < rows) {
            load_ch<T, CPL>(o + (size_t)r * D + c0, ov[rr]);
            load_ch<T, CPL>(z + (size_t)r * D + c0, zv[rr]);
        }
    }
#pragma unroll
    for (int rr = 0; rr < kGateRowsPerWarp; ++rr) {
        const int64_t r = r0 + rr;
        if (r >= rows) break;   // warp-uniform
        float sc = 1.f;
        if (norm_w) {
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < CPL; ++j) ss = fmaf(ov[rr][j], ov[rr][j], ss);
            sc = rsqrtf(warp_sum(ss) * (1.f / D) + eps);
        }
        float res[CPL];
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const float s = sigmoid_io<T>(zv[rr][j]);
            res[j] = ov[rr][j] * sc * wn[j] * (gate ? zv[rr][j] * s : s);
        }
        store_ch<T, CPL>(y + (size_t)r * D + c0, res);
    }
}

// One-time per device: the dynamic shared-memory limit of the kernel.
template <typename T, int D>
cudaError_t preprocess_attr() {
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaError_t ea = cudaGetDevice(&dev);
    if (ea != cudaSuccess) return ea;
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        ea = cudaFuncSetAttribute(gdn_preprocess_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)preprocess_smem<T, D>());
        if (ea != cudaSuccess) return ea;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    return cudaSuccess;
}

template <typename T, int D>
cudaError_t launch_preprocess_t(const PreprocessArgs &A, cudaStream_t stream) {
    const cudaError_t ea = preprocess_attr<T, D>();
    if (ea != cudaSuccess) return ea;
    const SeqBounds sb{A.cu_seqlens, A.cu_seqlens ? 0 : A.total_tokens / A.num_seqs};
    cudaError_t e = cudaSuccess;
    if (A.total_tokens > 0) {
    const dim3 grid((unsigned)((A.total_tokens + kPreTokens - 1) / kPreTokens), (unsigned)A.H);
    gdn_preprocess_kernel<T, D><<<grid, kPreWarps * 32, preprocess_smem<T, D>(), stream>>>(
        static_cast<const T *>(A.xq), static_cast<const T *>(A.xk), static_cast<const T *>(A.xv), A.conv_w,
        A.a_logit, A.b_logit, static_cast<const T *>(A.cs_in), static_cast<T *>(A.q), static_cast<T *>(A.k),
        static_cast<T *>(A.v), A.g, A.beta, sb, A.num_seqs, A.total_tokens, A.H, A.activation, A.eps);
    e = cudaGetLastError();
    }
    if (e != cudaSuccess || !A.cs_out) return e;
    return launch_conv_state(A.dtype, D, A.xq, A.xk, A.xv, A.cs_in, A.cs_out, A.cu_seqlens, A.num_seqs,
                             A.total_tokens, A.H, stream);
}

template <typename T, int D>
cudaError_t launch_gate_t(const void *o, const void *z, const float *norm_w, void *y, int64_t rows, int gate,
                          float eps, cudaStream_t stream) {
    const int64_t per_cta = (int64_t)kGateWarps * kGateRowsPerWarp;
    const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
    gdn_output_gate_kernel<T, D><<<grid, kGateWarps * 32, 0, stream>>>(
        static_cast<const T *>(o), static_cast<const T *>(z), norm_w, static_cast<T *>(y), rows, gate, eps);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_conv_state_t(int d, const void *xq, const void *xk, const void *xv, const void *cs_in, void *cs_out,
                                const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens, int H,
                                cudaStream_t stream) {
    const SeqBounds sb{cu_seqlens, cu_seqlens ? 0 : total_tokens / num_seqs};
    const int work = 3 * H * d;
    const dim3 sgrid((unsigned)num_seqs, (unsigned)((work + 255) / 256));
    gdn_conv_state_kernel<T><<<sgrid, 256, 0, stream>>>(
        static_cast<const T *>(xq), static_cast<const T *>(xk), static_cast<const T *>(xv),
        static_cast<const T *>(cs_in), static_cast<T *>(cs_out), sb, H, d);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv_state(int dtype, int d, const void *xq, const void *xk, const void *xv, const void *cs_in,
                              void *cs_out, const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens, int H,
                              cudaStream_t stream) {
    return dtype == 1 ? launch_conv_state_t<__nv_bfloat16>(d, xq, xk, xv, cs_in, cs_out, cu_seqlens, num_seqs,
                                                           total_tokens, H, stream)
                      : launch_conv_state_t<float>(d, xq, xk, xv, cs_in, cs_out, cu_seqlens, num_seqs,
                                                   total_tokens, H, stream);
}

cudaError_t launch_preprocess(const PreprocessArgs &A, cudaStream_t stream) {
    if (A.dtype == 1) return A.d == 128 ? launch_preprocess_t<__nv_bfloat16, 128>(A, stream)
                                        : launch_preprocess_t<__nv_bfloat16, 64>(A, stream);
    return A.d == 128 ? launch_preprocess_t<float, 128>(A, stream) : launch_preprocess_t<float, 64>(A, stream);
}

cudaError_t layer_ops_setup(int dtype, int d) {
    if (dtype == 1) return d == 128 ? preprocess_attr<__nv_bfloat16, 128>() : preprocess_attr<__nv_bfloat16, 64>();
    return d == 128 ? preprocess_attr<float, 128>() : preprocess_attr<float, 64>();
}

cudaError_t launch_output_gate(int dtype, int dv, const void *o, const void *z, const float *norm_w, void *y,
                               int64_t rows, int gate, float eps, cudaStream_t stream) {
    if (dtype == 1) return dv == 128 ? launch_gate_t<__nv_bfloat16, 128>(o, z, norm_w, y, rows, gate, eps, stream)
                                     : launch_gate_t<__nv_bfloat16, 64>(o, z, norm_w, y, rows, gate, eps, stream);
    return dv == 128 ? launch_gate_t<float, 128>(o, z, norm_w, y, rows, gate, eps, stream)
                     : launch_gate_t<float, 64>(o, z, norm_w, y, rows, gate, eps, stream);
}

}  // namespace gdn
