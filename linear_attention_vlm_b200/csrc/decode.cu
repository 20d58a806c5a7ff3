// Recurrent decode step of Gated DeltaNet: one token per sequence.
//
// Per (sequence, head), with a = exp(g), b = beta and the d_v x d_k state S:
//   s_k = S k,  s_q = S q                (row dot products)
//   u   = b (v - a s_k)
//   o   = a s_q + u (k . q)              (= S_new q, read-out after the write)
//   S  <- a S + u k^T
// Every row of S is independent given k and q, so the state is streamed once:
// each row is read, reduced against k and q, updated and written back by the
// same threads (in-place updates are safe).  The kernel is HBM-bound: 2 d_k
// d_v 4 bytes of state traffic against ~6 d_k d_v flops.
//
// Layout: one CTA of 4 warps per (sequence, head).  A row of 128 fp32 is
// split over LPR = d_k / 16 lanes (16 floats = four 128-bit loads each), so a
// warp covers 32 / LPR rows per pass; UNR passes are issued before any is
// consumed so that every thread keeps UNR x 64 bytes of loads in flight.
#include "gdn_internal.h"

namespace gdn {
namespace {

template <typename T>
__device__ __forceinline__ void load16(const T *p, float (&x)[16]);

template <>
__device__ __forceinline__ void load16<float>(const float *p, float (&x)[16]) {
    const float4 *p4 = reinterpret_cast<const float4 *>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float4 t = __ldg(p4 + i);
        x[4 * i] = t.x; x[4 * i + 1] = t.y; x[4 * i + 2] = t.z; x[4 * i + 3] = t.w;
    }
}

template <>
__device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[16]) {
    const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        uint4 t = __ldg(p4 + i);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&t);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float2 f = __bfloat1622float2(h[j]);
            x[8 * i + 2 * j] = f.x;
            x[8 * i + 2 * j + 1] = f.y;
        }
    }
}

template <typename T, int D, int UNR>
__global__ void __launch_bounds__(128)
gdn_decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                  const float *__restrict__ g, const float *__restrict__ beta,
                  const float *state_in, float *state_out, T *__restrict__ out) {
    constexpr int LPR = D / 16;           // lanes per row
    constexpr int RPW = 32 / LPR;         // rows per warp per pass
    constexpr int RPP = RPW * 4;          // rows per CTA per pass
    constexpr int PASSES = D / RPP;
    static_assert(PASSES % UNR == 0, "UNR must divide the pass count");

    const int bh = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = lane % LPR, rloc = lane / LPR;

    float kr[16], qr[16];
    load16<T>(k + (size_t)bh * D + seg * 16, kr);
    load16<T>(q + (size_t)bh * D + seg * 16, qr);
    float kq = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) kq = fmaf(kr[j], qr[j], kq);
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
    const float a = expf(__ldg(g + bh));
    const float b = __ldg(beta + bh);

    const size_t sbase = (size_t)bh * D * D;
    const float4 *Sin = reinterpret_cast<const float4 *>(state_in + sbase);
    float4 *Sout = reinterpret_cast<float4 *>(state_out + sbase);

#pragma unroll 1
    for (int p0 = 0; p0 < PASSES; p0 += UNR) {
        float4 s[UNR][4];
        float vr[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int row = (p0 + u) * RPP + warp * RPW + rloc;
            const float4 *src = Sin + ((size_t)row * D + seg * 16) / 4;
#pragma unroll
            for (int i = 0; i < 4; ++i) s[u][i] = src[i];
            vr[u] = to_f32(v[(size_t)bh * D + row]);
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int row = (p0 + u) * RPP + warp * RPW + rloc;
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sk = fmaf(s[u][i].x, kr[4 * i], sk);
                sk = fmaf(s[u][i].y, kr[4 * i + 1], sk);
                sk = fmaf(s[u][i].z, kr[4 * i + 2], sk);
                sk = fmaf(s[u][i].w, kr[4 * i + 3], sk);
                sq = fmaf(s[u][i].x, qr[4 * i], sq);
                sq = fmaf(s[u][i].y, qr[4 * i + 1], sq);
                sq = fmaf(s[u][i].z, qr[4 * i + 2], sq);
                sq = fmaf(s[u][i].w, qr[4 * i + 3], sq);
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
            }
            const float uu = b * (vr[u] - a * sk);
            float4 *dst = Sout + ((size_t)row * D + seg * 16) / 4;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float4 t;
                t.x = fmaf(a, s[u][i].x, uu * kr[4 * i]);
                t.y = fmaf(a, s[u][i].y, uu * kr[4 * i + 1]);
                t.z = fmaf(a, s[u][i].z, uu * kr[4 * i + 2]);
                t.w = fmaf(a, s[u][i].w, uu * kr[4 * i + 3]);
                dst[i] = t;
            }
            if (seg == 0) out[(size_t)bh * D + row] = from_f32<T>(fmaf(a, sq, uu * kq));
        }
    }
}

template <typename T, int D>
cudaError_t launch_decode_t(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *state_in, float *state_out,
                            void *out, int B, int H, cudaStream_t stream) {
    constexpr int UNR = (D == 128) ? 4 : 2;
    const unsigned grid = (unsigned)B * (unsigned)H;
    gdn_decode_kernel<T, D, UNR><<<grid, 128, 0, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), g, beta,
        state_in, state_out, static_cast<T *>(out));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(int dtype, int dk, const void *q, const void *k, const void *v,
                          const float *g, const float *beta, const float *state_in,
                          float *state_out, void *out, int B, int H, cudaStream_t stream) {
    if (dtype == 0) {
        return dk == 128 ? launch_decode_t<float, 128>(q, k, v, g, beta, state_in, state_out, out, B, H, stream)
                         : launch_decode_t<float, 64>(q, k, v, g, beta, state_in, state_out, out, B, H, stream);
    }
    return dk == 128
               ? launch_decode_t<__nv_bfloat16, 128>(q, k, v, g, beta, state_in, state_out, out, B, H, stream)
               : launch_decode_t<__nv_bfloat16, 64>(q, k, v, g, beta, state_in, state_out, out, B, H, stream);
}

}  // namespace gdn
