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
// Layout: one CTA of NW warps per (sequence, head).  A row of d_k fp32 is
// split over LPR = d_k / 16 lanes, 16 floats each, held as four 16-byte
// pieces.  With COAL the lanes of a row take consecutive 16-byte pieces, so
// each load instruction of a row covers whole 128-byte lines; otherwise a
// lane owns 64 contiguous bytes.  UNR passes (of 32 / LPR rows per warp) are
// loaded before any is consumed, so each thread keeps UNR x 64 bytes of loads
// in flight.
#include "gdn_internal.h"

namespace gdn {
namespace {

// column of the e-th float (e = 4 i + j) that lane `seg` owns
template <int LPR, bool COAL>
__device__ __forceinline__ int col_of(int seg, int i) {
    return COAL ? (i * LPR + seg) * 4 : seg * 16 + 4 * i;
}

template <typename T, int LPR, bool COAL>
__device__ __forceinline__ void load_vec(const T *p, int seg, float (&x)[16]);

template <>
__device__ __forceinline__ void load_vec<float, 8, true>(const float *p, int seg, float (&x)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(p + col_of<8, true>(seg, i)));
        x[4 * i] = t.x; x[4 * i + 1] = t.y; x[4 * i + 2] = t.z; x[4 * i + 3] = t.w;
    }
}

template <typename T, int LPR, bool COAL>
__device__ __forceinline__ void load_vec(const T *p, int seg, float (&x)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int c = col_of<LPR, COAL>(seg, i);
#pragma unroll
        for (int j = 0; j < 4; ++j) x[4 * i + j] = to_f32(p[c + j]);
    }
}

template <typename T, int D, int UNR, int NW, bool COAL>
__global__ void __launch_bounds__(NW * 32)
gdn_decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                  const float *__restrict__ g, const float *__restrict__ beta,
                  const float *state_in, float *state_out, T *__restrict__ out) {
    constexpr int LPR = D / 16;           // lanes per row
    constexpr int RPW = 32 / LPR;         // rows per warp per pass
    constexpr int RPP = RPW * NW;         // rows per CTA per pass
    constexpr int PASSES = D / RPP;
    static_assert(PASSES % UNR == 0, "UNR must divide the pass count");

    const int bh = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = lane % LPR, rloc = lane / LPR;

    float kr[16], qr[16];
    load_vec<T, LPR, COAL>(k + (size_t)bh * D, seg, kr);
    load_vec<T, LPR, COAL>(q + (size_t)bh * D, seg, qr);
    float kq = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) kq = fmaf(kr[j], qr[j], kq);
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
    const float a = expf(__ldg(g + bh));
    const float b = __ldg(beta + bh);

    const size_t sbase = (size_t)bh * D * D;
    const float *Sin = state_in + sbase;
    float *Sout = state_out + sbase;

#pragma unroll 1
    for (int p0 = 0; p0 < PASSES; p0 += UNR) {
        float4 s[UNR][4];
        float vr[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int row = (p0 + u) * RPP + warp * RPW + rloc;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                s[u][i] = *reinterpret_cast<const float4 *>(Sin + (size_t)row * D + col_of<LPR, COAL>(seg, i));
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
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float4 t;
                t.x = fmaf(a, s[u][i].x, uu * kr[4 * i]);
                t.y = fmaf(a, s[u][i].y, uu * kr[4 * i + 1]);
                t.z = fmaf(a, s[u][i].z, uu * kr[4 * i + 2]);
                t.w = fmaf(a, s[u][i].w, uu * kr[4 * i + 3]);
                *reinterpret_cast<float4 *>(Sout + (size_t)row * D + col_of<LPR, COAL>(seg, i)) = t;
            }
            if (seg == 0) out[(size_t)bh * D + row] = from_f32<T>(fmaf(a, sq, uu * kq));
        }
    }
}

}  // namespace

template <typename T, int D, int UNR, int NW, bool COAL>
static cudaError_t launch_decode_v(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *state_in, float *state_out,
                                   void *out, int B, int H, cudaStream_t stream) {
    const unsigned grid = (unsigned)B * (unsigned)H;
    gdn_decode_kernel<T, D, UNR, NW, COAL><<<grid, NW * 32, 0, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), g, beta,
        state_in, state_out, static_cast<T *>(out));
    return cudaGetLastError();
}

cudaError_t launch_decode(int dtype, int dk, const void *q, const void *k, const void *v,
                          const float *g, const float *beta, const float *state_in,
                          float *state_out, void *out, int B, int H, cudaStream_t stream) {
#define GDN_DEC(T, D, U, W, C) \
    return launch_decode_v<T, D, U, W, C>(q, k, v, g, beta, state_in, state_out, out, B, H, stream)
    // from a sweep on B200 (64 sequences x 16 heads, L2 flushed): coalesced
    // 128-byte row pieces, 8 warps, 4 passes in flight
    if (dtype == 0) {
        if (dk == 128) GDN_DEC(float, 128, 4, 8, true);
        GDN_DEC(float, 64, 2, 4, true);
    }
    if (dk == 128) GDN_DEC(__nv_bfloat16, 128, 4, 8, true);
    GDN_DEC(__nv_bfloat16, 64, 2, 4, true);
#undef GDN_DEC
}

}  // namespace gdn
