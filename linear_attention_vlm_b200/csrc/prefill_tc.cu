// Fused chunkwise Gated DeltaNet prefill on the sm_100a tensor cores.
//
// One CTA owns one (sequence, head) and walks its chunks of C = 64 tokens
// with the fp32 d_v x d_k state held in tensor memory.  Per chunk (G =
// cumsum of g inside the chunk, gamma = exp(G), D_t = exp(G_C - G_t)):
//
//   p1   [K;Q] K^T                     -> KK^T (rows 0-63), QK^T (rows 64-127)
//   prep A = strict_lower(beta_r exp(G_r - G_i) k_r.k_i);  T = (I + A)^-1
//        T' = diag(D) T diag(beta gamma),  T'' = diag(D) T diag(beta),
//        Phat = tril(Q K^T)
//   p2   W^T  = K^T T'^T               (W  = D o T diag(beta gamma) K)
//   p3   U^T  = V^T T''^T              (Ut = D o T diag(beta) V)
//   a    U^T -= S W^T                  (U  = D o (Ut - W S^T): the D-scaled residual)
//   c1   O1   = S Q^T
//   b    S   += U^T K                  (S was pre-scaled by gamma_C)
//   c2   O2   = U^T Phat^T
//   out  o_t  = gamma_t O1[:,t] + exp(G_t - G_C) O2[:,t]
//
// which is the token recurrence S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t
// k_t^T, o_t = S_t q_t unrolled over the chunk (the exp(G_t - G_C) factor
// undoes the D factor folded into the shared D-scaled residual operand).  All seven
// products are M = 128 tcgen05 MMAs (bf16 operands in 128-byte-swizzled
// shared memory, fp32 accumulators in TMEM); K, Q, V tiles arrive by TMA.
//
// Warp roles (320 threads):
//   warps 0-3  chain: U / S / O epilogues (thread i <-> TMEM lane i = row i)
//   warps 4-7  prep:  gates, A and Phat from p1, triangular solve, T', T'', W
//   warp  8    MMA issue (one thread) and TMEM allocation
//   warp  9    TMA producer (one thread)
// The prep of chunk n+1 overlaps the state chain of chunk n.
//
// Tokens past the end of a sequence inside its last chunk get g = 0 and
// beta = 0, which zeroes their rows of W and Ut and keeps the state
// untouched; their outputs are not stored.
#include <string.h>

#include "gdn_internal.h"
#include "prefill_tc.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = 64;
constexpr int D = 128;
constexpr int kThreads = 320;
constexpr int AP = 68;   // fp32 row pitch of the solve matrices

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_KQ = 0;                         // [2 stages][2 kb][128 rows][128 B]
constexpr uint32_t OFF_V = OFF_KQ + 2 * 32768;         // [2 kb][64 rows][128 B]
constexpr uint32_t OFF_S = OFF_V + 16384;              // S bf16 [2 kb][128 rows dv][128 B]
constexpr uint32_t OFF_W = OFF_S + 32768;              // W bf16 [2 kb][64 rows t][128 B]
constexpr uint32_t OFF_U = OFF_W + 16384;              // U^T bf16 [128 rows dv][128 B]; output staging
constexpr uint32_t OFF_TP = OFF_U + 16384;             // T'  bf16 [64 rows t][128 B]
constexpr uint32_t OFF_TPP = OFF_TP + 8192;            // T'' bf16 [64][128 B]
constexpr uint32_t OFF_PH = OFF_TPP + 8192;            // Phat bf16 [2 bufs][64][128 B]
constexpr uint32_t OFF_AF = OFF_PH + 16384;            // A fp32 [64][AP]
constexpr uint32_t OFF_TF = OFF_AF + 64 * AP * 4;      // T fp32 [64][AP]
constexpr uint32_t OFF_SCP = OFF_TF + 64 * AP * 4;     // prep scalars: G log2(e), beta, beta gamma, D
constexpr uint32_t OFF_SCE = OFF_SCP + 1024;           // chain scalars [3 bufs]: Dd, gam, invD [64], gC, len
constexpr uint32_t OFF_MM = OFF_SCE + 3072;            // solve scratch: 4 warps x 16x16 fp32
constexpr uint32_t OFF_BAR = OFF_MM + 4096;            // mbarriers, TMEM base, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 256;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;      // + alignment slack

// TMEM columns
constexpr uint32_t TM_C12 = 0;     // p1 output (64 cols)
constexpr uint32_t TM_C3 = 64;     // W^T from p2, then the U^T accumulator (64)
constexpr uint32_t TM_C4 = 128;    // state S (128)
constexpr uint32_t TM_C5 = 256;    // O1 [2 bufs] at 256, 384 (64 each)
constexpr uint32_t TM_C6 = 320;    // O2 [2 bufs] at 320, 448
constexpr uint32_t TM_COLS = 512;

// barrier indices
enum {
    B_FULL_KQ = 0,   // +stage
    B_EMPTY_KQ = 2,  // +stage
    B_FULL_V = 4,
    B_EMPTY_V = 5,
    B_P1 = 6,
    B_P2 = 7,
    B_A = 8,
    B_B = 9,
    B_C = 10,
    B_TREADY = 11,
    B_WREADY = 12,
    B_SREADY = 13,
    B_UREADY = 14,
    B_FIN = 15,
    B_P3 = 16,
    NUM_BARS = 17
};

struct ChainScalars {   // per chunk, chain group
    float Dd[C];        // exp(G_C - G_t)
    float gam[C];       // exp(G_t)
    float invD[C];      // exp(G_t - G_C)
    float gC;           // exp(G_C)
    int len;
    int pad[62];
};
static_assert(sizeof(ChainScalars) == 1024, "scalar block size");

struct PrepScalars {
    float inv[C];       // exp(-G_t) (at most e^80 under the documented gate domain)
    float beta[C];
    float bg[C];        // beta * gamma
    float Dd[C];        // exp(G_C - G_t)
};
static_assert(sizeof(PrepScalars) == 1024, "scalar block size");


__device__ __forceinline__ uint32_t bar_addr(uint8_t *sm, int i) {
    return smem_u32(sm + OFF_BAR + 8 * i);
}

// Raw gates of one chunk held by one warp (lane l owns rows l and l+32),
// loaded an iteration before use so that the global-load latency is hidden.
struct GateRegs {
    float g0, g1, b0, b1;
};

__device__ __forceinline__ GateRegs load_gates(const float *__restrict__ g, const float *__restrict__ beta,
                                               int64_t bos, int64_t eos, int m, int nchunks, int h,
                                               int H, int lane) {
    GateRegs r{0.f, 0.f, 0.f, 0.f};
    if (m < nchunks) {
        const int64_t t0 = bos + (int64_t)m * C;
        const int64_t rem = eos - t0;
        const int len = rem < C ? (int)rem : C;
        if (lane < len) {
            r.g0 = __ldg(g + (size_t)(t0 + lane) * H + h);
            r.b0 = __ldg(beta + (size_t)(t0 + lane) * H + h);
        }
        if (lane + 32 < len) {
            r.g1 = __ldg(g + (size_t)(t0 + lane + 32) * H + h);
            r.b1 = __ldg(beta + (size_t)(t0 + lane + 32) * H + h);
        }
    }
    return r;
}

// Inclusive cumsum of the gates inside the chunk (rows past the end are 0).
__device__ __forceinline__ void scan_gates(const GateRegs &r, int lane, float &G0, float &G1) {
    float x0 = r.g0, x1 = r.g1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, x0, o);
        const float y1 = __shfl_up_sync(0xffffffffu, x1, o);
        if (lane >= o) { x0 += y0; x1 += y1; }
    }
    const float tot0 = __shfl_sync(0xffffffffu, x0, 31);
    G0 = x0;
    G1 = x1 + tot0;
}

// ---------------------------------------------------------------- tf32 mma.sync

__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// acc(16x16) += X(16x16) * Y(16x16); X at (xr, xc), Y at (yr, yc) of fp32
// matrices with row pitch px / py.  acc[nt] holds output columns 8nt..8nt+7.
__device__ __forceinline__ void mma16(float (&acc)[2][4], const float *X, int px, const float *Y,
                                      int py, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = tf32(X[g * px + 8 * ks + t]);
        const uint32_t a1 = tf32(X[(g + 8) * px + 8 * ks + t]);
        const uint32_t a2 = tf32(X[g * px + 8 * ks + t + 4]);
        const uint32_t a3 = tf32(X[(g + 8) * px + 8 * ks + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = tf32(Y[(8 * ks + t) * py + 8 * nt + g]);
            const uint32_t b1 = tf32(Y[(8 * ks + t + 4) * py + 8 * nt + g]);
            mma_tf32(acc[nt], a0, a1, a2, a3, b0, b1);
        }
    }
}

// Off-diagonal block (i, j) of T = (I + A)^-1 (16x16 blocks):
//   T_ij = -T_ii * sum_{k=j}^{i-1} A_ik T_kj
// computed by one warp with tf32 tensor-core MMAs.
__device__ __forceinline__ void solve_block(const float *Af, float *Tf, float *scratch, int i, int j,
                                            int lane) {
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int k = j; k < i; ++k)
        mma16(acc, Af + (16 * i) * AP + 16 * k, AP, Tf + (16 * k) * AP + 16 * j, AP, lane);
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        scratch[g * 16 + 8 * nt + 2 * t] = acc[nt][0];
        scratch[g * 16 + 8 * nt + 2 * t + 1] = acc[nt][1];
        scratch[(g + 8) * 16 + 8 * nt + 2 * t] = acc[nt][2];
        scratch[(g + 8) * 16 + 8 * nt + 2 * t + 1] = acc[nt][3];
    }
    __syncwarp();
    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    mma16(acc2, Tf + (16 * i) * AP + 16 * i, AP, scratch, 16, lane);
    float *dst = Tf + (16 * i) * AP + 16 * j;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        dst[g * AP + 8 * nt + 2 * t] = -acc2[nt][0];
        dst[g * AP + 8 * nt + 2 * t + 1] = -acc2[nt][1];
        dst[(g + 8) * AP + 8 * nt + 2 * t] = -acc2[nt][2];
        dst[(g + 8) * AP + 8 * nt + 2 * t + 1] = -acc2[nt][3];
    }
    __syncwarp();
}

// ---------------------------------------------------------------- kernel

__global__ void __launch_bounds__(kThreads, 1)
gdn_prefill_tc_kernel(const __grid_constant__ TcParams p) {
    extern __shared__ uint8_t smraw[];
    // align to 1024 B by pointer arithmetic on the __shared__ array itself, so
    // that the compiler keeps shared-space (LDS/STS) addressing for `sm`
    uint8_t *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    uint32_t *tmem_base_ptr = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 8 * NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_BAR + 8 * NUM_BARS + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int H = p.H;
    // heads vary fastest; sequences are visited in the order given by p.order
    const int unit = blockIdx.x;
    const int nseq = p.order ? p.order[unit / H] : unit / H;
    const int h = unit % H;
    int64_t bos, eos;
    SeqBounds{p.cu_seqlens, p.uniform_len}.get(nseq, bos, eos);
    const int nchunks = (int)((eos - bos + C - 1) / C);
    const size_t state_off = ((size_t)nseq * H + h) * D * D;

    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) {
            uint32_t cnt = 1;
            if (i == B_TREADY || i == B_WREADY || i == B_SREADY || i == B_UREADY) cnt = 128;
            mbar_init(bar_addr(sm, i), cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(tmem_base_ptr), TM_COLS);
        tmem_relinquish();
    }
    if (warp == 9 && lane == 0) {
        tma_prefetch_desc(&p.map_k);
        tma_prefetch_desc(&p.map_q);
        tma_prefetch_desc(&p.map_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_base_ptr;
    const uint64_t lim = p.timeout_ns;

    auto fail = [&](int code) {
        *abort_flag = 1;
        if (p.err) atomicCAS(p.err, 0, code);
    };

    if (nchunks == 0) {
        // empty sequence: the state passes through unchanged
        if (tid < 128 && p.state_out) {
            for (int j = 0; j < D; j += 4) {
                float4 v = p.state_in ? *reinterpret_cast<const float4 *>(p.state_in + state_off + (size_t)tid * D + j)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4 *>(p.state_out + state_off + (size_t)tid * D + j) = v;
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued_kq[2] = {0, 0}, issued_v = 0;
            for (int n = 0; n < nchunks; ++n) {
                const int s = n & 1;
                const int z = (int)(bos + (int64_t)n * C);
                if (n >= 2 && !mbar_wait(bar_addr(sm, B_EMPTY_KQ + s), ((n - 2) >> 1) & 1, lim, abort_flag)) { fail(11); break; }
                mbar_arrive_expect_tx(bar_addr(sm, B_FULL_KQ + s), 32768);
                for (int kb = 0; kb < 2; ++kb) {
                    const uint32_t dst = smem_u32(sm + OFF_KQ + s * 32768 + kb * 16384);
                    tma_load_3d(dst, &p.map_k, kb * 64, h, z, bar_addr(sm, B_FULL_KQ + s));
                    tma_load_3d(dst + 8192, &p.map_q, kb * 64, h, z, bar_addr(sm, B_FULL_KQ + s));
                }
                ++issued_kq[s];
                if (n >= 1 && !mbar_wait(bar_addr(sm, B_EMPTY_V), (n - 1) & 1, lim, abort_flag)) { fail(12); break; }
                mbar_arrive_expect_tx(bar_addr(sm, B_FULL_V), 16384);
                for (int kb = 0; kb < 2; ++kb)
                    tma_load_3d(smem_u32(sm + OFF_V + kb * 8192), &p.map_v, kb * 64, h, z, bar_addr(sm, B_FULL_V));
                ++issued_v;
            }
            // no copy may still be landing in shared memory when the CTA exits
            const int zero = 0;
            for (int s = 0; s < 2; ++s)
                if (issued_kq[s]) mbar_wait(bar_addr(sm, B_FULL_KQ + s), (issued_kq[s] - 1) & 1, lim, &zero);
            if (issued_v) mbar_wait(bar_addr(sm, B_FULL_V), (issued_v - 1) & 1, lim, &zero);
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_p1 = idesc_bf16(128, 64, false, false);
            const uint32_t id_p2 = idesc_bf16(128, 64, true, false);
            const uint32_t id_a = idesc_bf16(128, 64, false, false, true);
            const uint32_t id_c1 = idesc_bf16(128, 64, false, false);
            const uint32_t id_b = idesc_bf16(128, 128, false, true);
            const uint32_t sKQ = smem_u32(sm + OFF_KQ), sV = smem_u32(sm + OFF_V);  // tile bases
            const uint32_t sS = smem_u32(sm + OFF_S), sW = smem_u32(sm + OFF_W);
            const uint32_t sU = smem_u32(sm + OFF_U), sTP = smem_u32(sm + OFF_TP);
            const uint32_t sTPP = smem_u32(sm + OFF_TPP), sPH = smem_u32(sm + OFF_PH);
            // descriptors are built once; a byte offset `o` inside a tile adds o >> 4
            const uint64_t dKQk = desc_sw128(sKQ, 16, 1024);         // K-major views
            const uint64_t dKQm = desc_sw128(sKQ, 16384, 1024);      // MN-major view of K
            const uint64_t dVm = desc_sw128(sV, 8192, 1024);
            const uint64_t dS = desc_sw128(sS, 16, 1024), dW = desc_sw128(sW, 16, 1024);
            const uint64_t dU = desc_sw128(sU, 16, 1024), dTP = desc_sw128(sTP, 16, 1024);
            const uint64_t dTPP = desc_sw128(sTPP, 16, 1024), dPH = desc_sw128(sPH, 16, 1024);
            auto issue_p1 = [&](int n) {
                const uint32_t base = (n & 1) * 32768;
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t a = dKQk + ((base + (ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
                    mma_bf16_ss(tm + TM_C12, a, a, id_p1, ks > 0);
                }
            };
            bool ok = mbar_wait(bar_addr(sm, B_FULL_KQ), 0, lim, abort_flag);
            if (!ok) fail(21);
            else {
                tc_fence_after();
                issue_p1(0);
                mma_commit(bar_addr(sm, B_P1));
            }
            for (int n = 0; ok && n < nchunks; ++n) {
                const int s = n & 1;
                const uint32_t kq = s * 32768;   // stage offset inside the KQ buffer
                if (!(ok = mbar_wait(bar_addr(sm, B_TREADY), n & 1, lim, abort_flag))) { fail(22); break; }
                tc_fence_after();
                // p2: W^T = K^T T'^T into the U^T columns (A = K tile MN-major; B = T')
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tm + TM_C3, dKQm + ((kq + ks * 2048) >> 4), dTP + ((ks * 32) >> 4),
                                id_p2, ks > 0);
                mma_commit(bar_addr(sm, B_P2));
                // p1 of the next chunk as early as possible: the prep group has
                // already consumed this chunk's p1 output
                if (n + 1 < nchunks) {
                    if (!(ok = mbar_wait(bar_addr(sm, B_FULL_KQ + ((n + 1) & 1)), ((n + 1) >> 1) & 1, lim, abort_flag))) { fail(26); break; }
                    tc_fence_after();
                    issue_p1(n + 1);
                    mma_commit(bar_addr(sm, B_P1));
                }
                if (!(ok = mbar_wait(bar_addr(sm, B_WREADY), n & 1, lim, abort_flag))) { fail(24); break; }
                if (!(ok = mbar_wait(bar_addr(sm, B_FULL_V), n & 1, lim, abort_flag))) { fail(23); break; }
                tc_fence_after();
                // p3: U^T = V^T T''^T (overwrites the extracted W^T)
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tm + TM_C3, dVm + ((ks * 2048) >> 4), dTPP + ((ks * 32) >> 4), id_p2,
                                ks > 0);
                mma_commit(bar_addr(sm, B_P3));
                mma_commit(bar_addr(sm, B_EMPTY_V));
                if (!(ok = mbar_wait(bar_addr(sm, B_SREADY), n & 1, lim, abort_flag))) { fail(25); break; }
                tc_fence_after();
                // a: U^T -= S W^T
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    const uint32_t offw = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_bf16_ss(tm + TM_C3, dS + (off >> 4), dW + (offw >> 4), id_a, 1);
                }
                mma_commit(bar_addr(sm, B_A));
                // c1: O1 = S Q^T  (B = Q rows of the KQ tile); off the state chain
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_bf16_ss(tm + TM_C5 + s * 128, dS + (off >> 4), dKQk + ((kq + off + 8192) >> 4),
                                id_c1, ks > 0);
                }
                if (!(ok = mbar_wait(bar_addr(sm, B_UREADY), n & 1, lim, abort_flag))) { fail(27); break; }
                tc_fence_after();
                // b: S += U^T K   (A = U tile K-major; B = K tile MN-major)
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tm + TM_C4, dU + ((ks * 32) >> 4), dKQm + ((kq + ks * 2048) >> 4), id_b, 1);
                mma_commit(bar_addr(sm, B_B));
                // c2: O2 = U^T Phat^T
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tm + TM_C6 + s * 128, dU + ((ks * 32) >> 4),
                                dPH + ((s * 8192 + ks * 32) >> 4), id_c1, ks > 0);
                mma_commit(bar_addr(sm, B_C));
                mma_commit(bar_addr(sm, B_EMPTY_KQ + s));
            }
            // drain: every issued MMA completes before TMEM is released
            mma_commit(bar_addr(sm, B_FIN));
            if (!mbar_wait(bar_addr(sm, B_FIN), 0, lim, abort_flag)) {
                // one more bounded wait that ignores the abort flag
                const int zero = 0;
                mbar_wait(bar_addr(sm, B_FIN), 0, lim, &zero);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ prep group
        const int pt = tid - 128, pw = warp - 4;
        PrepScalars *sc = reinterpret_cast<PrepScalars *>(sm + OFF_SCP);
        float *Af = reinterpret_cast<float *>(sm + OFF_AF);
        float *Tf = reinterpret_cast<float *>(sm + OFF_TF);
        float *mm = reinterpret_cast<float *>(sm + OFF_MM) + pw * 256;
        const uint32_t lane_off = static_cast<uint32_t>(pw * 32) << 16;
        GateRegs gr{0.f, 0.f, 0.f, 0.f};
        if (pw == 0) gr = load_gates(p.g, p.beta, bos, eos, 0, nchunks, h, H, lane);
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            if (named_bar_any(1, 128, *abort_flag != 0)) break;
            if (pw == 0) {
                float G0, G1;
                scan_gates(gr, lane, G0, G1);
                const float b0 = gr.b0, b1 = gr.b1;
                gr = load_gates(p.g, p.beta, bos, eos, n + 1, nchunks, h, H, lane);
                const float GC = __shfl_sync(0xffffffffu, G1, 31);
                sc->inv[lane] = expf(-G0); sc->inv[lane + 32] = expf(-G1);
                sc->beta[lane] = b0; sc->beta[lane + 32] = b1;
                sc->bg[lane] = b0 * expf(G0); sc->bg[lane + 32] = b1 * expf(G1);
                sc->Dd[lane] = expf(GC - G0); sc->Dd[lane + 32] = expf(GC - G1);
            }
            named_bar_sync(1, 128);
            // A (strictly lower, decayed, beta-scaled) and Phat from p1
            if (!mbar_wait(bar_addr(sm, B_P1), n & 1, lim, abort_flag)) fail(31);
            tc_fence_after();
            {
                float x[64];
                float (&x0)[32] = *reinterpret_cast<float (*)[32]>(&x[0]);
                float (&x1)[32] = *reinterpret_cast<float (*)[32]>(&x[32]);
                tmem_ld32(tm + lane_off + TM_C12, x0);
                tmem_ld32(tm + lane_off + TM_C12 + 32, x1);
                if (pt < 64) {
                    // A[r][i] = beta_r exp(G_r - G_i) k_r.k_i = (beta_r gamma_r) exp(-G_i) KK[r][i]
                    const int r = pt;
                    const float bgr = sc->bg[r];
#pragma unroll
                    for (int i = 0; i < 64; i += 4) {
                        const float4 iv = *reinterpret_cast<const float4 *>(&sc->inv[i]);
                        float4 a;
                        a.x = (i < r) ? bgr * iv.x * x[i] : 0.f;
                        a.y = (i + 1 < r) ? bgr * iv.y * x[i + 1] : 0.f;
                        a.z = (i + 2 < r) ? bgr * iv.z * x[i + 2] : 0.f;
                        a.w = (i + 3 < r) ? bgr * iv.w * x[i + 3] : 0.f;
                        *reinterpret_cast<float4 *>(&Af[r * AP + i]) = a;
                    }
                } else {
                    const int r = pt - 64;
                    const uint32_t row = smem_u32(sm + OFF_PH + s * 8192);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i0 = 8 * c + 2 * e;
                            w[e] = pack_bf16(i0 <= r ? x[i0] : 0.f, i0 + 1 <= r ? x[i0 + 1] : 0.f);
                        }
                        st_shared_v4(row + sw128_chunk(r, c), w[0], w[1], w[2], w[3]);
                    }
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            // T = (I + A)^-1: 16x16 diagonal blocks by forward substitution ...
            if (pt < 64) {
                const int b = pt >> 4, c = pt & 15;
                const float *Ab = Af + (16 * b) * AP + 16 * b;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < r; ++i) ps[i & 3] = fmaf(Ab[r * AP + i], x[i], ps[i & 3]);
                    x[r] = ((r == c) ? 1.f : 0.f) - ((ps[0] + ps[1]) + (ps[2] + ps[3]));
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) Tf[(16 * b + r) * AP + 16 * b + c] = x[r];
            } else {
                // zero the blocks above the diagonal
                for (int e = pt - 64; e < 6 * 256; e += 64) {
                    const int blk = e >> 8, w = e & 255;
                    const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                    const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                    Tf[(16 * bi + (w >> 4)) * AP + 16 * bj + (w & 15)] = 0.f;
                }
            }
            named_bar_sync(1, 128);
            // ... then the off-diagonal blocks, one band at a time
            if (pw < 3) solve_block(Af, Tf, mm, pw + 1, pw, lane);
            named_bar_sync(1, 128);
            if (pw < 2) solve_block(Af, Tf, mm, pw + 2, pw, lane);
            named_bar_sync(1, 128);
            if (pw == 0) solve_block(Af, Tf, mm, 3, 0, lane);
            named_bar_sync(1, 128);
            // T'' of the previous chunk may still be feeding its p3
            if (n > 0 && !mbar_wait(bar_addr(sm, B_P3), (n - 1) & 1, lim, abort_flag)) fail(33);
            // T' = diag(D) T diag(beta gamma), T'' = diag(D) T diag(beta), bf16, K-major rows t
            {
                const int which = pt >> 6, r = pt & 63;
                const uint32_t row = smem_u32(sm + (which ? OFF_TPP : OFF_TP));
                const float *colscale = which ? sc->beta : sc->bg;
                const float dr = sc->Dd[r];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 t0v = *reinterpret_cast<const float4 *>(&Tf[r * AP + 8 * c]);
                    const float4 t1v = *reinterpret_cast<const float4 *>(&Tf[r * AP + 8 * c + 4]);
                    const float4 s0v = *reinterpret_cast<const float4 *>(&colscale[8 * c]);
                    const float4 s1v = *reinterpret_cast<const float4 *>(&colscale[8 * c + 4]);
                    st_shared_v4(row + sw128_chunk(r, c),
                                 pack_bf16(dr * t0v.x * s0v.x, dr * t0v.y * s0v.y),
                                 pack_bf16(dr * t0v.z * s0v.z, dr * t0v.w * s0v.w),
                                 pack_bf16(dr * t1v.x * s1v.x, dr * t1v.y * s1v.y),
                                 pack_bf16(dr * t1v.z * s1v.z, dr * t1v.w * s1v.w));
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(bar_addr(sm, B_TREADY));
            // W from p2's W^T (TMEM lane = d_k index, column = t), in the U^T columns
            if (!mbar_wait(bar_addr(sm, B_P2), n & 1, lim, abort_flag)) fail(32);
            tc_fence_after();
            {
                float x[32];
                uint8_t *wt = sm + OFF_W + (pt >> 6) * 8192;
                const int col = pt & 63;
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tm + lane_off + TM_C3 + 32 * half, x);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        *reinterpret_cast<__nv_bfloat16 *>(wt + sw128_offset(32 * half + i, col)) =
                            __float2bfloat16_rn(x[i]);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            mbar_arrive(bar_addr(sm, B_WREADY));
        }
    } else {
        // ------------------------------------------------------------ chain group
        const int dv = tid;   // TMEM lane and state row
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        ChainScalars *scb = reinterpret_cast<ChainScalars *>(sm + OFF_SCE);
        GateRegs gr{0.f, 0.f, 0.f, 0.f};
        if (warp == 0) gr = load_gates(p.g, p.beta, bos, eos, 0, nchunks, h, H, lane);
        // scalars of chunk m from the prefetched gates; prefetch chunk m+1's
        auto compute_scalars = [&](int m) {
            if (warp == 0) {
                const int64_t t0 = bos + (int64_t)m * C;
                const int len = (int)((eos - t0) < C ? (eos - t0) : C);
                float G0, G1;
                scan_gates(gr, lane, G0, G1);
                gr = load_gates(p.g, p.beta, bos, eos, m + 1, nchunks, h, H, lane);
                const float GC = __shfl_sync(0xffffffffu, G1, 31);
                ChainScalars &cs = scb[m % 3];
                cs.Dd[lane] = expf(GC - G0); cs.Dd[lane + 32] = expf(GC - G1);
                cs.gam[lane] = expf(G0); cs.gam[lane + 32] = expf(G1);
                cs.invD[lane] = expf(G0 - GC); cs.invD[lane + 32] = expf(G1 - GC);
                if (lane == 0) { cs.gC = expf(GC); cs.len = len; }
            }
        };
        // write S (fp32 row dv, 32 columns starting at c0) as bf16 into the A tile
        auto store_s_bf16 = [&](const float (&x)[32], int c0) {
            const uint32_t base = smem_u32(sm + OFF_S + (c0 >> 6) * 16384);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const int chunk = ((c0 & 63) >> 3) + q4;
                st_shared_v4(base + sw128_chunk(dv, chunk), pack_bf16(x[8 * q4], x[8 * q4 + 1]),
                             pack_bf16(x[8 * q4 + 2], x[8 * q4 + 3]), pack_bf16(x[8 * q4 + 4], x[8 * q4 + 5]),
                             pack_bf16(x[8 * q4 + 6], x[8 * q4 + 7]));
            }
        };
        compute_scalars(0);
        named_bar_sync(2, 128);
        {
            const float gC0 = scb[0].gC;
            float x[32];
            for (int c0 = 0; c0 < D; c0 += 32) {
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 v = p.state_in ? *reinterpret_cast<const float4 *>(p.state_in + state_off + (size_t)dv * D + c0 + j)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                    x[j] = v.x; x[j + 1] = v.y; x[j + 2] = v.z; x[j + 3] = v.w;
                }
                store_s_bf16(x, c0);
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] *= gC0;
                tmem_st32(tm + lane_off + TM_C4 + c0, x);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_addr(sm, B_SREADY));
        }
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            // ring of three: warp 0 may write chunk n+1's scalars while a
            // slower warp still reads chunk n-1's in its output epilogue
            const ChainScalars &cs = scb[n % 3];
            // U epilogue: the D-scaled residual U^T -> U tile (row dv, 64 t)
            if (!mbar_wait(bar_addr(sm, B_A), n & 1, lim, abort_flag)) fail(41);
            tc_fence_after();
            {
                const uint32_t row = smem_u32(sm + OFF_U);
                float x[32];
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tm + lane_off + TM_C3 + 32 * half, x);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        st_shared_v4(row + sw128_chunk(dv, 4 * half + q4),
                                     pack_bf16(x[8 * q4], x[8 * q4 + 1]), pack_bf16(x[8 * q4 + 2], x[8 * q4 + 3]),
                                     pack_bf16(x[8 * q4 + 4], x[8 * q4 + 5]), pack_bf16(x[8 * q4 + 6], x[8 * q4 + 7]));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_addr(sm, B_UREADY));
            const bool last = (n + 1 == nchunks);
            if (!last) compute_scalars(n + 1);
            if (named_bar_any(2, 128, *abort_flag != 0)) break;
            // S epilogue
            if (!mbar_wait(bar_addr(sm, B_B), n & 1, lim, abort_flag)) fail(42);
            tc_fence_after();
            {
                float x[32];
                for (int c0 = 0; c0 < D; c0 += 32) {
                    tmem_ld32(tm + lane_off + TM_C4 + c0, x);
                    if (!last) {
                        store_s_bf16(x, c0);
                    } else if (p.state_out) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(p.state_out + state_off + (size_t)dv * D + c0 + j) =
                                make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                if (!last) {
                    // the next (a) may start now; rescale the fp32 state for the
                    // next (b), which the MMA thread issues only after U_READY
                    mbar_arrive(bar_addr(sm, B_SREADY));
                    const float gnext = scb[(n + 1) % 3].gC;
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        tmem_ld32(tm + lane_off + TM_C4 + c0, x);
#pragma unroll
                        for (int j = 0; j < 32; ++j) x[j] *= gnext;
                        tmem_st32(tm + lane_off + TM_C4 + c0, x);
                    }
                    tc_fence_before();
                }
            }
            // O epilogue: o_t = gamma_t O1 + exp(G_t - G_C) O2
            if (!mbar_wait(bar_addr(sm, B_C), n & 1, lim, abort_flag)) fail(43);
            tc_fence_after();
            {
                // stage the [64 t][128 dv] bf16 tile in the U buffer (free once
                // c2 has completed), then write whole 16-byte pieces of rows
                __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_U);
                float a[32], b[32];
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tm + lane_off + TM_C5 + s * 128 + 32 * half, a);
                    tmem_ld32(tm + lane_off + TM_C6 + s * 128 + 32 * half, b);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int t = 32 * half + j;
                        stage[t * D + dv] = __float2bfloat16_rn(fmaf(cs.gam[t], a[j], cs.invD[t] * b[j]));
                    }
                }
                tc_fence_before();
                named_bar_sync(2, 128);
                const int64_t t0 = bos + (int64_t)n * C;
                const int len = cs.len;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int idx = k * 128 + dv;          // 1024 pieces of 16 bytes
                    const int t = idx >> 4, piece = idx & 15;
                    if (t < len) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(stage + t * D + piece * 8);
                        *reinterpret_cast<uint4 *>(p.out + ((size_t)(t0 + t) * H + h) * D + piece * 8) = v;
                    }
                }
                named_bar_sync(2, 128);   // the U buffer is rewritten by the next U epilogue
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tm, TM_COLS);
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// [T, H, 128] bf16 viewed as 3-D (d, H, T); box (64, 1, 64), 128-byte swizzle.
bool make_token_map(CUtensorMap *m, const void *base, int64_t T, int H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)(T > 0 ? T : 1)};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_tc_smem_bytes() { return SMEM_ALLOC; }

cudaError_t launch_prefill_tc(const TcLaunch &L, cudaStream_t stream) {
    TcParams p;
    memset(&p, 0, sizeof(p));
    if (!make_token_map(&p.map_q, L.q, L.total_tokens, L.H) ||
        !make_token_map(&p.map_k, L.k, L.total_tokens, L.H) ||
        !make_token_map(&p.map_v, L.v, L.total_tokens, L.H))
        return cudaErrorInvalidValue;
    p.g = L.g;
    p.beta = L.beta;
    p.state_in = L.state_in;
    p.state_out = L.state_out;
    p.out = static_cast<__nv_bfloat16 *>(L.out);
    p.cu_seqlens = L.cu_seqlens;
    p.uniform_len = L.uniform_len;
    p.order = L.order;
    p.H = L.H;
    p.err = L.err;
    p.timeout_ns = L.timeout_ns;
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gdn_prefill_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    const unsigned grid = (unsigned)L.num_seqs * (unsigned)L.H;
    gdn_prefill_tc_kernel<<<grid, kThreads, SMEM_ALLOC, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
