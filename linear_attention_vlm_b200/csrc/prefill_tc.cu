// Chunkwise Gated DeltaNet prefill on the sm_100a tensor cores, as two
// kernels: a fully parallel chunk-prep kernel and a sequential chain kernel.
//
// Chunk algebra (chunk of C = 64 tokens, start state S, G = cumsum of g inside
// the chunk, gamma = exp(G), D_t = exp(G_C - G_t)):
//
//   A    = strict_lower(beta_r exp(G_r - G_i) k_r.k_i),   T = (I + A)^-1
//   T'   = diag(D) T diag(beta gamma),   T'' = diag(D) T diag(beta)
//   W    = T' K,   Pt = diag(exp(G_t - G_C)) tril(Q K^T)
//   U^T  = V^T T''^T - S W^T           (the D-scaled delta residual)
//   S   <- gamma_C S + U^T K
//   O^T  = (S Q^T) diag(gamma) + U^T Pt^T   (o_t = S_t q_t for every token of the chunk)
//
// which is the token recurrence S_t = a_t S_{t-1}(I - b_t k_t k_t^T) +
// b_t v_t k_t^T, o_t = S_t q_t unrolled over the chunk.
//
// gdn_chunk_prep_kernel: one CTA per (chunk, head), all chunks at once.
//   TMA brings K and Q; p1 = [K; Q] K^T on tcgen05 (TMEM); four warps form A
//   and Pt, invert I + A (16x16 diagonal blocks by substitution, the
//   off-diagonal blocks with tf32 mma.sync), scale T' and T''; p2 = K^T T'^T
//   on tcgen05 gives W.  -W, T'' and Pt (32 KB) are written to the workspace
//   in the 128-byte-swizzled layout the chain kernel's MMAs read, so that it
//   copies them with bulk copies.  Q itself is not rewritten: the chain
//   kernel reads it from the input and applies gamma in its output epilogue.
// gdn_chunk_chain_kernel: one CTA per (sequence, head, chunk range), fp32
//   state in TMEM: p3 U^T = V^T T''^T, (a + c1) [O1^T | U^T] += S [Q; -W]^T
//   as ONE N = 128 MMA, (b) S += U^T K, c2 O2^T = U^T Pt^T -- M = 128
//   tcgen05 MMAs, the S and U^T operands read from TMEM -- with a four-warp
//   state group (residual and state epilogues, the serial chain), a six-warp
//   output group (o_t = gamma_t O1_t + O2_t, off the chain), one MMA thread
//   and one TMA thread.  The state never leaves the SM between chunks.  A
//   tcgen05.mma costs its issuing thread some 60 cycles whatever its width,
//   while an M = 128, N = 64 MMA computes for 32: merging the two MMAs that
//   share the A operand S into one of twice the width removes eight issues
//   per chunk.
//
// Tokens past the end of a sequence inside its last chunk get g = 0 and
// beta = 0, which zeroes their rows of W and T'' and keeps the state
// untouched; their outputs are not stored.
#include <stddef.h>
#include <string.h>

#include "gdn_internal.h"
#include "prefill_tc.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = 64;
constexpr int D = 128;
// ------------------------------------------------------------ prep kernel layout
// 128 threads and ~56 KB of shared memory per CTA, so that four chunks are in
// flight per SM.  Thread 0 also issues the TMA copies and the two MMAs.
constexpr int kPrepThreads = 128;
constexpr uint32_t P_KQ = 0;                           // [2 kb][128 rows: K 0-63, Q 64-127][128 B]
constexpr uint32_t P_TP = P_KQ + 32768;                // T'  bf16 [64 t][128 B]
constexpr uint32_t P_TPP = P_TP + 8192;                // T'' bf16 [64 t][128 B] (p2 reads [T'; T''] as one A)
constexpr uint32_t P_SC = P_TPP + 8192;                // PrepScalars
constexpr uint32_t P_MM = P_SC + 1536;                 // solve scratch, 4 warps x 16 x 20 fp32
constexpr uint32_t P_BAR = P_MM + 4 * 16 * 20 * 4;     // mbarriers + TMEM base
constexpr uint32_t P_ALLOC = P_BAR + 64 + 1008;        // + alignment slack
constexpr uint32_t P_TM_COLS = 128;                    // p1 output at 0..63, then p2 output at 0..127
enum { PB_FULL = 0, PB_P1 = 1, PB_P2 = 2, PB_NUM = 3 };
// The lower block triangles of A and T = (I + A)^-1, as ten 16x16 fp32 blocks
// each (block (i, j), j <= i, at index i (i + 1) / 2 + j).  A lives over the
// T'/T'' buffers (written only after the solve), T over the Q rows of the KQ
// tile (dead once p1 has read them): five blocks in each 8 KB half.
constexpr int AB_P = 20, TB_P = 24;                    // row pitches: conflict-free mma fragment loads
constexpr uint32_t P_AB = P_TP;
// A blocks sit 1296 B apart (324 words, 4 banks of skew) so that the two
// diagonal blocks one warp reads during the substitution fall in different banks
// T blocks sit 1568 B apart (8 banks of skew), so that the blocks of one
// block-row, read side by side when T' and T'' are formed, use different banks
constexpr uint32_t AB_BYTES = 1296, TB_BYTES = 1568;
static_assert(AB_BYTES >= 16 * AB_P * 4 && AB_BYTES % 16 == 0, "A block stride");
static_assert(TB_BYTES >= 16 * TB_P * 4 && TB_BYTES % 16 == 0, "T block stride");
static_assert(10 * AB_BYTES <= 16384 && 5 * TB_BYTES <= 8192, "block triangles fit");
static_assert(4 * (P_ALLOC + 1024) <= 233472, "four prep CTAs per SM");

__device__ __forceinline__ int tri_blk(int i, int j) { return i * (i + 1) / 2 + j; }
__device__ __forceinline__ float *a_blk(uint8_t *sm, int i, int j) {
    return reinterpret_cast<float *>(sm + P_AB + tri_blk(i, j) * AB_BYTES);
}
__device__ __forceinline__ float *t_blk(uint8_t *sm, int i, int j) {
    const int b = tri_blk(i, j);
    return reinterpret_cast<float *>(sm + P_KQ + (b < 5 ? 8192 + b * TB_BYTES : 24576 + (b - 5) * TB_BYTES));
}

// ------------------------------------------------------------ chain kernel layout
// warps 0-3 chain, 4-7 output / chain X, 8 MMA, 9 TMA, 10 MMA of chain X /
// output stores, 11 output stores
constexpr int kChainThreads = 384;
// Stages of the load pipeline.  An output range needs all of a chunk's data
// (K, Q, V and the 32 KB prep tile: two stages of 80 KB); a transition range
// needs K, V, -W and T'' only, and runs three stages of 56 KB so that a
// chunk's loads are issued two chunks ahead.
template <int MODE> struct ChainLayout;
// An output stage keeps K, Q and -W as one K-major operand of 192 rows per
// 64-column block (K rows 0-63, Q 64-127, -W 128-191; blocks KB bytes
// apart): rows 64-191 are the merged MMA's B = [Q; -W], rows 0-63 (as an
// MN-major view) the B of (b).
template <> struct ChainLayout<0> {   // MODE_OUT
    static constexpr int NST = 2;
    static constexpr uint32_t STAGE = 81920;
    static constexpr uint32_t K = 0, KB = 24576, Q = 8192, NEGW = 16384, V = 49152, TPP = 65536, PT = 73728;
    static constexpr uint32_t LOADED = STAGE;
};
template <> struct ChainLayout<1> {   // MODE_TRANS
    static constexpr int NST = 3;
    static constexpr uint32_t STAGE = 57344;
    static constexpr uint32_t K = 0, KB = 8192, V = 16384, W = 32768, TPP = 49152;
    static constexpr uint32_t LOADED = STAGE;
};
static_assert(ChainLayout<0>::PT + 8192 == ChainLayout<0>::STAGE && 2 * ChainLayout<0>::KB == ChainLayout<0>::V,
              "stage layout");
// a tile: -W per 64-column block (8 KB each), T'' (8 KB), Pt (8 KB); a
// transition stage takes its first 24 KB, in that order, after K and V
constexpr uint32_t TILE_NEGW = 0, TILE_TPP = 16384, TILE_PT = 24576;
static_assert(TILE_PT + 8192 == kTileBytes, "tile layout");
static_assert(ChainLayout<1>::TPP + 8192 == ChainLayout<1>::STAGE &&
              ChainLayout<1>::STAGE - ChainLayout<1>::W == TILE_PT, "stage layout");
// After the stages: output staging [64 t][128 dv] bf16, ChainScalars x 3 per
// chain, mbarriers + TMEM base + abort flag.
template <int MODE> __host__ __device__ constexpr uint32_t c_u() { return ChainLayout<MODE>::NST * ChainLayout<MODE>::STAGE; }
// the output stage: [64 t][128 dv] bf16, or fp32 when the output gate is fused (MODE 0, the output pass)
template <int MODE> __host__ __device__ constexpr uint32_t c_sce() { return c_u<MODE>() + (MODE == 0 ? 32768 : 16384); }
template <int MODE> __host__ __device__ constexpr uint32_t c_scx() { return c_sce<MODE>() + 3072; }
template <int MODE> __host__ __device__ constexpr uint32_t c_bar() { return c_scx<MODE>() + 3072; }
template <int MODE> __host__ __device__ constexpr uint32_t c_alloc() { return c_bar<MODE>() + 256 + 1024; }
static_assert(c_alloc<0>() <= 232448 && c_alloc<1>() <= 232448, "chain kernel shared memory");
// TMEM columns of the chain kernel.  The MMA A operands produced by the chain
// itself (bf16 S and bf16 U^T) stay in TMEM: shared-memory bandwidth, not the
// tensor core, bounds these small-N MMAs, so only B is read from shared memory.
// O1^T sits right before U^T, so that the merged MMA writes [O1^T | U^T] as
// one 128-column accumulator.
constexpr uint32_t TM_S = 0;       // state S (128)
constexpr uint32_t TM_O = 128;     // O1^T = S Q^T (64)
constexpr uint32_t TM_U = 192;     // U^T accumulator (64); then U^T bf16 in its first 32
constexpr uint32_t TM_SBF = 256;   // S bf16, two per column (64)
// the identity chain of a transition range: its bf16 copy, U^T and state
constexpr uint32_t TM_XSBF = 128, TM_XU = 320, TM_XS = 384;
constexpr uint32_t TM_O2 = 320;    // an output range: O2^T = U^T Pt^T (64)
constexpr uint32_t TM_COLS = 512;
// Barriers that a role may complete twice before its consumer waits once are
// per buffer (FULL/EMPTY per stage) and waited with
// the parity of the buffer's use count, so that no phase can be skipped.
enum { CB_FULL = 0, CB_EMPTY = 3, CB_A = 6, CB_B = 7, CB_C = 8, CB_SREADY = 10, CB_UREADY = 11,
       CB_FIN = 12, CB_OFREE = 13, CB_A2 = 15, CB_B2 = 16, CB_SREADY2 = 17, CB_UREADY2 = 18,
       CB_FIN2 = 19, CB_NUM = 20 };   // FULL, EMPTY: one per stage (up to 3)
static_assert(8 * CB_NUM + 8 <= 256, "barriers, TMEM base and abort flag fit their block");

struct ChainScalars {   // per chunk, state group
    float gC;           // exp(G_C)
    int len;
    int pad[254];
};
static_assert(sizeof(ChainScalars) == 1024, "scalar block size");

struct PrepScalars {
    float inv[C];       // exp(-G_t) (at most e^80 under the documented gate domain)
    float beta[C];
    float bg[C];        // beta * gamma
    float Dd[C];        // exp(G_C - G_t)
    float invD[C];      // exp(G_t - G_C)
    float gam[C];       // exp(G_t) (layer mode: the q buffer gets diag(gamma) q)
};
static_assert(sizeof(PrepScalars) <= 1536, "scalar block size");

struct PrepParams {
    CUtensorMap map_q, map_k;
    CUtensorMap map_v;           // layer mode: the raw v projection
    const float *g, *beta;
    const int32_t *cu_seqlens;
    const int32_t *chunk_off;    // varlen: first global chunk of each sequence, [N+1]
    int64_t uniform_len;
    int cps;                     // uniform: chunks per sequence
    int num_seqs, H;
    uint8_t *tiles;
    int *err;
    uint64_t timeout_ns;         // bound on the waits of the work loops
    uint64_t drain_ns;           // bound on the waits that drain copies and MMAs before exit
    // layer mode (fused pre-processing; map_q, map_k and map_v then cover the
    // raw projections, and g, beta are unused)
    int keep_tiles;              // all tiles fit in L2 beside the streams: keep them there for the chain passes
    int layer;
    const __nv_bfloat16 *xq, *xk, *xv;     // raw projections (halo rows)
    const float *conv_w, *a_logit, *b_logit;
    const __nv_bfloat16 *cs_in;            // [N, 3, 3, H, 128] or null
    __nv_bfloat16 *q_out, *k_out, *v_out;  // processed q, k, v
    float *g_out, *beta_out;
    int act;
    float eps;
};

struct ChainParams {
    CUtensorMap map_k, map_v, map_q;   // map_q: output ranges only
    const float *g, *beta, *state_in;
    float *state_out;
    __nv_bfloat16 *out;
    const int32_t *cu_seqlens;
    const int32_t *chunk_off;
    int64_t uniform_len;
    int cps;
    int H;
    int nseg, seg_len;           // chunk ranges per sequence, chunks per range
    const uint8_t *tiles;
    const float *seg_start;      // start states of ranges 1.. [N][H][nseg-1][D][D]
    float *trans_r;              // transitions R of ranges 0..nseg-2, same layout
    float *trans_m;              // transitions M, same units; each as bf16 rows [k][n], hi then lo (M = hi + lo)
    int wait_tiles;              // the prep kernel may still run: wait before reading tiles
    int wait_start;              // the combine may still run: wait before reading seg_start
    int *err;
    uint64_t timeout_ns;         // bound on the waits of the work loops
    uint64_t drain_ns;           // bound on the waits that drain copies and MMAs before exit
    int wait_inputs;             // q, k, v, g, beta come from the prep kernel (layer mode): wait first
    int keep_tiles;              // the prep kernel left the tiles in L2 (see PrepParams)
    // output gate in the output epilogue (z null: plain outputs)
    const __nv_bfloat16 *z;
    const float *norm_w;
    int gate;
    float eps;
};

__device__ __forceinline__ uint8_t *aligned_smem(uint8_t *raw) {
    // align by pointer arithmetic on the __shared__ array so that the
    // compiler keeps shared-space (LDS/STS) addressing
    return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

// 1-D bulk copy global -> shared, completion as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// bulk_load with an L2 eviction-priority policy for the lines it reads.
__device__ __forceinline__ void bulk_load_hint(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                               uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

// 1-D bulk copy shared -> global (bulk async-group completion).
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(reinterpret_cast<uint64_t>(dst)), "r"(src), "r"(bytes)
                 : "memory");
}

// bulk_store with an L2 eviction-priority policy for the lines it writes.
__device__ __forceinline__ void bulk_store_hint(void *dst, uint32_t src, uint32_t bytes, uint64_t policy) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;"
                 ::"l"(reinterpret_cast<uint64_t>(dst)), "r"(src), "r"(bytes), "l"(policy)
                 : "memory");
}

// A 16-byte global store with an L2 eviction-priority policy.
__device__ __forceinline__ void st_global_v4_hint(void *dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                                  uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;"
                 ::"l"(reinterpret_cast<uint64_t>(dst)), "r"(a), "r"(b), "r"(c), "r"(d), "l"(policy)
                 : "memory");
}

// Drop a 128-byte line of workspace data that nothing reads again from L2
// without writing it back (its memory contents become indeterminate).
__device__ __forceinline__ void l2_discard_line(const void *p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(reinterpret_cast<uint64_t>(p)) : "memory");
}

// Commit this thread's bulk stores and wait until they have read shared memory.
__device__ __forceinline__ void bulk_commit_wait_read() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
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

// load_gates for g alone, with loads issued where the call stands (a plain
// load may be sunk to its first use, a chunk later, exposing its latency).
__device__ __forceinline__ GateRegs load_gates_pinned(const float *__restrict__ g, int64_t bos, int64_t eos, int m,
                                                      int nchunks, int h, int H, int lane) {
    GateRegs r{0.f, 0.f, 0.f, 0.f};
    if (m < nchunks) {
        const int64_t t0 = bos + (int64_t)m * C;
        const int64_t rem = eos - t0;
        const int len = rem < C ? (int)rem : C;
        if (lane < len)
            asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r.g0) : "l"(g + (size_t)(t0 + lane) * H + h));
        if (lane + 32 < len)
            asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r.g1) : "l"(g + (size_t)(t0 + lane + 32) * H + h));
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

// Store a 16x16 mma accumulator pair (columns 0-7, 8-15) as fp32 rows of
// pitch `pitch`, negated if `neg`.
__device__ __forceinline__ void store16(float *dst, int pitch, const float (&acc)[2][4], bool neg, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const float sg = neg ? -1.f : 1.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2 *>(dst + g * pitch + 8 * nt + 2 * t) = make_float2(sg * acc[nt][0], sg * acc[nt][1]);
        *reinterpret_cast<float2 *>(dst + (g + 8) * pitch + 8 * nt + 2 * t) = make_float2(sg * acc[nt][2], sg * acc[nt][3]);
    }
}

// Off-diagonal blocks of T = (I + A)^-1 from the diagonal ones (16x16 blocks
// b = 0..3), by the 2x2 block-inverse rule applied twice:
//   level 1:  T_10 = -T_11 A_10 T_00,  T_32 = -T_33 A_32 T_22
//   level 2:  X = A_[23][01] T_[01][01]  (the four blocks X_ij, i = 2,3, j = 0,1)
//             T_[23][01] = -T_[23][23] X
// Warp w does its share of each level; the caller separates the levels with
// CTA barriers.  tf32 tensor-core MMAs, fp32 accumulation.
__device__ __forceinline__ void merge_level1(uint8_t *sm, float *scratch, int w, int lane) {
    const int i = 2 * w + 1, j = 2 * w;   // (1, 0) for warp 0, (3, 2) for warp 1
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    mma16(acc, a_blk(sm, i, j), AB_P, t_blk(sm, j, j), TB_P, lane);
    store16(scratch, 20, acc, false, lane);
    __syncwarp();
    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    mma16(acc2, t_blk(sm, i, i), TB_P, scratch, 20, lane);
    store16(t_blk(sm, i, j), TB_P, acc2, true, lane);
}

// X_ij = sum_{k=j}^{1} A_ik T_kj for (i, j) = (2 + (w >> 1), w & 1), into scratch
__device__ __forceinline__ void merge_level2a(uint8_t *sm, float *scratch, int w, int lane) {
    const int i = 2 + (w >> 1), j = w & 1;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int k = j; k < 2; ++k) mma16(acc, a_blk(sm, i, k), AB_P, t_blk(sm, k, j), TB_P, lane);
    store16(scratch, 20, acc, false, lane);
}

// T_ij = -sum_{k=2}^{i} T_ik X_kj; X_kj is in the scratch of warp 2 (k - 2) + j
__device__ __forceinline__ void merge_level2b(uint8_t *sm, float *scratch0, int w, int lane) {
    const int i = 2 + (w >> 1), j = w & 1;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int k = 2; k <= i; ++k) mma16(acc, t_blk(sm, i, k), TB_P, scratch0 + (2 * (k - 2) + j) * 320, 20, lane);
    store16(t_blk(sm, i, j), TB_P, acc, true, lane);
}


// (x, y) -> packed bf16 hi = rn(x, y) and lo = rn(x - hi_x, y - hi_y)
__device__ __forceinline__ void split2(float x, float y, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const float2 hf = __bfloat1622float2(h);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = pack_bf16(x - hf.x, y - hf.y);
}

// ---------------------------------------------------------------- chunk offsets

// chunk_off[n] = sum_{m<n} ceil(L_m / 64) for n = 0..N (one block).
__global__ void __launch_bounds__(1024)
gdn_chunk_offsets_kernel(const int32_t *__restrict__ cu, int N, int32_t *__restrict__ chunk_off) {
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int base = 0; base < N; base += 1024) {
        const int n = base + (int)threadIdx.x;
        const int32_t c = n < N ? (cu[n + 1] - cu[n] + C - 1) / C : 0;
        int32_t x = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int32_t w = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sums[lane] = w;   // inclusive over warps
        }
        __syncthreads();
        const int32_t incl = x + (wid > 0 ? warp_sums[wid - 1] : 0) + carry;
        if (n < N) chunk_off[n + 1] = incl;
        if (base == 0 && threadIdx.x == 0) chunk_off[0] = 0;
        __syncthreads();
        if (threadIdx.x == 1023) carry = incl;
        __syncthreads();
    }
    if (N == 0 && threadIdx.x == 0) chunk_off[0] = 0;
}

// ---------------------------------------------------------------- layer pre-processing
//
// In layer mode (gdn_layer_prefill) the prep kernel forms its own inputs from
// the raw projections of its chunk: the TMA brings the raw q, k tiles into the
// MMA operand slots and the raw v tile into the T' region (idle until the
// solve), the three positions before the chunk come in as halo rows (the
// sequence's previous tokens, the carried convolution state, or zeros), and
//   y = act(sum_i w_i x[t - 3 + i]),   q, k = y / sqrt(|y|^2 + eps),   v = y
// is computed: q and k back into their operand rows, k and v to the
// workspace for the chain kernels, and q to it as diag(gamma) q once the
// gates are scanned (the gated output pass's Q operand).  Thread (tg, ci) owns the 8 tokens 8 tg .. 8 tg + 7
// and the 8 channels 8 ci .. 8 ci + 7 of a tensor; the 16 threads of a token
// row are 16 consecutive lanes, so the L2 norm is a 16-lane butterfly.

// Layer-phase scratch in the scalar block and the solve scratch (both idle
// until the gates are scanned): two 2 KiB buffers of convolution taps, then
// the halo rows.  Taps of channel 8 ci + c sit at float4 slot 16 c + ci, so
// the 16 lanes of a token row read 16 consecutive slots.
constexpr uint32_t P_LW = P_SC;              // taps, 2 x [8 c][16 ci] float4
constexpr uint32_t P_LH = P_SC + 4096;       // halo rows [3 X][3 r][16 pieces] of 16 B
static_assert(P_LH + 2304 <= P_BAR, "layer scratch fits before the barriers");

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// element e (0..7) of a 16-byte piece of 8 bf16
__device__ __forceinline__ float piece_elem(const uint4 &v, int e) {
    const uint32_t w = e < 2 ? v.x : (e < 4 ? v.y : (e < 6 ? v.z : v.w));
    return (e & 1) ? bf16_hi(w) : bf16_lo(w);
}

// shared-memory offset of piece ci (channels 8 ci .. 8 ci + 7) of row r of
// tensor X's tile (X: 0 q, 1 k, 2 v)
__device__ __forceinline__ uint32_t layer_piece_off(int X, int r, int ci) {
    const uint32_t base = X == 2 ? P_TP + (ci >> 3) * 8192 : P_KQ + (ci >> 3) * 16384 + (X == 0 ? 8192 : 0);
    return base + sw128_chunk(r, ci & 7);
}

// the raw row 8 tg - 3 + i (i < 3) of tensor X: from the halo rows for tg = 0
__device__ __forceinline__ void layer_halo(const uint8_t *sm, int X, int tg, int ci, uint4 (&hl)[3]) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int r = 8 * tg - 3 + i;
        hl[i] = r < 0 ? *reinterpret_cast<const uint4 *>(sm + P_LH + ((X * 3 + r + 3) * 16 + ci) * 16)
                      : *reinterpret_cast<const uint4 *>(sm + layer_piece_off(X, r, ci));
    }
}

// Taps of tensor X (2 KiB of head h) -> tap buffer `buf`, 16 bytes per
// thread and piece, asynchronously (cp.async group).
__device__ __forceinline__ void layer_taps_async(const PrepParams &p, uint8_t *sm, int X, int buf, int h, int H,
                                                 int tid) {
    for (int i = tid; i < D; i += kPrepThreads) {   // channel i
        const uint32_t dst = smem_u32(sm + P_LW + buf * 2048 + ((i & 7) * 16 + (i >> 3)) * 16);
        asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(dst),
                     "l"(reinterpret_cast<uint64_t>(p.conv_w + (((size_t)X * H + h) * D + i) * 4))
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// This thread's share of tensor X with the taps in buffer `buf` (rows past
// the sequence end, r >= len, become 0): q and k back into their operand rows,
// k and v to `gout` (the workspace).  Channel-outer, so that each raw value is
// widened once and used by the four outputs it feeds.  One out-of-line copy
// serves the three tensors: unrolled three times inline, the code no longer
// fits the instruction cache next to the rest of the kernel.
__device__ __noinline__ void layer_tensor(uint8_t *sm, int X, int buf, uint4 h0, uint4 h1, uint4 h2, int tg, int ci,
                                          int h, int H, int64_t t0, int len, __nv_bfloat16 *gout, int act, float eps) {
    uint4 raw[11];   // rows 8 tg - 3 .. 8 tg + 7
    raw[0] = h0; raw[1] = h1; raw[2] = h2;
#pragma unroll
    for (int r = 0; r < 8; ++r) raw[3 + r] = *reinterpret_cast<const uint4 *>(sm + layer_piece_off(X, 8 * tg + r, ci));
    const float4 *taps = reinterpret_cast<const float4 *>(sm + P_LW + buf * 2048) + ci;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float y[4][8], ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 w = taps[16 * c];
            float xr[7];
#pragma unroll
            for (int r = 0; r < 7; ++r) xr[r] = piece_elem(raw[4 * half + r], c);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float a = w.x * xr[u];
                a = fmaf(w.y, xr[u + 1], a);
                a = fmaf(w.z, xr[u + 2], a);
                a = fmaf(w.w, xr[u + 3], a);
                a = act ? silu_t(a) : a;
                y[u][c] = a;
                ss[u] = fmaf(a, a, ss[u]);
            }
        }
        if (X < 2) {
#pragma unroll
            for (int o = 1; o < 16; o <<= 1)
#pragma unroll
                for (int u = 0; u < 4; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float rn = rsqrtf(ss[u] + eps);
#pragma unroll
                for (int c = 0; c < 8; ++c) y[u][c] *= rn;
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = 8 * tg + 4 * half + u;
            const bool valid = r < len;
            const uint4 o = valid ? make_uint4(pack_bf16(y[u][0], y[u][1]), pack_bf16(y[u][2], y[u][3]),
                                               pack_bf16(y[u][4], y[u][5]), pack_bf16(y[u][6], y[u][7]))
                                  : make_uint4(0u, 0u, 0u, 0u);
            if (X < 2) *reinterpret_cast<uint4 *>(sm + layer_piece_off(X, r, ci)) = o;
            if (gout && valid) *reinterpret_cast<uint4 *>(gout + ((size_t)(t0 + r) * H + h) * D + 8 * ci) = o;
        }
    }
}

// ---------------------------------------------------------------- prep kernel

template <bool LAYER>
__global__ void __launch_bounds__(kPrepThreads, 4)
gdn_chunk_prep_kernel(const __grid_constant__ PrepParams p) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = aligned_smem(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, h = blockIdx.y;
    const int gc = blockIdx.x;
    grid_dep_launch();   // the next kernel may stage its prologue while this grid drains

    // which sequence and which of its chunks global chunk c is (false: a
    // padding chunk past the last sequence of a packed batch)
    auto locate = [&](int c, int &nseq_, int64_t &j_) {
        if (p.chunk_off) {
            if (c >= p.chunk_off[p.num_seqs]) return false;
            int lo = 0, hi = p.num_seqs - 1;                 // last n with chunk_off[n] <= c
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (p.chunk_off[mid] <= c) lo = mid; else hi = mid - 1;
            }
            nseq_ = lo;
            j_ = c - p.chunk_off[lo];
        } else {
            nseq_ = c / p.cps;
            j_ = c % p.cps;
        }
        return true;
    };
    int nseq;
    int64_t j;
    if (!locate(gc, nseq, j)) return;                        // uniform across the CTA
    int64_t bos, eos;
    SeqBounds{p.cu_seqlens, p.uniform_len}.get(nseq, bos, eos);
    const int64_t t0 = bos + j * C;

    uint32_t *tmem_base_ptr = reinterpret_cast<uint32_t *>(sm + P_BAR + 8 * PB_NUM);
    auto bar = [&](int i) { return smem_u32(sm + P_BAR + 8 * i); };
    if (tid == 0) {
        mbar_init(bar(PB_FULL), 1);
        mbar_init(bar(PB_P1), 1);
        mbar_init(bar(PB_P2), 1);
        fence_mbar_init();
        // K, Q (layer mode: raw k, q and v) -> shared memory, in flight
        // during the TMEM allocation.  L2, when the tiles are kept there: the
        // inputs are streamed (the chain passes read them again far later), so
        // that they do not push out the tiles this CTA writes.
        const int z = (int)t0;
        mbar_arrive_expect_tx(bar(PB_FULL), LAYER ? 49152 : 32768);
        for (int kb = 0; kb < 2; ++kb) {
            const uint32_t dst = smem_u32(sm + P_KQ + kb * 16384);
            if (p.keep_tiles) {
                const uint64_t stream_pol = l2_evict_first_policy();
                tma_load_3d_hint(dst, &p.map_k, kb * 64, h, z, bar(PB_FULL), stream_pol);
                tma_load_3d_hint(dst + 8192, &p.map_q, kb * 64, h, z, bar(PB_FULL), stream_pol);
            } else {
                tma_load_3d(dst, &p.map_k, kb * 64, h, z, bar(PB_FULL));
                tma_load_3d(dst + 8192, &p.map_q, kb * 64, h, z, bar(PB_FULL));
            }
            if (LAYER) tma_load_3d(smem_u32(sm + P_TP + kb * 8192), &p.map_v, kb * 64, h, z, bar(PB_FULL));
        }
    }
    GateRegs lg{0.f, 0.f, 0.f, 0.f};   // layer mode: g, beta of this chunk (warp 1)
    if (LAYER) {
        // halo rows: the raw q, k, v at positions t0 - 3 .. t0 - 1 -> P_MM
        for (int i = tid; i < 3 * 3 * 16; i += kPrepThreads) {
            const int X = i / 48, r = (i / 16) % 3, pc = i & 15;
            const int64_t pos = t0 - 3 + r;
            const __nv_bfloat16 *src = nullptr;
            if (pos >= bos) src = (X == 0 ? p.xq : (X == 1 ? p.xk : p.xv)) + ((size_t)pos * H + h) * D + pc * 8;
            else if (p.cs_in) src = p.cs_in + ((((size_t)nseq * 3 + (pos - bos + 3)) * 3 + X) * H + h) * D + pc * 8;
            *reinterpret_cast<uint4 *>(sm + P_LH + i * 16) =
                src ? __ldg(reinterpret_cast<const uint4 *>(src)) : make_uint4(0u, 0u, 0u, 0u);
        }
        layer_taps_async(p, sm, 1, 0, h, H, tid);   // k's taps -> buffer 0
        layer_taps_async(p, sm, 0, 1, h, H, tid);   // q's taps -> buffer 1
        if (warp == 1) {
            // g = log sigmoid(a), beta = sigmoid(b) for rows lane and lane + 32
            const int len = (int)((eos - t0) < C ? (eos - t0) : C);
            for (int e = 0; e < 2; ++e) {
                const int r = lane + 32 * e;
                if (r < len) {
                    const size_t i = (size_t)(t0 + r) * H + h;
                    const float gv = log_sigmoid_f(__ldg(p.a_logit + i)), bv = sigmoid_f(__ldg(p.b_logit + i));
                    p.g_out[i] = gv;
                    p.beta_out[i] = bv;
                    if (e == 0) { lg.g0 = gv; lg.b0 = bv; } else { lg.g1 = gv; lg.b1 = bv; }
                }
            }
        }
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_base_ptr), P_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_base_ptr;
    const uint64_t lim = p.timeout_ns;
    const int no_abort = 0;   // CTA-local failures end each wait by its own bound
    bool ok = true;
    PrepScalars *sc = reinterpret_cast<PrepScalars *>(sm + P_SC);
    uint8_t *tile = p.tiles + ((size_t)gc * H + h) * kTileBytes;   // [-W 16K][T'' 8K][Pt 8K]
    // the tile stays in L2 for the chain passes when all tiles fit beside the streams
    const uint64_t keep_pol = l2_evict_last_policy();
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    float *mm = reinterpret_cast<float *>(sm + P_MM);          // 4 warps x 16 x 20 fp32

    if (LAYER) {
        ok = mbar_wait(bar(PB_FULL), 0, lim, &no_abort);   // raw tiles landed
        asm volatile("cp.async.wait_all;" ::: "memory");  // this thread's taps
        const int tg = tid >> 4, ci = tid & 15;
        const int len = (int)((eos - t0) < C ? (eos - t0) : C);
        uint4 hl[3];
        // k, then q: every thread reads its halo rows before any rewrites them
        // (the barrier also publishes the taps)
        layer_halo(sm, 1, tg, ci, hl);
        __syncthreads();
        layer_tensor(sm, 1, 0, hl[0], hl[1], hl[2], tg, ci, h, H, t0, len, p.k_out, p.act, p.eps);
        layer_halo(sm, 0, tg, ci, hl);
        __syncthreads();                            // k's taps are read: v's go to buffer 0
        layer_taps_async(p, sm, 2, 0, h, H, tid);
        layer_tensor(sm, 0, 1, hl[0], hl[1], hl[2], tg, ci, h, H, t0, len, nullptr, p.act, p.eps);
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        layer_halo(sm, 2, tg, ci, hl);   // v is read from the T' region and leaves to HBM only
        layer_tensor(sm, 2, 0, hl[0], hl[1], hl[2], tg, ci, h, H, t0, len, p.v_out, p.act, p.eps);
        fence_proxy_async_smem();        // the K and Q rows, written here, are MMA operands
        __syncthreads();
    }

    if (tid == 0) {
        // p1 = [K; Q] K^T -> TMEM columns 0..63: K K^T in lanes 0..63, Q K^T in 64..127
        ok = mbar_wait(bar(PB_FULL), 0, lim, &no_abort);
        if (ok) {
            tc_fence_after();
            const uint64_t dKQk = desc_sw128(smem_u32(sm + P_KQ), 16, 1024);
            const uint32_t id_p1 = idesc_bf16(128, 64, false, false);
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = dKQk + (((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
                mma_bf16_ss(tm, a, a, id_p1, ks > 0);
            }
        }
        mma_commit(bar(PB_P1));   // also on failure, so that no thread waits out its bound
    } else if (warp == 1) {
        const GateRegs gr = LAYER ? lg : load_gates(p.g, p.beta, bos, eos, (int)j, (int)j + 1, h, H, lane);
        float G0, G1;
        scan_gates(gr, lane, G0, G1);
        const float GC = __shfl_sync(0xffffffffu, G1, 31);
        sc->inv[lane] = expf(-G0); sc->inv[lane + 32] = expf(-G1);
        sc->beta[lane] = gr.b0; sc->beta[lane + 32] = gr.b1;
        sc->bg[lane] = gr.b0 * expf(G0); sc->bg[lane + 32] = gr.b1 * expf(G1);
        sc->Dd[lane] = expf(GC - G0); sc->Dd[lane + 32] = expf(GC - G1);
        sc->invD[lane] = expf(G0 - GC); sc->invD[lane + 32] = expf(G1 - GC);
        if (LAYER) { sc->gam[lane] = expf(G0); sc->gam[lane + 32] = expf(G1); }
    }
    __syncwarp();
    __syncthreads();   // gates scanned; K and Q landed (thread 0 waited for them)
    float x[64];       // this lane's row of p1 (rows 64..127: Q K^T, kept for Pt)
    {
        float (&x0)[32] = *reinterpret_cast<float (*)[32]>(&x[0]);
        float (&x1)[32] = *reinterpret_cast<float (*)[32]>(&x[32]);
        ok = mbar_wait(bar(PB_P1), 0, lim, &no_abort) && ok;
        tc_fence_after();
        tmem_ld32(tm + lane_off, x0);
        tmem_ld32(tm + lane_off + 32, x1);
    }
    if (LAYER && tid >= 64) {
        // layer mode: diag(gamma) Q of the sequence's rows to the q buffer, the
        // output pass's Q operand (its gated epilogue then needs no gamma),
        // before T goes over the Q rows.  Thread tid takes the swizzled 16-byte
        // pieces tid - 64 + 64 k: piece pc of row r holds channels
        // 8 (pc ^ (r % 8)) .. + 7 of its 64-channel block.
        const int len = (int)((eos - t0) < C ? (eos - t0) : C);
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
            const int q = (tid - 64) + 64 * k, kb = q >> 9, r = (q >> 3) & 63, pc = q & 7;
            if (r < len) {
                const float gr = sc->gam[r];
                uint4 v = *reinterpret_cast<const uint4 *>(sm + P_KQ + kb * 16384 + 8192 + r * 128 + pc * 16);
                __nv_bfloat162 *hv = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(hv[e]);
                    hv[e] = __floats2bfloat162_rn(gr * f.x, gr * f.y);
                }
                *reinterpret_cast<uint4 *>(p.q_out + ((size_t)(t0 + r) * H + h) * D + kb * 64 + ((pc ^ (r & 7)) << 3)) = v;
            }
        }
    }
    if (tid < 64) {
        // A[r][i] = beta_r exp(G_r - G_i) k_r.k_i = (beta_r gamma_r) exp(-G_i) KK[r][i], i < r
        const int r = tid, rb = r >> 4;
        const float bgr = sc->bg[r];
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
            if (jb > rb) break;
            float *dst = a_blk(sm, rb, jb) + (r & 15) * AB_P;
#pragma unroll
            for (int c = 0; c < 16; c += 4) {
                const int i = 16 * jb + c;
                const float4 iv = *reinterpret_cast<const float4 *>(&sc->inv[i]);
                float4 a;
                a.x = (i < r) ? bgr * iv.x * x[i] : 0.f;
                a.y = (i + 1 < r) ? bgr * iv.y * x[i + 1] : 0.f;
                a.z = (i + 2 < r) ? bgr * iv.z * x[i + 2] : 0.f;
                a.w = (i + 3 < r) ? bgr * iv.w * x[i + 3] : 0.f;
                *reinterpret_cast<float4 *>(dst + c) = a;
            }
        }
    }
    tc_fence_before();
    __syncthreads();   // A complete; p1 has read the Q rows (T goes over them)
    if (tid < 64) {
        // T = (I + A)^-1: 16x16 diagonal blocks by forward substitution
        const int b = tid >> 4, c = tid & 15;
        const float *Ab = a_blk(sm, b, b);
        float y[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < r; ++i) ps[i & 3] = fmaf(Ab[r * AB_P + i], y[i], ps[i & 3]);
            y[r] = ((r == c) ? 1.f : 0.f) - ((ps[0] + ps[1]) + (ps[2] + ps[3]));
        }
        float *Tb = t_blk(sm, b, b);
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * TB_P + c] = y[r];
    }
    __syncthreads();
    if (warp < 2) merge_level1(sm, mm + warp * 320, warp, lane);
    __syncthreads();
    merge_level2a(sm, mm + warp * 320, warp, lane);
    __syncthreads();
    merge_level2b(sm, mm, warp, lane);
    __syncthreads();
    // T' = diag(D) T diag(beta gamma) into both row halves of the p2 A tile;
    // T'' = diag(D) T diag(beta) straight to the tile.  Thread tid takes the
    // 16-byte pieces tid + 128 k (row q / 8, physical chunk q % 8), so that
    // every warp writes 512 contiguous bytes.
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q = tid + 128 * k, r = q >> 3, pc = q & 7, c = pc ^ (r & 7), rb = r >> 4;
        const float dr = sc->Dd[r];
        uint32_t a0 = 0u, a1 = 0u, a2 = 0u, a3 = 0u, b0 = 0u, b1 = 0u, b2 = 0u, b3 = 0u;
        if ((c >> 1) <= rb) {
            const float *tr = t_blk(sm, rb, c >> 1) + (r & 15) * TB_P + 8 * (c & 1);
            const float4 t0v = *reinterpret_cast<const float4 *>(tr);
            const float4 t1v = *reinterpret_cast<const float4 *>(tr + 4);
            const float4 g0 = *reinterpret_cast<const float4 *>(&sc->bg[8 * c]);
            const float4 g1 = *reinterpret_cast<const float4 *>(&sc->bg[8 * c + 4]);
            const float4 e0 = *reinterpret_cast<const float4 *>(&sc->beta[8 * c]);
            const float4 e1 = *reinterpret_cast<const float4 *>(&sc->beta[8 * c + 4]);
            const float4 u0 = make_float4(dr * t0v.x, dr * t0v.y, dr * t0v.z, dr * t0v.w);
            const float4 u1 = make_float4(dr * t1v.x, dr * t1v.y, dr * t1v.z, dr * t1v.w);
            a0 = pack_bf16(u0.x * g0.x, u0.y * g0.y); a1 = pack_bf16(u0.z * g0.z, u0.w * g0.w);
            a2 = pack_bf16(u1.x * g1.x, u1.y * g1.y); a3 = pack_bf16(u1.z * g1.z, u1.w * g1.w);
            b0 = pack_bf16(u0.x * e0.x, u0.y * e0.y); b1 = pack_bf16(u0.z * e0.z, u0.w * e0.w);
            b2 = pack_bf16(u1.x * e1.x, u1.y * e1.y); b3 = pack_bf16(u1.z * e1.z, u1.w * e1.w);
        }
        const uint32_t off = r * 128 + pc * 16;
        st_shared_v4(smem_u32(sm + P_TP + off), a0, a1, a2, a3);
        st_shared_v4(smem_u32(sm + P_TP + 8192 + off), a0, a1, a2, a3);
        if (p.keep_tiles) st_global_v4_hint(tile + TILE_TPP + off, b0, b1, b2, b3, keep_pol);
        else *reinterpret_cast<uint4 *>(tile + TILE_TPP + off) = make_uint4(b0, b1, b2, b3);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        // p2: [T'; T'] K -> TMEM columns 0..127: W = T' K in lanes 0..63 and
        // again in lanes 64..127 (A K-major, B = the K tile MN-major)
        tc_fence_after();
        const uint64_t dTP = desc_sw128(smem_u32(sm + P_TP), 16, 1024);
        const uint64_t dKm = desc_sw128(smem_u32(sm + P_KQ), 16384, 1024);
        const uint32_t id_p2 = idesc_bf16(128, 128, false, true);
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16_ss(tm, dTP + ((ks * 32) >> 4), dKm + ((ks * 2048) >> 4), id_p2, ks > 0);
        mma_commit(bar(PB_P2));
    }
    __syncwarp();
    if (tid >= 64) {
        // Pt[r][i] = exp(G_r - G_C) q_r.k_i for i <= r, from this lane's p1 row,
        // staged over the Q rows (T, which lived there, is dead)
        const int r = tid - 64;
        const float sr = sc->invD[r];
        const uint32_t pt_s = smem_u32(sm + P_KQ + 8192);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i0 = 8 * c + 2 * e;
                w[e] = pack_bf16(i0 <= r ? sr * x[i0] : 0.f, i0 + 1 <= r ? sr * x[i0 + 1] : 0.f);
            }
            st_shared_v4(pt_s + sw128_chunk(r, c), w[0], w[1], w[2], w[3]);
        }
    }
    {
        // -W row t staged over the T' tile (p2, its last reader, has completed):
        // warps 0-1 stage d_k 0..63 (kb 0), warps 2-3 d_k 64..127 (kb 1)
        ok = mbar_wait(bar(PB_P2), 0, lim, &no_abort) && ok;
        tc_fence_after();
        const int t = tid & 63, kb = tid >> 6;
        const uint32_t w_s = smem_u32(sm + P_TP + kb * 8192);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            float y[32];
            tmem_ld32(tm + lane_off + 64 * kb + 32 * h2, y);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float *e = y + 8 * c4;
                st_shared_v4(w_s + sw128_chunk(t, 4 * h2 + c4), pack_bf16(-e[0], -e[1]), pack_bf16(-e[2], -e[3]),
                             pack_bf16(-e[4], -e[5]), pack_bf16(-e[6], -e[7]));
            }
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        if (p.keep_tiles) {
            bulk_store_hint(tile + TILE_NEGW, smem_u32(sm + P_TP), 16384, keep_pol);   // -W, both blocks
            bulk_store_hint(tile + TILE_PT, smem_u32(sm + P_KQ + 8192), 8192, keep_pol);  // Pt
        } else {
            bulk_store(tile + TILE_NEGW, smem_u32(sm + P_TP), 16384);
            bulk_store(tile + TILE_PT, smem_u32(sm + P_KQ + 8192), 8192);
        }
        bulk_commit_wait_read();
    }
    if (!ok && p.err) atomicCAS(p.err, 0, 52);
    if (tid == 0) {
        // no TMA copy still landing and no MMA still running at exit (p2's
        // commit covers p1 too), whatever became of the waits above
        mbar_wait(bar(PB_FULL), 0, p.drain_ns, &no_abort);
        mbar_wait(bar(PB_P2), 0, p.drain_ns, &no_abort);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, P_TM_COLS);
    }
}

// ---------------------------------------------------------------- chain kernel
//
// A CTA walks one range of chunks of one (sequence, head).
//   MODE_OUT:   from a known start state (state_in for a sequence's first
//               range, a combined state for the others); writes the outputs
//               and, for the last range, the final state.
//   MODE_TRANS: the range's affine transition S_end = S_start M + R.  Chain R
//               starts from zero with the values, chain X from the identity
//               without them; they run side by side, one state warpgroup
//               each, and R and M = X_end go to the workspace.
// With one range per sequence (nseg = 1) MODE_OUT is the whole prefill.

enum { MODE_OUT = 0, MODE_TRANS = 1 };

template <int MODE, bool GATED>
__global__ void __launch_bounds__(kChainThreads, 1)
gdn_chunk_chain_kernel(const __grid_constant__ ChainParams p) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = aligned_smem(smraw);
    using Lay = ChainLayout<MODE>;
    constexpr int NST = Lay::NST;
    constexpr uint32_t C_BAR = c_bar<MODE>();
    uint32_t *tmem_base_ptr = reinterpret_cast<uint32_t *>(sm + C_BAR + 8 * CB_NUM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C_BAR + 8 * CB_NUM + 4);
    auto bar = [&](int i) { return smem_u32(sm + C_BAR + 8 * i); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H;
    if (MODE == MODE_TRANS) grid_dep_launch();   // the combine may stage its prologue early
    // ranges per (sequence, head); CTAs are ordered range-major, so that the
    // first ranges (which need no combined start state) are scheduled first
    const int per = MODE == MODE_OUT ? p.nseg : p.nseg - 1;
    const int nunits = (int)(gridDim.x / per);
    const int seg = blockIdx.x / nunits, nseq = (blockIdx.x % nunits) / H, h = blockIdx.x % H;
    int64_t bos, eos;
    SeqBounds{p.cu_seqlens, p.uniform_len}.get(nseq, bos, eos);
    const int nchunks = (int)((eos - bos + C - 1) / C);
    const int cb = seg * p.seg_len;                                 // first chunk of the range
    const int ce = min(nchunks, cb + p.seg_len);
    const int nloc = ce > cb ? ce - cb : 0;
    const int64_t gc0 = (p.chunk_off ? (int64_t)p.chunk_off[nseq] : (int64_t)nseq * p.cps) + cb;
    const size_t state_off = ((size_t)nseq * H + h) * D * D;
    const size_t unit = ((size_t)nseq * H + h) * (p.nseg - 1) + (seg - (MODE == MODE_OUT ? 1 : 0));
    const float *start = MODE == MODE_TRANS ? nullptr
                         : (seg == 0 ? p.state_in : p.seg_start + unit * D * D);
    float *finish = MODE == MODE_TRANS ? nullptr : (seg == p.nseg - 1 ? p.state_out : nullptr);

    // The copies of local chunk n into its stage (K and V boxes, the prep
    // tile or the part of it a transition range reads), completing on the
    // stage's FULL barrier.  L2 policies: a transition range keeps what the
    // output pass reads again (ptile, evict_last): the tiles, and also K and V
    // (pin) when the tiles are too many to stay in L2 from the prep kernel on;
    // otherwise the inputs are streamed (evict_first) so that the kept tiles
    // stay, and the output pass drops each tile unwritten once it is read.
    auto issue_stage = [&](int n, uint64_t pin, uint64_t ptile) {
        const int s = n % NST;
        const uint32_t st = smem_u32(sm + s * Lay::STAGE);
        const int z = (int)(bos + (int64_t)(cb + n) * C);
        const uint32_t full = bar(CB_FULL + s);
        const uint8_t *tile = p.tiles + ((size_t)(gc0 + n) * H + h) * kTileBytes;
        mbar_arrive_expect_tx(full, Lay::LOADED);
        for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d_hint(st + Lay::K + kb * Lay::KB, &p.map_k, kb * 64, h, z, full, pin);
            tma_load_3d_hint(st + Lay::V + kb * 8192, &p.map_v, kb * 64, h, z, full, pin);
            if (MODE == MODE_OUT)
                tma_load_3d_hint(st + ChainLayout<0>::Q + kb * ChainLayout<0>::KB, &p.map_q, kb * 64, h, z, full, pin);
        }
        if (n == 0 && p.wait_tiles) grid_dep_wait();   // tiles come from the prep kernel
        if (MODE == MODE_TRANS) {   // -W and T'': the tile's first 24 KB
            bulk_load_hint(st + ChainLayout<1>::W, tile, TILE_PT, full, ptile);
        } else {                    // -W per block after K and Q, then T'' and Pt
            for (int kb = 0; kb < 2; ++kb)
                bulk_load_hint(st + ChainLayout<0>::NEGW + kb * ChainLayout<0>::KB, tile + TILE_NEGW + kb * 8192,
                               8192, full, ptile);
            bulk_load_hint(st + ChainLayout<0>::TPP, tile + TILE_TPP, 16384, full, ptile);   // T'', Pt
        }
    };
    // When nothing upstream still writes this kernel's inputs (an output
    // range after the combine: the tiles are complete and K, V are inputs),
    // the load thread initialises the barriers itself and has the first
    // stages in flight before the rest of the prologue.
    const bool early = !p.wait_tiles && !p.wait_inputs;
    const int n_early = early ? min(NST, nloc) : 0;
    if (warp == 9 && lane == 0) {
        for (int i = 0; i < CB_NUM; ++i) {
            uint32_t cnt = (i == CB_SREADY || i == CB_UREADY || i == CB_SREADY2 || i == CB_UREADY2 ||
                            i == CB_OFREE) ? 128 : 1;
            if (MODE == MODE_TRANS && i >= CB_EMPTY && i < CB_EMPTY + 3) cnt = 2;   // both chains' MMAs
            mbar_init(bar(i), cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.map_k);
        tma_prefetch_desc(&p.map_v);
        if (MODE == MODE_OUT) tma_prefetch_desc(&p.map_q);
        const uint64_t pin = MODE == MODE_TRANS && !p.keep_tiles ? l2_evict_last_policy() : l2_evict_first_policy();
        const uint64_t ptile = MODE == MODE_TRANS ? l2_evict_last_policy() : l2_evict_first_policy();
        for (int n = 0; n < n_early; ++n) issue_stage(n, pin, ptile);
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(tmem_base_ptr), TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_base_ptr;
    const uint64_t lim = p.timeout_ns;
    if (p.wait_inputs) grid_dep_wait();   // k, v, g and beta are the prep kernel's outputs
    auto fail = [&](int code) {
        *abort_flag = 1;
        if (p.err) atomicCAS(p.err, 0, code);
    };

    if (nloc == 0) {
        // empty range: the state passes through (MODE_OUT); an empty transition
        // is R = 0, M = I (MODE_TRANS)
        if (tid < 128) {
            for (int j = 0; j < D; j += 4) {
                if (MODE == MODE_OUT && finish) {
                    const float4 v = start ? *reinterpret_cast<const float4 *>(start + (seg == 0 ? state_off : 0) + (size_t)tid * D + j)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4 *>(finish + state_off + (size_t)tid * D + j) = v;
                }
                if (MODE == MODE_TRANS) {
                    *reinterpret_cast<float4 *>(p.trans_r + unit * D * D + (size_t)tid * D + j) = make_float4(0.f, 0.f, 0.f, 0.f);
                    // M = I: hi = I, lo = 0; row tid, columns j .. j + 3 (in the
                    // combine's swizzled layout: piece j / 8 stored at (j / 8) ^ (tid & 7))
                    uint32_t *hi = reinterpret_cast<uint32_t *>(p.trans_m + unit * D * D) + (size_t)tid * (D / 2) +
                                   4 * ((j >> 3) ^ (tid & 7)) + ((j >> 1) & 3);
                    uint32_t *lo = hi + D * D / 2;
                    hi[0] = pack_bf16(tid == j ? 1.f : 0.f, tid == j + 1 ? 1.f : 0.f);
                    hi[1] = pack_bf16(tid == j + 2 ? 1.f : 0.f, tid == j + 3 ? 1.f : 0.f);
                    lo[0] = 0u;
                    lo[1] = 0u;
                }
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ TMA / bulk producer
        if (lane == 0) {
            const uint64_t pin = MODE == MODE_TRANS && !p.keep_tiles ? l2_evict_last_policy() : l2_evict_first_policy();
            const uint64_t ptile = MODE == MODE_TRANS ? l2_evict_last_policy() : l2_evict_first_policy();
            int issued[NST] = {};
            for (int s = 0; s < n_early; ++s) issued[s] = 1;
            // Pull chunk m's data into L2 while its stage is still in use, so
            // that the copy into shared memory, once the stage frees up, is an
            // L2 hit.
            auto prefetch = [&](int m) {
                if (m >= nloc) return;
                const int zm = (int)(bos + (int64_t)(cb + m) * C);
                for (int kb = 0; kb < 2; ++kb) {
                    tma_prefetch_3d(&p.map_k, kb * 64, h, zm);
                    tma_prefetch_3d(&p.map_v, kb * 64, h, zm);
                    if (MODE == MODE_OUT) tma_prefetch_3d(&p.map_q, kb * 64, h, zm);
                }
                bulk_prefetch_l2(p.tiles + ((size_t)(gc0 + m) * H + h) * kTileBytes,
                                 MODE == MODE_TRANS ? TILE_PT : (uint32_t)kTileBytes);
            };
            for (int n = n_early; n < nloc; ++n) {
                const int s = n % NST;
                if (n >= NST) {
                    prefetch(n);   // (the tiles are complete: the wait below chunk 0's loads came first)
                    if (!mbar_wait(bar(CB_EMPTY + s), ((n - NST) / NST) & 1, lim, abort_flag)) { fail(61); break; }
                }
                issue_stage(n, pin, ptile);
                ++issued[s];
            }
            const int zero = 0;   // no copy may still be landing in shared memory at exit
            for (int s = 0; s < NST; ++s)
                if (issued[s]) mbar_wait(bar(CB_FULL + s), (issued[s] - 1) & 1, p.drain_ns, &zero);
        }
    } else if (warp == 8 || (MODE == MODE_TRANS && warp == 10)) {
        // ------------------------------------------------------------ MMA issuers
        // warp 8: the state chain (p3, the residual and state products and,
        // for outputs, c1 and c2); warp 10 (MODE_TRANS): the identity chain,
        // issued alongside so that the two chains' MMA issues overlap
        const bool xissuer = warp == 10;
        if (lane == 0 && (!xissuer || MODE == MODE_TRANS)) {
            const uint32_t id_n64 = idesc_bf16(128, 64, false, false);
            const uint32_t id_n128 = idesc_bf16(128, 128, false, false);
            const uint32_t id_p3 = idesc_bf16(128, 64, true, false);
            const uint32_t id_b = idesc_bf16(128, 128, false, true);
            // descriptors are built once; a byte offset o inside the stages adds o >> 4
            const uint64_t dSTk = desc_sw128(smem_u32(sm), 16, 1024);      // K-major views of stage data
            const uint64_t dSTm = desc_sw128(smem_u32(sm), 8192, 1024);    // MN-major views of V (and K, MODE_TRANS)
            const uint64_t dKm = desc_sw128(smem_u32(sm), Lay::KB, 1024);  // MN-major view of K
            const int zero = 0;
            bool ok = true;
            // transition ranges: U^T (+)= S (-W)^T, -W as 64 rows per block, 8 KB apart
            auto issue_a = [&](uint32_t col_u, uint32_t col_sbf, uint32_t st, uint32_t accumulate_first) {
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t offw = st + ChainLayout<1>::W + (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_bf16_ts(tm + col_u, tm + col_sbf + 8 * ks, dSTk + (offw >> 4), id_n64,
                                ks > 0 ? 1u : accumulate_first);
                }
            };
            // (b): S += U^T K  (A = U^T bf16 in TMEM; B = K tile MN-major)
            auto issue_b = [&](uint32_t col_s, uint32_t col_u, uint32_t st) {
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tm + col_s, tm + col_u + 8 * ks, dKm + ((st + Lay::K + ks * 2048) >> 4), id_b, 1);
            };
            for (int n = 0; ok && n < nloc; ++n) {
                const int s = n % NST;
                const uint32_t st = s * Lay::STAGE;
                if (!(ok = mbar_wait(bar(CB_FULL + s), (n / NST) & 1, lim, abort_flag))) { fail(62); break; }
                tc_fence_after();
                if (MODE == MODE_TRANS && xissuer) {
                    // chain X: U_X^T = X (-W)^T (no values), then X += U_X^T K
                    if (!(ok = mbar_wait(bar(CB_SREADY2), n & 1, lim, abort_flag))) { fail(66); break; }
                    tc_fence_after();
                    issue_a(TM_XU, TM_XSBF, st, 0);
                    mma_commit(bar(CB_A2));
                    if (!(ok = mbar_wait(bar(CB_UREADY2), n & 1, lim, abort_flag))) { fail(67); break; }
                    tc_fence_after();
                    issue_b(TM_XS, TM_XU, st);
                    mma_commit(bar(CB_B2));
                    mma_commit(bar(CB_EMPTY + s));
                    continue;
                }
                // p3: U^T = V^T T''^T (the previous residual was consumed: U_READY(n-1))
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tm + TM_U, dSTm + ((st + Lay::V + ks * 2048) >> 4),
                                dSTk + ((st + Lay::TPP + ks * 32) >> 4), id_p3, ks > 0);
                if (!(ok = mbar_wait(bar(CB_SREADY), n & 1, lim, abort_flag))) { fail(63); break; }
                // the output group has read O^T of chunk n-1 and cleared it
                if (MODE == MODE_OUT && !(ok = mbar_wait(bar(CB_OFREE), n & 1, lim, abort_flag))) { fail(65); break; }
                tc_fence_after();
                if (MODE == MODE_TRANS) {
                    issue_a(TM_U, TM_SBF, st, 1);
                    mma_commit(bar(CB_A));
                    if (!(ok = mbar_wait(bar(CB_UREADY), n & 1, lim, abort_flag))) { fail(64); break; }
                    tc_fence_after();
                    issue_b(TM_S, TM_U, st);
                    mma_commit(bar(CB_B));
                    mma_commit(bar(CB_EMPTY + s));
                } else {
                    // (a) and c1 share A = S: [O1^T | U^T] += S [Q; -W]^T as one N = 128 MMA
                    // per K step, B = rows 64-191 of the stage's operand block (O1^T
                    // starts cleared, U^T holds p3)
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t off = st + ChainLayout<0>::Q + (ks >> 2) * ChainLayout<0>::KB + (ks & 3) * 32;
                        mma_bf16_ts(tm + TM_O, tm + TM_SBF + 8 * ks, dSTk + (off >> 4), id_n128, 1);
                    }
                    mma_commit(bar(CB_A));
                    if (!(ok = mbar_wait(bar(CB_UREADY), n & 1, lim, abort_flag))) { fail(64); break; }
                    tc_fence_after();
                    issue_b(TM_S, TM_U, st);
                    mma_commit(bar(CB_B));
                    // c2: O2^T = U^T Pt^T (gated: Q is diag(gamma) Q, and c2 accumulates onto O1^T)
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ts(tm + (GATED ? TM_O : TM_O2), tm + TM_U + 8 * ks,
                                    dSTk + ((st + ChainLayout<0>::PT + ks * 32) >> 4), id_n64,
                                    GATED ? 1u : (ks > 0 ? 1u : 0u));
                    mma_commit(bar(CB_C));
                    mma_commit(bar(CB_EMPTY + s));
                }
            }
            const int fin = xissuer ? CB_FIN2 : CB_FIN;
            mma_commit(bar(fin));   // every issued MMA completes before TMEM is released
            mbar_wait(bar(fin), 0, p.drain_ns, &zero);
        }
    } else if (warp < 4 || (MODE == MODE_TRANS && warp < 8)) {
        // ------------------------------------------------------------ state group(s)
        // warps 0-3: the state chain (R in MODE_TRANS); warps 4-7 in MODE_TRANS: chain X
        const bool xchain = warp >= 4;
        const int wg = warp & 3;
        const int dv = tid & 127;   // TMEM lane and state row
        const uint32_t lane_off = static_cast<uint32_t>(wg * 32) << 16;
        const uint32_t col_u = xchain ? TM_XU : TM_U, col_s = xchain ? TM_XS : TM_S;
        const uint32_t col_sbf = xchain ? TM_XSBF : TM_SBF;
        const int bA = xchain ? CB_A2 : CB_A, bB = xchain ? CB_B2 : CB_B;
        const int bS = xchain ? CB_SREADY2 : CB_SREADY, bU = xchain ? CB_UREADY2 : CB_UREADY;
        const int nb = xchain ? 3 : 2;    // named barrier of this group
        ChainScalars *scb = reinterpret_cast<ChainScalars *>(sm + (xchain ? c_scx<MODE>() : c_sce<MODE>()));
        GateRegs gr{0.f, 0.f, 0.f, 0.f};
        if (wg == 0) gr = load_gates(p.g, p.beta, bos, eos, cb, ce, h, H, lane);
        // scalars of local chunk m from the prefetched gates; prefetch chunk m+1's
        auto compute_scalars = [&](int m) {
            if (wg == 0) {
                float G0, G1;
                scan_gates(gr, lane, G0, G1);
                gr = load_gates(p.g, p.beta, bos, eos, cb + m + 1, ce, h, H, lane);
                const float GC = __shfl_sync(0xffffffffu, G1, 31);
                if (lane == 0) scb[m % 3].gC = expf(GC);
            }
        };
        // write 64 fp32 values of this lane's row as 32 packed bf16 columns
        auto st_bf16_cols = [&](uint32_t col, const float (&x0)[32], const float (&x1)[32]) {
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                pk[j] = pack_bf16(x0[2 * j], x0[2 * j + 1]);
                pk[16 + j] = pack_bf16(x1[2 * j], x1[2 * j + 1]);
            }
            tmem_st32u(tm + lane_off + col, pk);
        };
        compute_scalars(0);
        if (MODE == MODE_OUT && seg > 0 && p.wait_start) grid_dep_wait();   // start state from the combine
        named_bar_sync(nb, 128);
        {
            // start state: given (MODE_OUT), zero (chain R) or the identity (chain X)
            const float gC0 = scb[0].gC;
            float x0[32], x1[32];
            for (int c0 = 0; c0 < D; c0 += 64) {
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
                    if (start) {
                        const float *src = start + (seg == 0 ? state_off : 0) + (size_t)dv * D + c0 + j;
                        a = *reinterpret_cast<const float4 *>(src);
                        b = *reinterpret_cast<const float4 *>(src + 32);
                    }
                    x0[j] = a.x; x0[j + 1] = a.y; x0[j + 2] = a.z; x0[j + 3] = a.w;
                    x1[j] = b.x; x1[j + 1] = b.y; x1[j + 2] = b.z; x1[j + 3] = b.w;
                }
                if (xchain) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        x0[j] = (dv == c0 + j) ? 1.f : 0.f;
                        x1[j] = (dv == c0 + 32 + j) ? 1.f : 0.f;
                    }
                }
                st_bf16_cols(col_sbf + c0 / 2, x0, x1);
#pragma unroll
                for (int j = 0; j < 32; ++j) { x0[j] *= gC0; x1[j] *= gC0; }
                tmem_st32(tm + lane_off + col_s + c0, x0);
                tmem_st32(tm + lane_off + col_s + c0 + 32, x1);
            }
            tc_fence_before();
            mbar_arrive(bar(bS));
        }
        for (int n = 0; n < nloc; ++n) {
            // residual epilogue: U^T (fp32, lane dv, 64 t) -> bf16 in its own first 32 columns
            if (!mbar_wait(bar(bA), n & 1, lim, abort_flag)) fail(71);
            tc_fence_after();
            {
                float x0[32], x1[32];
                tmem_ld32(tm + lane_off + col_u, x0);
                tmem_ld32(tm + lane_off + col_u + 32, x1);
                st_bf16_cols(col_u, x0, x1);
            }
            tc_fence_before();
            mbar_arrive(bar(bU));
            const bool last = (n + 1 == nloc);
            if (!last) compute_scalars(n + 1);
            if (named_bar_any(nb, 128, *abort_flag != 0)) break;
            // state epilogue: publish the bf16 copy for the next (a), then rescale
            if (!mbar_wait(bar(bB), n & 1, lim, abort_flag)) fail(72);
            tc_fence_after();
            {
                float x0[32], x1[32];
                for (int c0 = 0; c0 < D; c0 += 64) {
                    tmem_ld32(tm + lane_off + col_s + c0, x0);
                    tmem_ld32(tm + lane_off + col_s + c0 + 32, x1);
                    if (!last) {
                        st_bf16_cols(col_sbf + c0 / 2, x0, x1);
                    }   // the last state stays in TMEM; it leaves at teardown (coalesced)
                }
                tc_fence_before();
                if (!last) {
                    // the next (a) may start now; the fp32 state is rescaled for the
                    // next (b), which the MMA thread issues only after U_READY
                    mbar_arrive(bar(bS));
                    const float gnext = scb[(n + 1) % 3].gC;
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        tmem_ld32(tm + lane_off + col_s + c0, x0);
#pragma unroll
                        for (int j = 0; j < 32; ++j) x0[j] *= gnext;
                        tmem_st32(tm + lane_off + col_s + c0, x0);
                    }
                    tc_fence_before();
                }
            }
        }
    } else if (MODE == MODE_OUT && warp != 8 && warp != 9) {
        // ------------------------------------------------------------ output group (MODE_OUT)
        // o_t = gamma_t O1_t + O2_t (lane dv, 64 t) -> bf16 rows of out; off the
        // state chain.  Warps 4-7 (TMEM lanes dv) stage the tile; warps 10-11
        // join them for the stores (and the output gate, the longest part of
        // the gated pass).  O2 of chunk n is read before OFREE(n + 1) is
        // signalled, and c2(n + 1), which overwrites it, is issued after the
        // merged MMA that waits for OFREE(n + 1).  Gated (layer mode), the q
        // buffer holds diag(gamma) q and c2 accumulates onto O1, so that
        // o_t = O1_t.
        constexpr int kOut = 192;                    // output threads
        constexpr int kRows = kOut / 16;             // rows per store pass (16 pieces a row)
        constexpr int kPasses = (C + kRows - 1) / kRows;
        const bool tw = warp < 8;                    // a TMEM warp
        const int dv = tid - 128;                    // TMEM lane (warps 4-7)
        const int so = tw ? dv : 128 + (warp - 10) * 32 + lane;   // 0 .. kOut - 1
        const int piece = so & 15, rsub = so >> 4;   // 16-byte piece, and row within a pass
        const uint32_t lane_off = static_cast<uint32_t>(tw ? (warp - 4) * 32 : 0) << 16;
        float *gam = reinterpret_cast<float *>(sm + c_scx<MODE>()) + (tw ? warp - 4 : 0) * C;   // this warp's gamma_t
        GateRegs gn{0.f, 0.f, 0.f, 0.f};
        if constexpr (!GATED) {
            if (tw) gn = load_gates_pinned(p.g, bos, eos, cb, ce, h, H, lane);
        }
        __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(sm + c_u<MODE>());
        float *stagef = reinterpret_cast<float *>(sm + c_u<MODE>());   // gated: the norm and gate take fp32 o
        float a[32];
        if (tw) {
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = 0.f;
            // O1^T starts cleared: the merged MMA accumulates c1 onto it
            tmem_st32(tm + lane_off + TM_O, a);
            tmem_st32(tm + lane_off + TM_O + 32, a);
            tc_fence_before();
            mbar_arrive(bar(CB_OFREE));
        }
        // output gate (layer mode): y = n(o) * act(z), n an RMS norm over the
        // row's d_v values (or the identity); a thread always takes the same
        // 8 channels (piece) of its rows, the 16 pieces of a row lying in 16
        // consecutive lanes
        constexpr bool gated = GATED;
        float nw[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) nw[e] = (gated && p.norm_w) ? __ldg(p.norm_w + piece * 8 + e) : 1.f;
        // z of this thread's pieces of local chunk m (rows past the end: 0),
        // issued where it stands (a plain load may be sunk to its use, a chunk
        // later, which would expose its latency there)
        auto load_z = [&](uint4 (&zz)[kPasses], int m) {
            const int64_t tz = bos + (int64_t)(cb + m) * C;
            const int lz = m < nloc ? (int)((eos - tz) < C ? (eos - tz) : C) : 0;
#pragma unroll
            for (int k = 0; k < kPasses; ++k) {
                const int t = kRows * k + rsub;
                zz[k] = make_uint4(0u, 0u, 0u, 0u);
                if (t < lz)
                    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(zz[k].x), "=r"(zz[k].y), "=r"(zz[k].z), "=r"(zz[k].w)
                                 : "l"(p.z + ((size_t)(tz + t) * H + h) * D + piece * 8));
            }
        };
        uint4 zr[kPasses], zn[kPasses];   // z of chunk n, and of chunk n + 1 in flight a whole chunk ahead
        if constexpr (gated) load_z(zr, 0);
        for (int n = 0; n < nloc; ++n) {
            // all output warps are done with chunk n-1's staging buffer
            if (named_bar_any(3, kOut, *abort_flag != 0)) break;
            const int64_t t0 = bos + (int64_t)(cb + n) * C;
            const int len = (int)((eos - t0) < C ? (eos - t0) : C);
            if constexpr (!gated) {
                if (tw) {
                    // gamma_t = exp(G_t) of chunk n (the state group's scan of the same
                    // gates), before this iteration's loads are issued: a wait for the
                    // gates must not also wait for them
                    float G0, G1;
                    scan_gates(gn, lane, G0, G1);
                    gam[lane] = expf(G0);
                    gam[lane + 32] = expf(G1);
                    __syncwarp();
                    gn = load_gates_pinned(p.g, bos, eos, cb + n + 1, ce, h, H, lane);
                }
            }
            if constexpr (gated) load_z(zn, n + 1);
            if (tw) {
                if (!mbar_wait(bar(CB_C), n & 1, lim, abort_flag)) fail(73);
                tc_fence_after();
                // o_t = gamma_t O1_t + O2_t (gated: O1_t), 32 columns t at a time,
                // into the staging tile
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    tmem_ld32(tm + lane_off + TM_O + 32 * hh, a);
                    if constexpr (!gated) {
                        float o2[32];
                        tmem_ld32(tm + lane_off + TM_O2 + 32 * hh, o2);
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 gv = *reinterpret_cast<const float4 *>(gam + 32 * hh + j);
                            a[j] = fmaf(gv.x, a[j], o2[j]);
                            a[j + 1] = fmaf(gv.y, a[j + 1], o2[j + 1]);
                            a[j + 2] = fmaf(gv.z, a[j + 2], o2[j + 2]);
                            a[j + 3] = fmaf(gv.w, a[j + 3], o2[j + 3]);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if constexpr (gated) stagef[(32 * hh + j) * D + dv] = a[j];
                        else stage[(32 * hh + j) * D + dv] = __float2bfloat16_rn(a[j]);
                    }
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) a[j] = 0.f;
                tmem_st32(tm + lane_off + TM_O, a);
                tmem_st32(tm + lane_off + TM_O + 32, a);
                tc_fence_before();
                mbar_arrive(bar(CB_OFREE));   // the MMA thread may accumulate chunk n+1's O1^T
            }
            named_bar_sync(3, kOut);
            if (p.keep_tiles) {
                // chunk n's prep tile, kept in L2, has been read for the last time
                // (its copies completed before c2(n)): drop it without a write-back
                const uint8_t *tl = p.tiles + ((size_t)(gc0 + n) * H + h) * kTileBytes;
                for (int i = so; i < (int)(kTileBytes / 128); i += kOut) l2_discard_line(tl + 128 * i);
            }
            // whole 16-byte pieces of the [64 t][128 dv] tile, rows t < len (a row
            // past 63 in the last pass is read as row 63, so that every lane takes
            // part in the shuffles, and not stored)
#pragma unroll
            for (int k = 0; k < kPasses; ++k) {
                const int t = kRows * k + rsub, tc = t < C ? t : C - 1;
                uint4 v;
                if constexpr (gated) {
                    const float4 f0 = *reinterpret_cast<const float4 *>(stagef + tc * D + piece * 8);
                    const float4 f1 = *reinterpret_cast<const float4 *>(stagef + tc * D + piece * 8 + 4);
                    const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
                    float ss = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
                    for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                    const float sc = p.norm_w ? rsqrtf(ss * (1.f / D) + p.eps) : 1.f;
                    float yv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float zv = piece_elem(zr[k], e), sg = sigmoid_t(zv);
                        yv[e] = f[e] * sc * nw[e] * (p.gate ? zv * sg : sg);
                    }
                    v = make_uint4(pack_bf16(yv[0], yv[1]), pack_bf16(yv[2], yv[3]), pack_bf16(yv[4], yv[5]),
                                   pack_bf16(yv[6], yv[7]));
                } else {
                    v = *reinterpret_cast<const uint4 *>(stage + tc * D + piece * 8);
                }
                if (t < len) *reinterpret_cast<uint4 *>(p.out + ((size_t)(t0 + t) * H + h) * D + piece * 8) = v;
            }
            if constexpr (gated) {
#pragma unroll
                for (int k = 0; k < kPasses; ++k) zr[k] = zn[k];
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    if (p.wait_tiles) grid_dep_wait();   // (also for an empty range: completion implies the prep's)
    tc_fence_before();
    __syncthreads();   // every MMA has completed (the MMA thread waited for them) and no copy is landing
    // Final states (R and M of a transition range, state_out of a sequence's
    // last output range) leave TMEM through shared memory, whose stages are
    // idle now: each state warp writes its rows (padded pitch, conflict-free),
    // then all threads store 16-byte pieces in row order.
    if (nloc > 0 && *abort_flag == 0) {
        constexpr int PITCH = D + 4;   // fp32 rows
        constexpr int MPW = D / 2 + 4;  // 32-bit words per bf16 row (M of a transition range)
        static_assert(4 * (D * PITCH + 2 * D * MPW) <= Lay::NST * Lay::STAGE, "staging fits the idle stages");
        const int nchains = MODE == MODE_TRANS ? 2 : 1;
        for (int c = 0; c < nchains; ++c) {
            float *dst = MODE == MODE_TRANS ? (c ? p.trans_m : p.trans_r) + unit * D * D
                                            : (finish ? finish + state_off : nullptr);
            if (!dst) break;   // uniform over the CTA
            float *stg = reinterpret_cast<float *>(sm) + c * D * PITCH;
            if ((warp >> 2) == c && warp < 8) {
                tc_fence_after();
                const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
                const int row = (warp & 3) * 32 + lane;
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float x[32];
                    tmem_ld32(tm + lane_off + (c ? TM_XS : TM_S) + c0, x);
                    if (MODE == MODE_TRANS && c == 1) {
                        // M leaves as bf16 hi and lo rows (M = hi + lo to about
                        // 16 mantissa bits), the form the combine's mma.sync
                        // consumes: rows of MPW words, hi rows then lo rows
                        uint32_t *sh = reinterpret_cast<uint32_t *>(stg);
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            uint32_t h_[4], l_[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) split2(x[j + 2 * e], x[j + 2 * e + 1], h_[e], l_[e]);
                            *reinterpret_cast<uint4 *>(sh + row * MPW + (c0 + j) / 2) = make_uint4(h_[0], h_[1], h_[2], h_[3]);
                            *reinterpret_cast<uint4 *>(sh + (D + row) * MPW + (c0 + j) / 2) = make_uint4(l_[0], l_[1], l_[2], l_[3]);
                        }
                        continue;
                    }
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(stg + row * PITCH + c0 + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
                }
            }
        }
        __syncthreads();
        for (int c = 0; c < nchains; ++c) {
            float *dst = MODE == MODE_TRANS ? (c ? p.trans_m : p.trans_r) + unit * D * D
                                            : (finish ? finish + state_off : nullptr);
            if (!dst) break;
            const float *stg = reinterpret_cast<const float *>(sm) + c * D * PITCH;
            if (MODE == MODE_TRANS && c == 1) {
                // 2 D rows of 16 pieces (hi, then lo); piece p of row r is stored at
                // p ^ (r & 7), the swizzle under which the combine's ldmatrix reads
                // eight rows at one column without bank conflicts
                const uint32_t *sh = reinterpret_cast<const uint32_t *>(stg);
                for (int i = threadIdx.x; i < 2 * D * 16; i += blockDim.x) {
                    const int row = i >> 4, piece = i & 15;
                    reinterpret_cast<uint4 *>(dst)[row * 16 + (piece ^ (row & 7))] =
                        *reinterpret_cast<const uint4 *>(sh + row * MPW + 4 * piece);
                }
                continue;
            }
            for (int i = threadIdx.x; i < D * D / 4; i += blockDim.x) {
                const int row = i >> 5, c4 = i & 31;
                *reinterpret_cast<float4 *>(dst + row * D + 4 * c4) =
                    *reinterpret_cast<const float4 *>(stg + row * PITCH + 4 * c4);
            }
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tm, TM_COLS);
    }
}

// ---------------------------------------------------------------- segment combine
//
// Start state of every range after the first: S_{j+1} = S_j M_j + R_j,
// sequentially over the ranges of one (sequence, head).  Rows of S are
// independent, so a CTA owns 16 of them: grid (N*H, 8), eight warps.  Warp w
// computes columns [16 w, +16) of S_{j+1} over the whole k range and adds R_j
// to them, so that no partial sums cross warps; S_j and S_{j+1} alternate
// between two shared-memory row buffers.
// The products run on bf16 mma.sync with each fp32 operand split in two
// (x = hi + lo, both bf16; S M ~= S_hi M_hi + S_hi M_lo + S_lo M_hi), which
// keeps about 16 mantissa bits; accumulation is fp32.  M_j arrives already
// split from the transition ranges (bf16 hi and lo rows [k][n], each row's
// 16-byte pieces swizzled by row % 8) and ldmatrix (.trans) turns its rows into
// B fragments.  S_{j+1} is split once, by the warp that computes it, into bf16
// hi and lo rows, from which every warp takes its A fragments with ldmatrix.
// M_{j+1} and this CTA's rows of R_{j+1} stream into the other half of a
// double buffer as bulk copies (one thread, an mbarrier) while step j computes.
constexpr int kCombRows = 16;
constexpr int kCombThreads = 256;
constexpr int kCombAP = 136;                                    // bf16 row pitch of S: conflict-free ldmatrix
constexpr uint32_t kCombSBytes = 2 * kCombRows * kCombAP * 2;   // one S buffer: hi rows, then lo rows
constexpr uint32_t kCombMBytes = 2 * D * D * 2;                 // M_j: hi and lo bf16 rows
constexpr uint32_t kCombRBytes = kCombRows * D * 4;             // 16 rows of R_j
constexpr uint32_t kCombBufBytes = kCombMBytes + kCombRBytes;
constexpr size_t kCombSmem = (size_t)2 * kCombBufBytes + (size_t)2 * kCombSBytes + 64;

// four 8x8 bf16 blocks as they are stored: the row-major A fragments of mma.sync
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const __nv_bfloat16 *row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(row)));
}

// four 8x8 bf16 blocks, transposed on the way: the col-major B fragments of mma.sync
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const __nv_bfloat16 *row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(row)));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kCombThreads, 1)
gdn_scan_combine_kernel(const float *__restrict__ state_in, const float *__restrict__ trans_r,
                        const float *__restrict__ trans_m, float *__restrict__ seg_start, int nseg,
                        int *err, uint64_t timeout_ns, uint64_t drain_ns) {
    extern __shared__ __align__(128) uint8_t smc[];
    // [buffer 0: M hi, M lo, R rows][buffer 1: the same][S hi and lo rows, two buffers][2 mbarriers, abort flag]
    __nv_bfloat16 *Ss = reinterpret_cast<__nv_bfloat16 *>(smc + 2 * kCombBufBytes);   // [2][hi, lo][16][kCombAP]
    uint8_t *ctl = smc + 2 * kCombBufBytes + 2 * kCombSBytes;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(ctl + 16);
    auto bar = [&](int b) { return smem_u32(ctl + 8 * b); };
    const int nh = blockIdx.x, r0 = blockIdx.y * kCombRows;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g = lane >> 2, q = lane & 3;
    if (t == 0) {
        mbar_init(bar(0), 1);
        mbar_init(bar(1), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    grid_dep_wait();     // the transitions come from the previous kernel
    grid_dep_launch();   // the output pass may launch; its first ranges do not need this grid
    // without an initial state S_0 = 0, so S_1 = R_0: step 0 neither reads M_0 nor forms products
    auto has_products = [&](int j) { return j > 0 || state_in != nullptr; };
    auto stage = [&](int j) {   // thread 0
        const size_t unit = ((size_t)nh * (nseg - 1) + j) * D * D;
        const uint32_t dst = smem_u32(smc + (j & 1) * kCombBufBytes);
        mbar_arrive_expect_tx(bar(j & 1), has_products(j) ? kCombBufBytes : kCombRBytes);
        if (has_products(j))
            for (uint32_t o = 0; o < kCombMBytes; o += 16384)
                bulk_load(dst + o, reinterpret_cast<const uint8_t *>(trans_m + unit) + o, 16384, bar(j & 1));
        bulk_load(dst + kCombMBytes, trans_r + unit + (size_t)r0 * D, kCombRBytes, bar(j & 1));
    };
    int pending = -1;   // the last step whose copies were issued and not yet waited for
    if (nseg > 1 && t == 0) stage(0);
    if (nseg > 1) pending = 0;
    // S_0: this CTA's rows of the initial state, split into buffer 0
    for (int i = t; i < kCombRows * D / 2; i += kCombThreads) {
        const int row = i >> 6, col = 2 * (i & 63);
        const float2 v = state_in ? *reinterpret_cast<const float2 *>(state_in + (size_t)nh * D * D +
                                                                       (size_t)(r0 + row) * D + col)
                                  : make_float2(0.f, 0.f);
        uint32_t hi, lo;
        split2(v.x, v.y, hi, lo);
        *reinterpret_cast<uint32_t *>(Ss + row * kCombAP + col) = hi;
        *reinterpret_cast<uint32_t *>(Ss + (kCombRows + row) * kCombAP + col) = lo;
    }
    for (int j = 0; j + 1 < nseg; ++j) {
        const size_t u = ((size_t)nh * (nseg - 1) + j) * D * D + (size_t)r0 * D;   // rows r0.. of step j
        float acc[2][4], accx[2][4], accy[2][4];   // hi*hi terms; lo*hi; hi*lo
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = accx[nt][e] = accy[nt][e] = 0.f;
        if (!mbar_wait(bar(j & 1), (j >> 1) & 1, timeout_ns, abort_flag)) {
            *abort_flag = 1;
            if (err) atomicCAS(err, 0, 81);
        }
        __syncthreads();   // M_j and R_j landed (or the wait gave up); S_j rows are written, S_{j-1} read
        if (*abort_flag) break;
        pending = -1;
        if (j + 2 < nseg) {
            if (t == 0) {
                fence_proxy_async_smem();   // step j-1's reads of that buffer come before the copy
                stage(j + 1);
            }
            pending = j + 1;
        }
        const __nv_bfloat16 *Mh = reinterpret_cast<const __nv_bfloat16 *>(smc + (j & 1) * kCombBufBytes);
        const __nv_bfloat16 *Ml = Mh + D * D;
        const float *Rs = reinterpret_cast<const float *>(smc + (j & 1) * kCombBufBytes + kCombMBytes);
        const __nv_bfloat16 *Sc = Ss + (j & 1) * (kCombSBytes / 2);         // S_j: hi rows, lo rows
        __nv_bfloat16 *Sn = Ss + ((j + 1) & 1) * (kCombSBytes / 2);         // S_{j+1}
        if (has_products(j)) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int k0 = 16 * ks;
                // lane -> row lane & 15 of the 16-row block, columns k0 + 8 (lane >> 4) ..: the four
                // 8x8 blocks {rows 0-7, 8-15} x {k0, k0 + 8} are the A fragments {a0, a1, a2, a3}
                const int aoff = (lane & 15) * kCombAP + k0 + 8 * (lane >> 4);
                uint32_t ah[4], al[4];
                ldmatrix_x4(ah, Sc + aoff);
                ldmatrix_x4(al, Sc + kCombRows * kCombAP + aoff);
                // lane -> row of one of four 8x8 blocks: k0 + (lane & 7) + 8 ((lane >> 3) & 1),
                // 16-byte piece 2 w + (lane >> 4) of that row (stored at piece ^ (row % 8));
                // .trans turns them into the B fragments {b0, b1} of n-tiles 0 and 1
                const int krow = k0 + (lane & 7) + 8 * ((lane >> 3) & 1);
                const int off = krow * D + (((2 * warp + (lane >> 4)) ^ (krow & 7)) << 3);
                uint32_t bh[4], bl[4];
                ldmatrix_x4_trans(bh, Mh + off);
                ldmatrix_x4_trans(bl, Ml + off);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    mma_bf16_16816(accx[nt], al[0], al[1], al[2], al[3], bh[2 * nt], bh[2 * nt + 1]);
                    mma_bf16_16816(accy[nt], ah[0], ah[1], ah[2], ah[3], bl[2 * nt], bl[2 * nt + 1]);
                    mma_bf16_16816(acc[nt], ah[0], ah[1], ah[2], ah[3], bh[2 * nt], bh[2 * nt + 1]);
                }
            }
        }
        // S_{j+1} = S_j M_j + R_j: rows g and g + 8, columns 16 w + 8 nt + 2 q, + 1
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = 16 * warp + 8 * nt + 2 * q;
            const float2 ra = *reinterpret_cast<const float2 *>(Rs + g * D + col);
            const float2 rb = *reinterpret_cast<const float2 *>(Rs + (g + 8) * D + col);
            const float2 va = make_float2(acc[nt][0] + (accx[nt][0] + accy[nt][0]) + ra.x,
                                          acc[nt][1] + (accx[nt][1] + accy[nt][1]) + ra.y);
            const float2 vb = make_float2(acc[nt][2] + (accx[nt][2] + accy[nt][2]) + rb.x,
                                          acc[nt][3] + (accx[nt][3] + accy[nt][3]) + rb.y);
            *reinterpret_cast<float2 *>(seg_start + u + g * D + col) = va;
            *reinterpret_cast<float2 *>(seg_start + u + (g + 8) * D + col) = vb;
            uint32_t hi, lo;
            split2(va.x, va.y, hi, lo);
            *reinterpret_cast<uint32_t *>(Sn + g * kCombAP + col) = hi;
            *reinterpret_cast<uint32_t *>(Sn + (kCombRows + g) * kCombAP + col) = lo;
            split2(vb.x, vb.y, hi, lo);
            *reinterpret_cast<uint32_t *>(Sn + (g + 8) * kCombAP + col) = hi;
            *reinterpret_cast<uint32_t *>(Sn + (kCombRows + g + 8) * kCombAP + col) = lo;
        }
    }
    // no bulk copy may still be landing in shared memory at exit
    const int zero = 0;
    if (t == 0 && pending >= 0) mbar_wait(bar(pending & 1), (pending >> 1) & 1, drain_ns, &zero);
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


size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr size_t kKeepTileBytes = (size_t)96 << 20;   // tiles kept in L2 up to this size

size_t chunk_off_bytes(int num_seqs) { return align_up(4 * (size_t)(num_seqs + 1), 1024); }

// units of the range-transition arrays (R, M, start states)
size_t scan_units(int num_seqs, int H, int nseg) {
    return (size_t)num_seqs * H * (size_t)(nseg > 1 ? nseg - 1 : 0);
}

// Launch with programmatic stream serialization (see launch_prefill_tc).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

bool set_smem_attrs() {
    static bool done[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (dev >= 0 && dev < 64 && done[dev]) return true;
    if (cudaFuncSetAttribute(gdn_chunk_prep_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)P_ALLOC) != cudaSuccess ||
        cudaFuncSetAttribute(gdn_chunk_prep_kernel<false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             100) != cudaSuccess ||
        cudaFuncSetAttribute(gdn_chunk_prep_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)P_ALLOC) != cudaSuccess ||
        cudaFuncSetAttribute(gdn_chunk_prep_kernel<true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             100) != cudaSuccess ||
        cudaFuncSetAttribute(gdn_chunk_chain_kernel<MODE_OUT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)c_alloc<MODE_OUT>()) != cudaSuccess ||
        cudaFuncSetAttribute(gdn_chunk_chain_kernel<MODE_OUT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)c_alloc<MODE_OUT>()) != cudaSuccess ||
        cudaFuncSetAttribute(gdn_chunk_chain_kernel<MODE_TRANS, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)c_alloc<MODE_TRANS>()) != cudaSuccess ||
        cudaFuncSetAttribute(gdn_scan_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kCombSmem) != cudaSuccess)
        return false;
    if (dev >= 0 && dev < 64) done[dev] = true;
    return true;
}

// SM count of the current device, capped at the reference count the
// workspace is sized for (host query only).
int scan_sm_count() {
    int dev = 0, sms = kScanRefSMs;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms < kScanRefSMs ? sms : kScanRefSMs;
}

}  // namespace

size_t tc_workspace_bytes(int num_seqs, int64_t total_tokens, int H, bool varlen) {
    // range states are sized for an unpacked call on the reference SM count;
    // packed (varlen) calls run one range per sequence and leave them unused
    const int nseg = tc_scan_segments(num_seqs, total_tokens, H, false, kScanRefSMs);
    return 1024 + chunk_off_bytes(num_seqs) +
           (size_t)tc_chunk_bound(num_seqs, total_tokens, varlen) * (size_t)H * kTileBytes +
           3 * scan_units(num_seqs, H, nseg) * D * D * sizeof(float);
}

int tc_kernel_count(int num_seqs, int64_t total_tokens, int H, bool varlen) {
    if (varlen) return 3;
    return tc_scan_segments(num_seqs, total_tokens, H, false, scan_sm_count()) > 1 ? 4 : 2;
}

cudaError_t prefill_tc_setup() {
    if (set_smem_attrs()) return cudaSuccess;
    const cudaError_t e = cudaGetLastError();
    return e != cudaSuccess ? e : cudaErrorUnknown;
}

cudaError_t launch_prefill_tc(const TcLaunch &L, cudaStream_t stream) {
    const bool varlen = L.cu_seqlens != nullptr;
    uint8_t *ws = static_cast<uint8_t *>(L.workspace);
    int32_t *chunk_off = varlen ? reinterpret_cast<int32_t *>(ws + 1024) : nullptr;
    uint8_t *tiles = ws + 1024 + chunk_off_bytes(L.num_seqs);
    const int cps = varlen ? 0 : (int)((L.uniform_len + C - 1) / C);
    const int64_t bound = tc_chunk_bound(L.num_seqs, L.total_tokens, varlen);
    if (bound <= 0) return cudaSuccess;
    if (bound > 0x7fffffff || L.H > 65535) return cudaErrorInvalidValue;
    // sequence-parallel ranges for few long sequences (never more than the
    // workspace was sized for: the SM count is capped at the reference count)
    const int nseg = tc_scan_segments(L.num_seqs, L.total_tokens, L.H, varlen, scan_sm_count());
    const int seg_len = nseg > 1 ? (cps + nseg - 1) / nseg : 0x3fffffff;
    uint8_t *scan_base = tiles + (size_t)bound * L.H * kTileBytes;
    const size_t su = scan_units(L.num_seqs, L.H, nseg);

    PrepParams pp;
    ChainParams cp;
    memset(&pp, 0, sizeof(pp));
    memset(&cp, 0, sizeof(cp));
    const TcLayer *Ly = L.layer;
    if (Ly) {
        // the prep kernel reads the raw projections; the chains read the
        // q, k, v, g and beta it writes
        if (!make_token_map(&pp.map_q, Ly->xq, L.total_tokens, L.H) ||
            !make_token_map(&pp.map_k, Ly->xk, L.total_tokens, L.H) ||
            !make_token_map(&pp.map_v, Ly->xv, L.total_tokens, L.H) ||
            !make_token_map(&cp.map_q, Ly->q, L.total_tokens, L.H) ||
            !make_token_map(&cp.map_k, Ly->k, L.total_tokens, L.H) ||
            !make_token_map(&cp.map_v, Ly->v, L.total_tokens, L.H))
            return cudaErrorInvalidValue;
        pp.layer = 1;
        pp.xq = static_cast<const __nv_bfloat16 *>(Ly->xq);
        pp.xk = static_cast<const __nv_bfloat16 *>(Ly->xk);
        pp.xv = static_cast<const __nv_bfloat16 *>(Ly->xv);
        pp.conv_w = Ly->conv_w;
        pp.a_logit = Ly->a_logit;
        pp.b_logit = Ly->b_logit;
        pp.cs_in = static_cast<const __nv_bfloat16 *>(Ly->cs_in);
        pp.q_out = static_cast<__nv_bfloat16 *>(Ly->q);
        pp.k_out = static_cast<__nv_bfloat16 *>(Ly->k);
        pp.v_out = static_cast<__nv_bfloat16 *>(Ly->v);
        pp.g_out = Ly->g;
        pp.beta_out = Ly->beta;
        pp.act = Ly->activation;
        pp.eps = Ly->eps;
        pp.g = cp.g = Ly->g;
        pp.beta = cp.beta = Ly->beta;
    } else {
        if (!make_token_map(&pp.map_q, L.q, L.total_tokens, L.H) ||
            !make_token_map(&pp.map_k, L.k, L.total_tokens, L.H) ||
            !make_token_map(&cp.map_v, L.v, L.total_tokens, L.H))
            return cudaErrorInvalidValue;
        cp.map_q = pp.map_q;
        cp.map_k = pp.map_k;
        pp.g = cp.g = L.g;
        pp.beta = cp.beta = L.beta;
    }
    pp.cu_seqlens = cp.cu_seqlens = L.cu_seqlens;
    pp.chunk_off = cp.chunk_off = chunk_off;
    pp.uniform_len = cp.uniform_len = L.uniform_len;
    pp.cps = cp.cps = cps;
    pp.num_seqs = L.num_seqs;
    // tiles of at most three quarters of the 126 MB L2 stay there from the prep
    // kernel to the chain passes (evict_last); larger sets stream
    pp.keep_tiles = cp.keep_tiles = (size_t)bound * L.H * kTileBytes <= kKeepTileBytes ? 1 : 0;
    pp.H = cp.H = L.H;
    pp.tiles = tiles;
    cp.tiles = tiles;
    pp.err = cp.err = L.err;
    pp.timeout_ns = cp.timeout_ns = L.timeout_ns;
    pp.drain_ns = cp.drain_ns = L.drain_ns;
    cp.state_in = L.state_in;
    cp.state_out = L.state_out;
    cp.out = static_cast<__nv_bfloat16 *>(L.out);
    cp.nseg = nseg;
    cp.seg_len = seg_len;
    cp.trans_r = reinterpret_cast<float *>(scan_base);
    cp.trans_m = cp.trans_r + su * D * D;
    cp.seg_start = cp.trans_m + su * D * D;

    if (!set_smem_attrs()) return cudaGetLastError() != cudaSuccess ? cudaGetLastError() : cudaErrorUnknown;
    if (varlen) gdn_chunk_offsets_kernel<<<1, 1024, 0, stream>>>(L.cu_seqlens, L.num_seqs, chunk_off);
    dim3 pgrid((unsigned)bound, (unsigned)L.H);
    if (Ly)
        gdn_chunk_prep_kernel<true><<<pgrid, kPrepThreads, P_ALLOC, stream>>>(pp);
    else
        gdn_chunk_prep_kernel<false><<<pgrid, kPrepThreads, P_ALLOC, stream>>>(pp);
    const unsigned units = (unsigned)L.num_seqs * (unsigned)L.H;
    // TRANS, the combine and OUT are launched with programmatic stream
    // serialization: each may start its prologue while the previous kernel
    // drains, and waits (griddepcontrol.wait) before it reads that kernel's
    // results.
    if (nseg > 1) {
        ChainParams ct = cp;
        ct.wait_tiles = 1;
        ct.wait_start = 0;
        ct.wait_inputs = Ly ? 1 : 0;
        cudaError_t e = launch_pdl(gdn_chunk_chain_kernel<MODE_TRANS, false>, dim3(units * (nseg - 1)), dim3(kChainThreads),
                                   c_alloc<MODE_TRANS>(), stream, ct);
        if (e != cudaSuccess) return e;
        e = launch_pdl(gdn_scan_combine_kernel, dim3(units, D / kCombRows), dim3(kCombThreads), kCombSmem, stream,
                       L.state_in, static_cast<const float *>(cp.trans_r), static_cast<const float *>(cp.trans_m),
                       const_cast<float *>(cp.seg_start), nseg, L.err, L.timeout_ns, L.drain_ns);
        if (e != cudaSuccess) return e;
    }
    ChainParams co = cp;
    co.wait_tiles = nseg > 1 ? 0 : 1;   // after the combine, the prep kernel has completed
    co.wait_start = nseg > 1 ? 1 : 0;
    co.wait_inputs = (Ly && nseg == 1) ? 1 : 0;
    if (Ly && Ly->z) {
        co.z = static_cast<const __nv_bfloat16 *>(Ly->z);
        co.norm_w = Ly->norm_w;
        co.gate = Ly->gate;
        co.eps = Ly->eps;
    }
    const cudaError_t e = co.z ? launch_pdl(gdn_chunk_chain_kernel<MODE_OUT, true>, dim3(units * nseg),
                                            dim3(kChainThreads), c_alloc<MODE_OUT>(), stream, co)
                               : launch_pdl(gdn_chunk_chain_kernel<MODE_OUT, false>, dim3(units * nseg),
                                            dim3(kChainThreads), c_alloc<MODE_OUT>(), stream, co);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn
