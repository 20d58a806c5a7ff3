// Sliding-window attention forward and rotary position embedding: the local
// softmax attention layer of InfiniteVL's hybrid block.
//
// The InfiniteVL explainer page ("Step 2: Process tokens with Hybrid Blocks"
// and the "Sliding Window Attention" concept box) pairs every three Gated
// DeltaNet layers with one attention layer that only looks at a recent
// window of tokens (8K), with rotary positions and grouped-query heads (16
// query heads share 2 key/value heads).  Readings taken: query token t of a
// sequence attends to the keys s of the same sequence with
// t - window < s <= t; scores are (q . k) * scale; query head h reads
// key/value head h / (Hq / Hkv); RoPE is the rotate-half form at the token's
// position inside its sequence plus an offset.
//
// Two attention kernels.  For grouped heads with an even group size the
// head-pair kernel further down (two query heads of one key/value group per
// CTA) is used; this one covers the rest.
//
// Single-tile kernel: one CTA per (128 query tokens, query head), 320 threads.
//   warps 0-7  softmax: warps w and w + 4 share query rows 32(w%4) ..
//              32(w%4) + 31 (TMEM lanes); each takes one 64-column half of a
//              score block, and the pair agrees on the row maximum through
//              shared memory once per block
//   warp 8     TMA producer: the Q tile once, then K and V blocks of 128 keys
//              through two 3-stage rings
//   warp 9     MMA issuer (one lane)
// Per key block j: S_j = Q K_j^T on the tensor core (fp32 in TMEM, two
// buffers), the softmax threads turn S_j into P_j = 2^(c S_j - m) (bf16, in
// TMEM) and the tensor core accumulates O += P_j V_j in TMEM with P_j as the
// TMEM-resident A operand.  The running maximum m only moves (and O is
// rescaled) when a block raises it by more than 8 (a factor 256), so
// rescales are rare; P, the row sum and O all use the same m, so the final
// O / sum is exact up to rounding.  A block is therefore read once: its
// probabilities are formed against the current m while its maximum is
// tracked, and formed again only when that maximum moves m.  S_{j+1} and
// P_{j-1} V_{j-1} run on the tensor core while the softmax of block j runs.
//
// The key range of a CTA is [max(bos(t0), t0 - window + 1), t_last]; blocks
// of that range that every row of the tile sees whole skip the mask.  Query
// tiles may straddle sequence starts: rows are masked one by one.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "gdn.h"
#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kD = 128;                 // head dimension
constexpr int kBM = 128;                // query rows per CTA
constexpr int kBN = 128;                // keys per block
constexpr int kKVStages = 3;
constexpr uint32_t kHalf = 16384;       // [128 rows][64 bf16] swizzled half tile
constexpr uint32_t kBlk = 2 * kHalf;    // [128 rows][128 bf16]

// shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t SM_Q = 0;
constexpr uint32_t SM_K = kBlk;
constexpr uint32_t SM_V = SM_K + kKVStages * kBlk;
constexpr uint32_t SM_BAR = SM_V + kKVStages * kBlk;
enum : int {
    BR_Q = 0,
    BR_KFULL = 1,                       // + stage
    BR_KEMPTY = BR_KFULL + kKVStages,
    BR_VFULL = BR_KEMPTY + kKVStages,
    BR_VEMPTY = BR_VFULL + kKVStages,
    BR_SFULL = BR_VEMPTY + kKVStages,   // + S buffer (2)
    BR_PREADY = BR_SFULL + 2,           // + P buffer (2)
    BR_PVDONE = BR_PREADY + 2,          // + P buffer (2): P V with that buffer completed
    BR_FIN = BR_PVDONE + 2,
    BR_NUM = BR_FIN + 1
};
constexpr uint32_t SM_TMEM_SLOT = SM_BAR + 8 * BR_NUM;
constexpr uint32_t SM_ABORT = SM_TMEM_SLOT + 4;
constexpr uint32_t SM_XCH = SM_BAR + 176;       // [2 parities][2 column halves][128 rows] fp32
constexpr uint32_t SM_ALLOC = SM_XCH + 2 * 2 * 128 * 4;
constexpr size_t kSwaSmem = 232448;             // the per-CTA maximum; the rest is alignment slack
static_assert(8 * BR_NUM + 8 <= 176, "barrier area");
static_assert(SM_ALLOC <= kSwaSmem, "shared memory per CTA");

// tensor memory columns (512 allocated: the CTA owns the SM)
constexpr uint32_t TM_S = 0;      // 2 x 128: scores
constexpr uint32_t TM_P = 256;    // 2 x 64: bf16 probabilities (2 per column)
constexpr uint32_t TM_O = 384;    // 128: output accumulator
constexpr uint32_t kTmemCols = 512;

constexpr int kSoftmaxWarps = 8;       // two per TMEM lane quarter: one per 64-column half
constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.f;   // log2 units

struct SwaParams {
    __nv_bfloat16 *o;                   // [T, Hq, 128]
    const int32_t *cu;                  // [num_seqs + 1] or null
    int64_t uniform_len;                // sequence length when cu is null
    int num_seqs;
    int T, Hq, Hkv, window;
    float c;                            // scale * log2(e)
    int *err;                           // device status word, or null
    uint64_t timeout_ns;                // bound on the waits of the work loops
    uint64_t drain_ns;                  // bound on the waits that drain copies and MMAs before exit
};

// First token of the sequence that holds token t.
__device__ __forceinline__ int seq_start(const SwaParams &p, int t) {
    if (!p.cu) return static_cast<int>(t - t % p.uniform_len);
    int a = 0, b = p.num_seqs;   // cu[a] <= t < cu[b]
    while (b - a > 1) {
        const int m = (a + b) >> 1;
        if (__ldg(p.cu + m) <= t) a = m;
        else b = m;
    }
    return __ldg(p.cu + a);
}

__global__ void __launch_bounds__(kThreads, 1)
    swa_fwd_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                   const __grid_constant__ CUtensorMap mV, const SwaParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad + SM_ALLOC > kSwaSmem) {   // cannot happen with an aligned dynamic base; never touch past the end
        if (threadIdx.x == 0 && p.err) atomicCAS(p.err, 0, 80);
        return;
    }
    uint8_t *sm = smem_raw + pad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto bar = [&](int i) { return smem_u32(sm + SM_BAR + 8 * i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + SM_TMEM_SLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + SM_ABORT);
    auto fail = [&](int code) {
        *abort_flag = 1;
        if (p.err) atomicCAS(p.err, 0, code);
    };

    // heaviest tiles (longest key ranges) first
    const int qb = gridDim.x - 1 - blockIdx.x;
    const int h = blockIdx.y, kvh = h / (p.Hq / p.Hkv);
    const int t0 = qb * kBM;
    const int tlast = min(t0 + kBM - 1, p.T - 1);
    const int kstart = max(seq_start(p, t0), t0 - p.window + 1);
    const int nkb = (tlast + 1 - kstart + kBN - 1) / kBN;
    // lowest key every row of the tile may see (row lower bounds grow with t)
    const int lo_all = max(seq_start(p, tlast), tlast - p.window + 1);

    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32 * kProducerWarp) {
        mbar_init(bar(BR_Q), 1);
        for (int s = 0; s < kKVStages; ++s) {
            mbar_init(bar(BR_KFULL + s), 1);
            mbar_init(bar(BR_KEMPTY + s), 1);
            mbar_init(bar(BR_VFULL + s), 1);
            mbar_init(bar(BR_VEMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(BR_SFULL + b), 1);
            mbar_init(bar(BR_PREADY + b), 32 * kSoftmaxWarps);
        }
        mbar_init(bar(BR_PVDONE), 1);
        mbar_init(bar(BR_PVDONE + 1), 1);
        mbar_init(bar(BR_FIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mQ);
        tma_prefetch_desc(&mK);
        tma_prefetch_desc(&mV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const uint64_t lim = p.timeout_ns, drain = p.drain_ns;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued_k[kKVStages] = {}, issued_v[kKVStages] = {};
            mbar_arrive_expect_tx(bar(BR_Q), kBlk);
            tma_load_3d(smem_u32(sm + SM_Q), &mQ, 0, h, t0, bar(BR_Q));
            tma_load_3d(smem_u32(sm + SM_Q + kHalf), &mQ, 64, h, t0, bar(BR_Q));
            for (int j = 0; j < nkb; ++j) {
                const int s = j % kKVStages, kb = kstart + j * kBN;
                const uint32_t ph = ((j - kKVStages) / kKVStages) & 1;
                if (j >= kKVStages && !mbar_wait(bar(BR_KEMPTY + s), ph, lim, abort_flag)) { fail(81); break; }
                mbar_arrive_expect_tx(bar(BR_KFULL + s), kBlk);
                tma_load_3d(smem_u32(sm + SM_K + s * kBlk), &mK, 0, kvh, kb, bar(BR_KFULL + s));
                tma_load_3d(smem_u32(sm + SM_K + s * kBlk + kHalf), &mK, 64, kvh, kb, bar(BR_KFULL + s));
                ++issued_k[s];
                if (j >= kKVStages && !mbar_wait(bar(BR_VEMPTY + s), ph, lim, abort_flag)) { fail(82); break; }
                mbar_arrive_expect_tx(bar(BR_VFULL + s), kBlk);
                tma_load_3d(smem_u32(sm + SM_V + s * kBlk), &mV, 0, kvh, kb, bar(BR_VFULL + s));
                tma_load_3d(smem_u32(sm + SM_V + s * kBlk + kHalf), &mV, 64, kvh, kb, bar(BR_VFULL + s));
                ++issued_v[s];
            }
            // no copy may still be landing in shared memory at exit
            const int zero = 0;
            mbar_wait(bar(BR_Q), 0, drain, &zero);
            for (int s = 0; s < kKVStages; ++s) {
                if (issued_k[s]) mbar_wait(bar(BR_KFULL + s), (issued_k[s] - 1) & 1, drain, &zero);
                if (issued_v[s]) mbar_wait(bar(BR_VFULL + s), (issued_v[s] - 1) & 1, drain, &zero);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(kBM, kBN, false, false);   // Q (K-major) x K (K-major)
            const uint32_t id_o = idesc_bf16(kBM, kD, false, true);     // P (TMEM) x V (MN-major)
            const uint64_t dKm = desc_sw128(smem_u32(sm), 16, 1024);    // K-major views (Q, K)
            const uint64_t dMN = desc_sw128(smem_u32(sm), kHalf, 1024); // MN-major view of V
            auto qk = [&](int j) -> bool {
                const int s = j % kKVStages;
                if (!mbar_wait(bar(BR_KFULL + s), (j / kKVStages) & 1, lim, abort_flag)) { fail(83); return false; }
                tc_fence_after();
                const uint32_t kofs = SM_K + s * kBlk;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                    mma_bf16_ss(tm + TM_S + (j & 1) * kBN, dKm + ((SM_Q + off) >> 4), dKm + ((kofs + off) >> 4),
                                id_s, ks > 0);
                }
                mma_commit(bar(BR_SFULL + (j & 1)));
                mma_commit(bar(BR_KEMPTY + s));
                return true;
            };
            bool ok = mbar_wait(bar(BR_Q), 0, lim, abort_flag);
            if (!ok) fail(84);
            if (ok) ok = qk(0);
            if (ok && nkb > 1) ok = qk(1);
            for (int j = 0; ok && j < nkb; ++j) {
                const int s = j % kKVStages, b = j & 1;
                if (!mbar_wait(bar(BR_VFULL + s), (j / kKVStages) & 1, lim, abort_flag)) { fail(85); break; }
                if (!mbar_wait(bar(BR_PREADY + b), (j >> 1) & 1, lim, abort_flag)) { fail(86); break; }
                tc_fence_after();
                const uint32_t vofs = SM_V + s * kBlk;
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks)
                    mma_bf16_ts(tm + TM_O, tm + TM_P + b * (kBN / 2) + 8 * ks, dMN + ((vofs + ks * 2048) >> 4), id_o,
                                (j > 0 || ks > 0) ? 1u : 0u);
                mma_commit(bar(BR_PVDONE + b));
                mma_commit(bar(BR_VEMPTY + s));
                if (j + 2 < nkb) ok = qk(j + 2);
            }
            mma_commit(bar(BR_FIN));   // every issued MMA completes before TMEM is released
            if (!mbar_wait(bar(BR_FIN), 0, lim, abort_flag)) {
                const int zero = 0;
                mbar_wait(bar(BR_FIN), 0, drain, &zero);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax (warps 0-7)
        const int quarter = warp & 3, half = warp >> 2;
        const int r = 32 * quarter + lane;           // query row = TMEM lane
        const int t = t0 + r;
        const bool vrow = t < p.T;
        int lo_t = kstart, hi_t = kstart;   // rows past the end: one key, never stored
        if (vrow) {
            lo_t = max(seq_start(p, t), t - p.window + 1);
            hi_t = t;
        }
        const uint32_t span = static_cast<uint32_t>(hi_t - lo_t);
        const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
        const float c = p.c;
        constexpr unsigned kAll = 0xffffffffu;
        float *xch = reinterpret_cast<float *>(sm + SM_XCH);
        // this row's value from the other half of the pair (a named barrier
        // per lane quarter; two parities keep consecutive exchanges apart)
        auto partner = [&](float v, int parity) -> float {
            xch[(parity * 2 + half) * 128 + r] = v;
            named_bar_sync(1 + quarter, 64);
            return xch[(parity * 2 + (half ^ 1)) * 128 + r];
        };
        // Both halves of a row hold the same m at all times, and the two warps
        // of a pair take the same branches and exchanges: every decision
        // between them is made from exchanged values.  A wait that gives up
        // therefore does not leave the loop (the partner could be waiting at
        // an exchange); with the abort flag set the remaining waits return at
        // once and the results are dropped.
        float m = -INFINITY, l = 0.f;   // l: this half's share of the row sum
        bool ok = true;
        for (int j = 0; j < nkb; ++j) {
            const int b = j & 1, kb = kstart + j * kBN + 64 * half;
            const bool masked = !(kstart + j * kBN + kBN - 1 <= t0 && kstart + j * kBN >= lo_all);
            const int rel = kb - lo_t;   // key kb + i is visible iff (rel + i) in [0, span]
            if (!__all_sync(kAll, mbar_wait(bar(BR_SFULL + b), (j >> 1) & 1, lim, abort_flag))) {
                fail(87);
                ok = false;
            }
            // P buffer b was last read by P_{j-2} V_{j-2}
            if (j >= 2 && !__all_sync(kAll, mbar_wait(bar(BR_PVDONE + b), ((j - 2) >> 1) & 1, lim, abort_flag))) {
                fail(88);
                ok = false;
            }
            tc_fence_after();
            const uint32_t sa = tm + lane_off + TM_S + b * kBN + 64 * half;
            const uint32_t pa = tm + lane_off + TM_P + b * (kBN / 2) + 32 * half;
            float alpha = 1.f;
            bool rescale = false;
            // move m up to mb when that raises it by more than the threshold
            auto raise = [&](float mb) {
                if (mb > m + kRescaleThreshold) {   // also taken when m is still -inf
                    if (m != -INFINITY) {
                        alpha *= ex2_approx(m - mb);
                        rescale = true;
                    }
                    m = mb;
                }
            };
            const bool need_max = __any_sync(kAll, m == -INFINITY);   // the same in both warps of the pair
            if (need_max) {
                // a row without a maximum yet: find this block's first
                float mx = -INFINITY;
#pragma unroll 1
                for (int c4 = 0; c4 < 2; ++c4) {
                    float v[32];
                    tmem_ld32(sa + 32 * c4, v);
                    float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (!masked || static_cast<uint32_t>(rel + 32 * c4 + i) <= span) a[i & 3] = fmaxf(a[i & 3], v[i]);
                    mx = fmaxf(mx, fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])));
                }
                raise(fmaxf(mx, partner(mx, j & 1)) * c);
            }
            // probabilities against the current maximum, written to P chunk by
            // chunk; formed again (rarely) when this block raises the maximum
            // too far
            float sum;
            for (int attempt = 0;; ++attempt) {
                const float msub = (m == -INFINITY) ? 0.f : m;
                float mx = -INFINITY;
                sum = 0.f;
#pragma unroll 1
                for (int c4 = 0; c4 < 2; ++c4) {
                    float v[32];
                    tmem_ld32(sa + 32 * c4, v);
                    uint32_t pk[16];
                    float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY}, sm4[4] = {0.f, 0.f, 0.f, 0.f};
                    if (masked) {
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            float x0 = v[i], x1 = v[i + 1];
                            float p0 = ex2_approx(fmaf(x0, c, -msub)), p1 = ex2_approx(fmaf(x1, c, -msub));
                            if (static_cast<uint32_t>(rel + 32 * c4 + i) > span) { p0 = 0.f; x0 = -INFINITY; }
                            if (static_cast<uint32_t>(rel + 32 * c4 + i + 1) > span) { p1 = 0.f; x1 = -INFINITY; }
                            a[(i >> 1) & 3] = fmaxf(a[(i >> 1) & 3], fmaxf(x0, x1));
                            sm4[(i >> 1) & 3] += p0 + p1;
                            pk[i >> 1] = pack_bf16(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const float p0 = ex2_approx(fmaf(v[i], c, -msub)), p1 = ex2_approx(fmaf(v[i + 1], c, -msub));
                            a[(i >> 1) & 3] = fmaxf(a[(i >> 1) & 3], fmaxf(v[i], v[i + 1]));
                            sm4[(i >> 1) & 3] += p0 + p1;
                            pk[i >> 1] = pack_bf16(p0, p1);
                        }
                    }
                    tmem_st16u(pa + 16 * c4, pk);
                    mx = fmaxf(mx, fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])));
                    sum += (sm4[0] + sm4[1]) + (sm4[2] + sm4[3]);
                }
                // after a max pass, or on the second attempt, m already covers the block
                if (need_max || attempt > 0) break;
                const float mb = fmaxf(mx, partner(mx, j & 1)) * c;
                if (!__any_sync(kAll, mb > m + kRescaleThreshold)) break;   // the same in both warps
                raise(mb);
            }
            l = l * alpha + sum;
            if (__any_sync(kAll, rescale)) {
                // O holds the sum over blocks < j: wait for P_{j-1} V_{j-1}, then scale this half
                if (!__all_sync(kAll, mbar_wait(bar(BR_PVDONE + (b ^ 1)), ((j - 1) >> 1) & 1, lim, abort_flag))) {
                    fail(88);
                    ok = false;
                }
                tc_fence_after();
#pragma unroll 1
                for (int c4 = 0; c4 < 2; ++c4) {
                    const uint32_t oa = tm + lane_off + TM_O + 64 * half + 32 * c4;
                    float v[32];
                    tmem_ld32(oa, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st32(oa, v);
                }
            }
            tc_fence_before();
            mbar_arrive(bar(BR_PREADY + b));
        }
        if (ok && !__all_sync(kAll, mbar_wait(bar(BR_PVDONE + ((nkb - 1) & 1)), ((nkb - 1) >> 1) & 1, lim,
                                               abort_flag)))
            ok = false;
        // the pair meets here in every case and skips the output together
        const bool pair_ok = !named_bar_any(5 + quarter, 64, !ok);
        if (pair_ok) {
            tc_fence_after();
            xch[((nkb & 1) * 2 + half) * 128 + r] = l;
            named_bar_sync(5 + quarter, 64);
            const float inv = 1.f / (l + xch[((nkb & 1) * 2 + (half ^ 1)) * 128 + r]);
            uint4 *dst = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(t) * p.Hq + h) * kD + 64 * half);
#pragma unroll 1
            for (int c4 = 0; c4 < 2; ++c4) {
                float v[32];
                tmem_ld32(tm + lane_off + TM_O + 64 * half + 32 * c4, v);
                if (vrow) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[c4 * 4 + q4] = make_uint4(pack_bf16(v[8 * q4] * inv, v[8 * q4 + 1] * inv),
                                                      pack_bf16(v[8 * q4 + 2] * inv, v[8 * q4 + 3] * inv),
                                                      pack_bf16(v[8 * q4 + 4] * inv, v[8 * q4 + 5] * inv),
                                                      pack_bf16(v[8 * q4 + 6] * inv, v[8 * q4 + 7] * inv));
                }
            }
        } else if (!*abort_flag) {
            fail(89);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, kTmemCols);
    }
}

// ------------------------------------------------------------------ head-pair kernel
//
// For grouped heads (an even number of query heads per key/value head) a CTA
// takes the same 128 tokens of two query heads that read the same key/value
// head, as two tiles A and B.  Every K and V block is loaded once for both,
// and the tensor core works on one tile's products while the other tile's
// softmax runs, so the softmax round trip of one tile no longer leaves the
// tensor pipe idle.
//   warps 0-7  softmax of tile A, warps 8-15 tile B; as in the single-tile
//              kernel, warps w and w + 4 of a tile split the columns of the
//              rows of TMEM lane quarter w%4 and agree on the row maximum
//              through shared memory
//   warp 16    TMA producer (both Q tiles, then K and V through 2-stage rings)
//   warp 17    MMA issuer
// Tensor memory: S_A, S_B (128 columns each) and O_A, O_B (128 each).  The
// column half h of S_X (columns 64h .. 64h + 63) receives, once read, the bf16
// probabilities of its 64 keys in its first 32 columns.  The softmax makes a
// max pass over the block first, so P never has to be formed twice; the
// rescale rule is that of the single-tile kernel.  QK_X(j+1) goes
// into S_X only after P_X(j) V_j has completed, which also means O_X is
// stable whenever the softmax of tile X runs.
constexpr int kPairKV = 2;                       // K and V ring stages
constexpr uint32_t PS_Q = 0;                     // Q_A, Q_B
constexpr uint32_t PS_K = 2 * kBlk;
constexpr uint32_t PS_V = PS_K + kPairKV * kBlk;
constexpr uint32_t PS_BAR = PS_V + kPairKV * kBlk;
enum : int {
    PB_Q = 0,
    PB_KFULL = 1,
    PB_KEMPTY = PB_KFULL + kPairKV,
    PB_VFULL = PB_KEMPTY + kPairKV,
    PB_VEMPTY = PB_VFULL + kPairKV,
    PB_SFULL = PB_VEMPTY + kPairKV,   // + tile
    PB_PREADY = PB_SFULL + 2,         // + tile
    PB_PVDONE = PB_PREADY + 2,        // + tile
    PB_FIN = PB_PVDONE + 2,
    PB_NUM = PB_FIN + 1
};
constexpr uint32_t PS_TMEM_SLOT = PS_BAR + 8 * PB_NUM;
constexpr uint32_t PS_ABORT = PS_TMEM_SLOT + 4;
constexpr uint32_t PS_XCH = PS_BAR + 256;   // [2 tiles][2 parities][2 halves][128 rows] fp32
constexpr uint32_t PS_ALLOC = PS_XCH + 2 * 2 * 2 * 128 * 4;
constexpr size_t kPairSmem = PS_ALLOC + 1024;
static_assert(8 * PB_NUM + 8 <= 256, "barrier area");
static_assert(kPairSmem <= 232448, "shared memory per CTA");
constexpr uint32_t PT_S = 0;      // + 128 * tile
constexpr uint32_t PT_O = 256;    // + 128 * tile
constexpr int kPairSoftmaxWarps = 16;
constexpr int kPairProducerWarp = kPairSoftmaxWarps, kPairMmaWarp = kPairSoftmaxWarps + 1;
constexpr int kPairThreads = 32 * (kPairSoftmaxWarps + 2);

__global__ void __launch_bounds__(kPairThreads, 1)
    swa_fwd_pair_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                        const __grid_constant__ CUtensorMap mV, const SwaParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *sm = smem_raw + pad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto bar = [&](int i) { return smem_u32(sm + PS_BAR + 8 * i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + PS_TMEM_SLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + PS_ABORT);
    auto fail = [&](int code) {
        *abort_flag = 1;
        if (p.err) atomicCAS(p.err, 0, code);
    };

    const int qb = gridDim.x - 1 - blockIdx.x;
    const int h0 = 2 * blockIdx.y, kvh = h0 / (p.Hq / p.Hkv);   // heads h0, h0 + 1 share kvh
    const int t0 = qb * kBM;
    const int tlast = min(t0 + kBM - 1, p.T - 1);
    const int kstart = max(seq_start(p, t0), t0 - p.window + 1);
    const int nkb = (tlast + 1 - kstart + kBN - 1) / kBN;
    const int lo_all = max(seq_start(p, tlast), tlast - p.window + 1);

    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32 * kPairProducerWarp) {
        mbar_init(bar(PB_Q), 1);
        for (int s = 0; s < kPairKV; ++s) {
            mbar_init(bar(PB_KFULL + s), 1);
            mbar_init(bar(PB_KEMPTY + s), 1);
            mbar_init(bar(PB_VFULL + s), 1);
            mbar_init(bar(PB_VEMPTY + s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar(PB_SFULL + x), 1);
            mbar_init(bar(PB_PREADY + x), 32 * kPairSoftmaxWarps / 2);
            mbar_init(bar(PB_PVDONE + x), 1);
        }
        mbar_init(bar(PB_FIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mQ);
        tma_prefetch_desc(&mK);
        tma_prefetch_desc(&mV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const uint64_t lim = p.timeout_ns, drain = p.drain_ns;

    if (warp == kPairProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued_k[kPairKV] = {}, issued_v[kPairKV] = {};
            mbar_arrive_expect_tx(bar(PB_Q), 2 * kBlk);
            for (int x = 0; x < 2; ++x) {
                tma_load_3d(smem_u32(sm + PS_Q + x * kBlk), &mQ, 0, h0 + x, t0, bar(PB_Q));
                tma_load_3d(smem_u32(sm + PS_Q + x * kBlk + kHalf), &mQ, 64, h0 + x, t0, bar(PB_Q));
            }
            for (int j = 0; j < nkb; ++j) {
                const int s = j % kPairKV, kb = kstart + j * kBN;
                const uint32_t ph = ((j - kPairKV) / kPairKV) & 1;
                if (j >= kPairKV && !mbar_wait(bar(PB_KEMPTY + s), ph, lim, abort_flag)) { fail(91); break; }
                mbar_arrive_expect_tx(bar(PB_KFULL + s), kBlk);
                tma_load_3d(smem_u32(sm + PS_K + s * kBlk), &mK, 0, kvh, kb, bar(PB_KFULL + s));
                tma_load_3d(smem_u32(sm + PS_K + s * kBlk + kHalf), &mK, 64, kvh, kb, bar(PB_KFULL + s));
                ++issued_k[s];
                if (j >= kPairKV && !mbar_wait(bar(PB_VEMPTY + s), ph, lim, abort_flag)) { fail(92); break; }
                mbar_arrive_expect_tx(bar(PB_VFULL + s), kBlk);
                tma_load_3d(smem_u32(sm + PS_V + s * kBlk), &mV, 0, kvh, kb, bar(PB_VFULL + s));
                tma_load_3d(smem_u32(sm + PS_V + s * kBlk + kHalf), &mV, 64, kvh, kb, bar(PB_VFULL + s));
                ++issued_v[s];
            }
            const int zero = 0;   // no copy may still be landing in shared memory at exit
            mbar_wait(bar(PB_Q), 0, drain, &zero);
            for (int s = 0; s < kPairKV; ++s) {
                if (issued_k[s]) mbar_wait(bar(PB_KFULL + s), (issued_k[s] - 1) & 1, drain, &zero);
                if (issued_v[s]) mbar_wait(bar(PB_VFULL + s), (issued_v[s] - 1) & 1, drain, &zero);
            }
        }
    } else if (warp == kPairMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(kBM, kBN, false, false);
            const uint32_t id_o = idesc_bf16(kBM, kD, false, true);
            const uint64_t dKm = desc_sw128(smem_u32(sm), 16, 1024);
            const uint64_t dMN = desc_sw128(smem_u32(sm), kHalf, 1024);
            auto qk = [&](int x, int j) {   // S_x = Q_x K_j^T (K_j already waited for)
                const uint32_t kofs = PS_K + (j % kPairKV) * kBlk, qofs = PS_Q + x * kBlk;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                    mma_bf16_ss(tm + PT_S + x * kBN, dKm + ((qofs + off) >> 4), dKm + ((kofs + off) >> 4), id_s,
                                ks > 0);
                }
                mma_commit(bar(PB_SFULL + x));
            };
            auto pv = [&](int x, int j) {   // O_x += P_x V_j (keys 0..63 in columns 0..31, 64..127 in 64..95)
                const uint32_t vofs = PS_V + (j % kPairKV) * kBlk;
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks)
                    mma_bf16_ts(tm + PT_O + x * kD, tm + PT_S + x * kBN + (ks >> 2) * 64 + (ks & 3) * 8,
                                dMN + ((vofs + ks * 2048) >> 4), id_o, (j > 0 || ks > 0) ? 1u : 0u);
                mma_commit(bar(PB_PVDONE + x));
            };
            bool ok = mbar_wait(bar(PB_Q), 0, lim, abort_flag) && mbar_wait(bar(PB_KFULL), 0, lim, abort_flag);
            if (!ok) fail(93);
            if (ok) {
                tc_fence_after();
                qk(0, 0);
                qk(1, 0);
                mma_commit(bar(PB_KEMPTY));
            }
            for (int j = 0; ok && j < nkb; ++j) {
                const int s = j % kPairKV, sn = (j + 1) % kPairKV;
                const uint32_t par = j & 1;
                const bool more = j + 1 < nkb;
                for (int x = 0; x < 2; ++x) {
                    if (!mbar_wait(bar(PB_PREADY + x), par, lim, abort_flag)) { fail(94); ok = false; break; }
                    if (x == 0 && !mbar_wait(bar(PB_VFULL + s), (j / kPairKV) & 1, lim, abort_flag)) {
                        fail(95);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    pv(x, j);
                    if (x == 1) mma_commit(bar(PB_VEMPTY + s));
                    if (more) {
                        if (x == 0 && !mbar_wait(bar(PB_KFULL + sn), ((j + 1) / kPairKV) & 1, lim, abort_flag)) {
                            fail(96);
                            ok = false;
                            break;
                        }
                        // S_x is overwritten only after P_x V_j has read it
                        if (!mbar_wait(bar(PB_PVDONE + x), par, lim, abort_flag)) { fail(97); ok = false; break; }
                        tc_fence_after();
                        qk(x, j + 1);
                        if (x == 1) mma_commit(bar(PB_KEMPTY + sn));
                    }
                }
            }
            mma_commit(bar(PB_FIN));
            if (!mbar_wait(bar(PB_FIN), 0, lim, abort_flag)) {
                const int zero = 0;
                mbar_wait(bar(PB_FIN), 0, drain, &zero);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax (warps 0-15)
        const int x = warp >> 3, quarter = warp & 3, half = (warp >> 2) & 1;
        const int r = 32 * quarter + lane;
        const int t = t0 + r;
        const bool vrow = t < p.T;
        int lo_t = kstart, hi_t = kstart;
        if (vrow) {
            lo_t = max(seq_start(p, t), t - p.window + 1);
            hi_t = t;
        }
        const uint32_t span = static_cast<uint32_t>(hi_t - lo_t);
        const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
        const uint32_t sa = tm + lane_off + PT_S + x * kBN + 64 * half;
        const uint32_t oa = tm + lane_off + PT_O + x * kD + 64 * half;
        const float c = p.c;
        constexpr unsigned kAll = 0xffffffffu;
        float *xch = reinterpret_cast<float *>(sm + PS_XCH) + x * (2 * 2 * 128);
        const int bar_id = 1 + 4 * x + quarter;
        // the row's value from the other column half (two parities keep
        // consecutive exchanges apart); both warps of a pair call this the
        // same number of times, whatever happens to their waits
        auto partner = [&](float v, int parity) -> float {
            xch[(parity * 2 + half) * 128 + r] = v;
            named_bar_sync(bar_id, 64);
            return xch[(parity * 2 + (half ^ 1)) * 128 + r];
        };
        float m = -INFINITY, l = 0.f;   // m: the same in both halves of a row; l: this half's share
        bool ok = true;
        for (int j = 0; j < nkb; ++j) {
            const int kb0 = kstart + j * kBN;
            const bool masked = !(kb0 + kBN - 1 <= t0 && kb0 >= lo_all);
            const int rel = kb0 + 64 * half - lo_t;
            // S_x(j) written (which also means P_x(j-1) V_{j-1} has completed)
            if (!__all_sync(kAll, mbar_wait(bar(PB_SFULL + x), j & 1, lim, abort_flag))) {
                fail(98);
                ok = false;
            }
            tc_fence_after();
            float mx = -INFINITY;
#pragma unroll 1
            for (int c4 = 0; c4 < 2; ++c4) {
                float v[32];
                tmem_ld32(sa + 32 * c4, v);
                float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (masked) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (static_cast<uint32_t>(rel + 32 * c4 + i) <= span) a[i & 3] = fmaxf(a[i & 3], v[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) a[i & 3] = fmaxf(a[i & 3], v[i]);
                }
                mx = fmaxf(mx, fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])));
            }
            const float mb = fmaxf(mx, partner(mx, j & 1)) * c;
            float alpha = 1.f;
            bool rescale = false;
            if (mb > m + kRescaleThreshold) {
                if (m != -INFINITY) {
                    alpha = ex2_approx(m - mb);
                    rescale = true;
                }
                m = mb;
            }
            const float msub = (m == -INFINITY) ? 0.f : m;
            float sum = 0.f;
            // P chunk c4 of this half goes over its columns 16 c4 .. 16 c4 + 15, read by then
#pragma unroll 1
            for (int c4 = 0; c4 < 2; ++c4) {
                float v[32];
                tmem_ld32(sa + 32 * c4, v);
                uint32_t pk[16];
                float sm4[4] = {0.f, 0.f, 0.f, 0.f};
                if (masked) {
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float p0 = ex2_approx(fmaf(v[i], c, -msub)), p1 = ex2_approx(fmaf(v[i + 1], c, -msub));
                        if (static_cast<uint32_t>(rel + 32 * c4 + i) > span) p0 = 0.f;
                        if (static_cast<uint32_t>(rel + 32 * c4 + i + 1) > span) p1 = 0.f;
                        sm4[(i >> 1) & 3] += p0 + p1;
                        pk[i >> 1] = pack_bf16(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const float p0 = ex2_approx(fmaf(v[i], c, -msub)), p1 = ex2_approx(fmaf(v[i + 1], c, -msub));
                        sm4[(i >> 1) & 3] += p0 + p1;
                        pk[i >> 1] = pack_bf16(p0, p1);
                    }
                }
                tmem_st16u(sa + 16 * c4, pk);
                sum += (sm4[0] + sm4[1]) + (sm4[2] + sm4[3]);
            }
            l = l * alpha + sum;
            if (__any_sync(kAll, rescale)) {
#pragma unroll 1
                for (int c4 = 0; c4 < 2; ++c4) {
                    float v[32];
                    tmem_ld32(oa + 32 * c4, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= alpha;
                    tmem_st32(oa + 32 * c4, v);
                }
            }
            tc_fence_before();
            mbar_arrive(bar(PB_PREADY + x));
        }
        if (ok && !__all_sync(kAll, mbar_wait(bar(PB_PVDONE + x), (nkb - 1) & 1, lim, abort_flag))) {
            fail(99);
            ok = false;
        }
        // the halves' row sums (an exchange both warps always make)
        xch[((nkb & 1) * 2 + half) * 128 + r] = l;
        named_bar_sync(bar_id, 64);
        const float lsum = l + xch[((nkb & 1) * 2 + (half ^ 1)) * 128 + r];
        if (ok) {
            tc_fence_after();
            const float inv = 1.f / lsum;
            uint4 *dst = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(t) * p.Hq + h0 + x) * kD + 64 * half);
#pragma unroll 1
            for (int c4 = 0; c4 < 2; ++c4) {
                float v[32];
                tmem_ld32(oa + 32 * c4, v);
                if (vrow) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[c4 * 4 + q4] = make_uint4(pack_bf16(v[8 * q4] * inv, v[8 * q4 + 1] * inv),
                                                      pack_bf16(v[8 * q4 + 2] * inv, v[8 * q4 + 3] * inv),
                                                      pack_bf16(v[8 * q4 + 4] * inv, v[8 * q4 + 5] * inv),
                                                      pack_bf16(v[8 * q4 + 6] * inv, v[8 * q4 + 7] * inv));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, kTmemCols);
    }
}

// ------------------------------------------------------------------ RoPE

constexpr int kRopeThreads = 256;

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    using type = float4;
    __device__ static void load(const float *p, float (&x)[4]) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    __device__ static void store(float *p, const float (&x)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};
template <> struct Vec4<__nv_bfloat16> {
    __device__ static void load(const __nv_bfloat16 *p, float (&x)[4]) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&v.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&v.y);
        x[0] = __low2float(a); x[1] = __high2float(a); x[2] = __low2float(b); x[3] = __high2float(b);
    }
    __device__ static void store(__nv_bfloat16 *p, const float (&x)[4]) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(sm100::pack_bf16(x[0], x[1]), sm100::pack_bf16(x[2], x[3]));
    }
};

// Rotate-half RoPE.  A thread owns 4 consecutive pairs (i, i + d/2) of one
// token and rotates them in every head, so each angle is formed once per
// token: p * theta_i is computed and reduced to [-pi, pi] in double
// (theta_i = base^(-2i/d) kept per block in shared memory), so the fp32 sine
// and cosine see an exact argument even at positions of 10^5 and beyond.
// Tokens are walked grid-stride.
template <typename T>
__global__ void __launch_bounds__(kRopeThreads)
    rope_kernel(const T *__restrict__ x, T *out, const int32_t *__restrict__ cu, int num_seqs, int64_t uniform_len,
                int64_t tokens, int H, int d, int offset, double log2_base) {
    __shared__ double theta[128];
    const int half = d >> 1, groups = half >> 2;
    for (int i = threadIdx.x; i < half; i += blockDim.x) theta[i] = exp2(-(2.0 * i / d) * log2_base);
    __syncthreads();
    const int tok_per_block = kRopeThreads / groups;
    const int g = threadIdx.x % groups, tb = threadIdx.x / groups;
    if (tb >= tok_per_block) return;
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    for (int64_t t = (int64_t)blockIdx.x * tok_per_block + tb; t < tokens; t += (int64_t)gridDim.x * tok_per_block) {
        int64_t bos;
        if (cu) {
            int a = 0, b = num_seqs;   // cu[a] <= t < cu[b]
            while (b - a > 1) {
                const int mid = (a + b) >> 1;
                if (__ldg(cu + mid) <= t) a = mid;
                else b = mid;
            }
            bos = __ldg(cu + a);
        } else {
            bos = t - t % uniform_len;
        }
        const double pos = static_cast<double>(t - bos + offset);
        float cs[4], sn[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double ang = pos * theta[4 * g + e];
            sincosf(static_cast<float>(ang - kTwoPi * rint(ang / kTwoPi)), &sn[e], &cs[e]);
        }
        const T *src = x + t * H * d + 4 * g;
        T *dst = out + t * H * d + 4 * g;
        for (int h = 0; h < H; ++h, src += d, dst += d) {
            float x1[4], x2[4], y1[4], y2[4];
            Vec4<T>::load(src, x1);
            Vec4<T>::load(src + half, x2);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                y1[e] = x1[e] * cs[e] - x2[e] * sn[e];
                y2[e] = x2[e] * cs[e] + x1[e] * sn[e];
            }
            Vec4<T>::store(dst, y1);
            Vec4<T>::store(dst + half, y2);
        }
    }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tensor_map_encoder() {
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

// [T, H, 128] bf16 as 3-D (d, H, T); box (64, 1, 128), 128-byte swizzle,
// rows past T read as zeros.
bool make_head_map(CUtensorMap *m, const void *base, int T, int H) {
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kBN};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t swa_setup() {
    static bool done[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(swa_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSwaSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(swa_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPairSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) done[dev] = true;
    return cudaSuccess;
}

cudaError_t launch_swa(const SwaLaunch &L, cudaStream_t stream) {
    if (L.total_tokens == 0) return cudaSuccess;
    cudaError_t e = swa_setup();
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv;
    const int T = static_cast<int>(L.total_tokens);
    if (!make_head_map(&mq, L.q, T, L.Hq) || !make_head_map(&mk, L.k, T, L.Hkv) || !make_head_map(&mv, L.v, T, L.Hkv))
        return cudaErrorInvalidValue;
    SwaParams p;
    p.o = static_cast<__nv_bfloat16 *>(L.o);
    p.cu = L.cu_seqlens;
    p.uniform_len = L.cu_seqlens ? 1 : L.total_tokens / L.num_seqs;
    p.num_seqs = L.num_seqs;
    p.T = T;
    p.Hq = L.Hq;
    p.Hkv = L.Hkv;
    p.window = L.window;
    p.c = L.scale * kLog2e;
    p.err = L.err;
    p.timeout_ns = L.timeout_ns;
    p.drain_ns = L.drain_ns;
    if ((L.Hq / L.Hkv) % 2 == 0) {   // head pairs that share a key/value head
        const dim3 grid((T + kBM - 1) / kBM, L.Hq / 2);
        swa_fwd_pair_kernel<<<grid, kPairThreads, kPairSmem, stream>>>(mq, mk, mv, p);
    } else {
        const dim3 grid((T + kBM - 1) / kBM, L.Hq);
        swa_fwd_kernel<<<grid, kThreads, kSwaSmem, stream>>>(mq, mk, mv, p);
    }
    return cudaGetLastError();
}

cudaError_t launch_rope(int dtype, const void *x, void *out, const int32_t *cu_seqlens, int num_seqs,
                        int64_t total_tokens, int H, int d, int offset, double base, cudaStream_t stream) {
    if (total_tokens == 0 || H == 0) return cudaSuccess;
    const int groups = d / 8, tok_per_block = kRopeThreads / groups;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (total_tokens + tok_per_block - 1) / tok_per_block;
    const int64_t cap = (int64_t)sms * 8;
    if (blocks > cap) blocks = cap;
    const int64_t uniform_len = cu_seqlens ? 1 : total_tokens / num_seqs;
    const double lb = log2(base);
    if (dtype == GDN_BF16)
        rope_kernel<__nv_bfloat16><<<(unsigned)blocks, kRopeThreads, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(out), cu_seqlens, num_seqs,
            uniform_len, total_tokens, H, d, offset, lb);
    else
        rope_kernel<float><<<(unsigned)blocks, kRopeThreads, 0, stream>>>(static_cast<const float *>(x),
                                                                           static_cast<float *>(out), cu_seqlens,
                                                                           num_seqs, uniform_len, total_tokens, H, d, offset,
                                                                           lb);
    return cudaGetLastError();
}

}  // namespace gdn
