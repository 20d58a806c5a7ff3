/*
 * gdn.h -- C ABI of the B200 Gated DeltaNet hot path (libgdn.so).
 *
 * The operation.  InfiniteVL's linear-complexity token mixer is Gated
 * DeltaNet (InfiniteVL explainer page, "Gated DeltaNet" concept box and
 * "Building Blocks": a fixed-size memory matrix per head, a gate on the old
 * memory, an erase along the key, a write, a read with the query; 16 heads
 * per layer, "Step 2").  Per sequence and head, token by token:
 *
 *     alpha_t = exp(g_t)
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t                       (read-out after the write)
 *
 * S is d_v x d_k (fp32).  Nothing else is applied: no 1/sqrt(d_k) scale, no
 * L2 norm, no short convolution, no output gate -- the caller passes q, k, v
 * (normalised as it wishes), g = log(alpha) and beta.
 *
 * Streaming with a carried state (InfiniteVL project page, "Accelerated
 * Streaming Inference": the linear memory state is updated on the fly with a
 * constant-size cache) is the state_in / state_out pair of gdn_prefill:
 * running a sequence in segments with the state carried gives the result of
 * one run.  gdn_decode_step is the same recurrence for one token per
 * sequence.
 *
 * Conventions shared by every entry point:
 *  - All data pointers are DEVICE pointers (cu_seqlens and the workspace
 *    included).  The caller owns every buffer; the library allocates nothing
 *    and keeps no pointer after a call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    is the legacy default stream).  Host-side argument errors are returned
 *    before anything is enqueued.  A launch failure returns GDN_ERR_CUDA.
 *    The library never synchronises the device.
 *  - Layouts are contiguous and row-major.  Every base pointer must be 16-byte
 *    aligned (GDN_ERR_INVALID_ARG otherwise).
 *  - Inputs are never written.
 *  - The kernels require finite inputs, g <= 0 and beta in [0, 1]; the sum of g
 *    over any 64 consecutive tokens of a sequence must stay above -80 (the
 *    chunkwise prefill forms exp(G_r - G_i) inside a chunk).  Nothing on the
 *    device checks this; results for other inputs are unspecified.
 *
 * Thread safety: entry points keep no mutable global state apart from a
 * one-time per-device kernel attribute set-up, and may be called from several
 * host threads on different streams.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes of every entry point. */
typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad cu_seqlens length */
    GDN_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement (dk, dv, chunk, dtype) */
    GDN_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
    GDN_ERR_TIMEOUT = 4,       /* a wait inside a kernel gave up (gdn_read_status) */
    GDN_ERR_WORKSPACE = 5      /* workspace NULL or smaller than gdn_prefill_workspace_size() */
} gdn_status;

/* Storage type of q, k, v and out.  g, beta and the state are always fp32. */
typedef enum gdn_dtype {
    GDN_F32 = 0,               /* fp32 in and out; fp32 arithmetic throughout (SIMT) */
    GDN_BF16 = 1               /* bf16 in and out; bf16 tensor-core operands, fp32 accumulation and state */
} gdn_dtype;

/*
 * Bytes of device workspace gdn_prefill needs for these sizes (0 is possible).
 * Pure host arithmetic; never touches the device.  Returns 0 for arguments
 * gdn_prefill would reject.
 */
size_t gdn_prefill_workspace_size(int num_seqs, int64_t total_tokens, int H,
                                  int dk, int dv, int chunk, int dtype);

/*
 * Chunkwise-parallel prefill over a packed batch of num_seqs sequences.
 *
 *   q, k        [total_tokens, H, dk]   dtype
 *   v           [total_tokens, H, dv]   dtype
 *   g, beta     [total_tokens, H]       fp32  (g = log alpha)
 *   state_in    [num_seqs, H, dv, dk]   fp32, or NULL for a zero initial state
 *   out         [total_tokens, H, dv]   dtype (written)
 *   state_out   [num_seqs, H, dv, dk]   fp32 final states (written), or NULL
 *   cu_seqlens  [num_seqs + 1]          int32, device; cu_seqlens[0] = 0,
 *               non-decreasing, cu_seqlens[num_seqs] = total_tokens; empty
 *               sequences are allowed (their state_out = state_in).  NULL means
 *               num_seqs sequences of total_tokens / num_seqs tokens each
 *               (must divide exactly).
 *   chunk       64 (the only chunk length implemented)
 *   workspace   device scratch of at least gdn_prefill_workspace_size() bytes
 *               (may be NULL when that size is 0); contents need not be
 *               initialised and are garbage afterwards.
 *
 * state_out may equal state_in exactly (in-place update); other overlaps, and
 * any overlap of out with an input, are not allowed.  Supported: dk = dv in
 * {64, 128}; dtype GDN_F32 or GDN_BF16.  total_tokens may be 0 (nothing is
 * launched except the state copy).  The device contents of cu_seqlens are
 * trusted (not validated).
 */
int gdn_prefill(const void *q, const void *k, const void *v, const float *g,
                const float *beta, const float *state_in, void *out,
                float *state_out, const int32_t *cu_seqlens, int num_seqs,
                int64_t total_tokens, int H, int dk, int dv, int chunk,
                int dtype, void *workspace, size_t workspace_bytes,
                void *stream);

/*
 * One recurrent decode step: one new token for each of B sequences.
 *
 *   q, k        [B, H, dk]   dtype
 *   v           [B, H, dv]   dtype
 *   g, beta     [B, H]       fp32
 *   state_in    [B, H, dv, dk] fp32 (read)
 *   state_out   [B, H, dv, dk] fp32 (written); may equal state_in (in place)
 *   out         [B, H, dv]   dtype (written)
 *
 * Reads and writes each state exactly once (bandwidth bound).  Supported:
 * dk = dv in {64, 128}; dtype GDN_F32 or GDN_BF16.  B = 0 is a no-op.
 */
int gdn_decode_step(const void *q, const void *k, const void *v,
                    const float *g, const float *beta, const float *state_in,
                    float *state_out, void *out, int B, int H, int dk, int dv,
                    int dtype, void *stream);

/*
 * Number of kernel launches gdn_prefill makes for these sizes on the current
 * device (0 for arguments it would reject); `packed` is nonzero when
 * cu_seqlens will be passed.  Host-side only (it may query the device's SM
 * count); lets callers account for the library's launches inside a CUDA graph
 * or a timed region.
 */
int gdn_prefill_kernel_count(int num_seqs, int64_t total_tokens, int H, int dk, int dv,
                             int chunk, int dtype, int packed);

/*
 * gdn_prefill_noalloc -- gdn_prefill for callers that cannot allocate device
 * memory (for instance a serving loop that reserves all of its device memory
 * at start-up and forbids any later cudaMalloc, or a host that cannot pass the
 * library a workspace pointer).  The InfiniteVL pages have no counterpart: it
 * changes only where the scratch lives, not what is computed.
 *
 * Arguments, layouts, results and status codes are those of gdn_prefill,
 * without the workspace pair.  The scratch is one array of
 * GDN_NOALLOC_SCRATCH_BYTES compiled into libgdn.so, which every GPU that
 * loads the library holds until the process exits.  Requests whose
 * gdn_prefill_workspace_size() exceeds it return GDN_ERR_WORKSPACE before
 * anything is enqueued (16 MiB covers, e.g., 16 heads x 1024 tokens in one
 * sequence); shapes that need no workspace are not limited.
 *
 * The function calls no cudaMalloc, cudaFree or other allocating routine.  The
 * first call on a device looks the array's device address up (with that
 * device current) and caches it.  Every call on a device shares the one
 * array: calls whose work
 * overlaps on the GPU (different streams, or other host threads) race on it
 * and must be serialised by the caller.  Each call clears what has to start
 * at zero, so stale contents from an earlier call are harmless.
 */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int gdn_prefill_noalloc(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *state_in, void *out,
                        float *state_out, const int32_t *cu_seqlens, int num_seqs,
                        int64_t total_tokens, int H, int dk, int dv, int chunk,
                        int dtype, void *stream);

/*
 * Status word of gdn_prefill_noalloc on the current device.  The tensor-core
 * kernels of a no-alloc call record a wait that gave up in the first int32 of
 * the library's scratch array, whose address callers cannot see; this reads
 * that word exactly as gdn_read_status reads a caller's workspace: it waits
 * for `stream`, returns GDN_OK when the word is 0 and GDN_ERR_TIMEOUT
 * otherwise, and stores the word in *code (may be NULL).  Read it before the
 * next no-alloc call on the device, which clears the word.  Like the
 * no-alloc call itself it allocates nothing; it synchronises with `stream`.
 */
int gdn_noalloc_read_status(void *stream, int32_t *code);

/* Static, human-readable name of a gdn_status value. */
const char *gdn_status_string(int status);

/*
 * Device status word of the tensor-core kernels.  Every wait inside them
 * (on a copy, an MMA or another role of the CTA) gives up after 2 s; the
 * kernel then records a nonzero code in a device int32 and returns, leaving
 * its outputs invalid but the GPU usable.  The word is the first int32 of the
 * workspace of gdn_prefill (and of a session's workspace; cleared by every
 * call that uses the tensor-core path) and the `status` argument of
 * gdn_swa_attention (cleared by the caller).
 *
 * gdn_read_status waits for `stream`, then reads the int32 at `word` (device,
 * 4-byte aligned): GDN_OK if it is 0, GDN_ERR_TIMEOUT otherwise; *code (may
 * be NULL) receives the word.  It is the one entry point that synchronises.
 */
int gdn_read_status(const int32_t *word, void *stream, int32_t *code);

/*
 * Test hook of those bounded waits.  Sets, for the calling host thread, the
 * bound on the waits of the work loops of the tensor-core kernels that its
 * later calls launch (gdn_prefill, gdn_prefill_noalloc, gdn_swa_attention,
 * and the prefill steps a session captures).  With ns = 0 a wait gives up as
 * soon as the phase it waits for is not already complete, so a call's first
 * wait on a copy or an MMA in flight gives up; GDN_WAIT_LIMIT_DEFAULT
 * restores the 2 s default.  Whatever the bound, the waits that drain a
 * kernel's copies and MMAs before it exits keep 2 s: a kernel whose waits
 * gave up records its code in the status word and returns with no work in
 * flight and its outputs invalid, and later calls on the device run normally.
 */
#define GDN_WAIT_LIMIT_DEFAULT ((uint64_t)2000000000)
void gdn_set_wait_limit(uint64_t ns);

/* Text of the most recent CUDA error seen by this host thread inside the
 * library ("" if none).  Valid until the next call on this thread. */
const char *gdn_last_cuda_error(void);

/* ------------------------------------------------------------------ layer steps around the recurrence
 *
 * The explainer page (InfiniteVL, "Step 2: Process tokens with Hybrid
 * Blocks") gives every Gated DeltaNet layer a 1-D convolution of window 4 and
 * an output gate, and fixes nothing else about them.  These two entry points
 * take the plainest reading: the convolution is causal and depthwise over the
 * q, k and v channels (restarted at each sequence start), q and k are then
 * L2-normalised, beta = sigmoid(b) and g = log(sigmoid(a)); the output gate is
 * y = n(o) * act(z).  Conventions are those above (device pointers, 16-byte
 * alignment, asynchronous, no allocation).
 */

typedef enum gdn_activation { GDN_ACT_NONE = 0, GDN_ACT_SILU = 1 } gdn_activation;
typedef enum gdn_gate { GDN_GATE_SIGMOID = 0, GDN_GATE_SILU = 1 } gdn_gate;

/*
 * From a layer's raw projections to gdn_prefill's inputs, per (token, head):
 *
 *   y_X[t] = act( sum_{i=0..3} conv_w[X][h][c][i] * x_X[t - 3 + i] )
 *            for X = q, k, v; positions before a sequence's first token come
 *            from conv_state_in (slot j = position start - 3 + j), or are 0
 *   q = y_q / sqrt(sum_c y_q^2 + eps),   k likewise,   v = y_v
 *   g = log(sigmoid(a)) = -softplus(-a),   beta = sigmoid(b)
 *
 *   xq, xk, xv     [total_tokens, H, d]  dtype  raw projections
 *   conv_w         [3, H, d, 4]          fp32   (q, k, v; tap 3 = current token)
 *   a_logit, b_logit [total_tokens, H]   fp32
 *   conv_state_in  [num_seqs, 3, 3, H, d] dtype (slot, tensor, head, channel),
 *                  or NULL for zeros
 *   q, k, v        [total_tokens, H, d]  dtype (written)
 *   g, beta        [total_tokens, H]     fp32  (written)
 *   conv_state_out [num_seqs, 3, 3, H, d] dtype (written: the raw inputs at the
 *                  last three positions of each sequence, older ones from
 *                  conv_state_in when a sequence is shorter), or NULL; it may
 *                  equal conv_state_in (in-place update)
 *   cu_seqlens     as in gdn_prefill (NULL: num_seqs equal sequences)
 *   activation     GDN_ACT_NONE or GDN_ACT_SILU (applied after the convolution)
 *   eps            in [0, 1]
 *
 * With cu_seqlens = [0, 1, ..., B] this is the per-token step of decoding.
 * Supported: d in {64, 128}, dtype GDN_F32 or GDN_BF16.  Outputs may not
 * overlap inputs or each other (GDN_ERR_INVALID_ARG).
 */
int gdn_preprocess(const void *xq, const void *xk, const void *xv, const float *conv_w,
                   const float *a_logit, const float *b_logit, const void *conv_state_in, void *q,
                   void *k, void *v, float *g, float *beta, void *conv_state_out,
                   const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens, int H, int d,
                   int activation, float eps, int dtype, void *stream);

/*
 * Output gate over rows of d_v values (rows = tokens x heads):
 *
 *   n = o                                        if norm_w is NULL
 *   n = o / sqrt(mean_c o^2 + eps) * norm_w[c]   otherwise (RMS norm per row)
 *   y = n * sigmoid(z)   (GDN_GATE_SIGMOID)   or   n * z * sigmoid(z)   (GDN_GATE_SILU)
 *
 *   o, z, y   [rows, dv] dtype;  norm_w [dv] fp32 or NULL.
 * y may equal o (in place); no other overlap.  Supported: dv in {64, 128}.
 */
int gdn_output_gate(const void *o, const void *z, const float *norm_w, void *y, int64_t rows, int dv,
                    int gate, float eps, int dtype, void *stream);

/*
 * One Gated DeltaNet layer's token mixer over a packed batch, from the raw
 * projections to the gated output: gdn_preprocess, gdn_prefill and
 * gdn_output_gate in one call, with their arguments and their results (up to
 * the rounding order of sums):
 *
 *   (q, k, v, g, beta) = pre-processing of (xq, xk, xv, a_logit, b_logit)
 *   (o, state_out)     = the chunkwise recurrence from state_in
 *   y                  = n(o) * act(z)
 *
 * On the tensor-core path (GDN_BF16, d = 128, total_tokens > 0) the steps
 * are fused: the chunk-prep kernel forms q, k, v, g and beta from its chunk's
 * raw projections and leaves them in the workspace for the state and output
 * passes (q already scaled, row by row, by the decay exp(G_t) from the start
 * of its 64-token chunk, the form the output pass consumes), and the output
 * pass writes y in place of o.  Otherwise the three steps run one after
 * another through the workspace.
 *
 *   xq, xk, xv, conv_w, a_logit, b_logit, conv_state_in, conv_state_out,
 *   activation   as in gdn_preprocess (conv_state_out may equal
 *                conv_state_in, or be NULL)
 *   state_in, state_out, cu_seqlens, num_seqs, total_tokens, H   as in
 *                gdn_prefill, with d_k = d_v = d (state_out may equal
 *                state_in, or be NULL)
 *   z            [total_tokens, H, d] dtype; norm_w [d] fp32 or NULL; gate
 *                as in gdn_output_gate
 *   y            [total_tokens, H, d] dtype (written)
 *   eps          of the q/k L2 norm and of the RMS norm, in [0, 1]
 *   workspace    gdn_layer_prefill_workspace_size(...) bytes, 16-byte aligned,
 *                owned by the caller; its first int32 is the status word of
 *                the tensor-core kernels (gdn_read_status)
 * y, the workspace and the output states may not overlap the inputs or one
 * another, except that each state may be updated in place
 * (GDN_ERR_INVALID_ARG).  Supported: d in {64, 128}; dtype GDN_F32 or
 * GDN_BF16.
 */
size_t gdn_layer_prefill_workspace_size(int num_seqs, int64_t total_tokens, int H, int d, int dtype);
int gdn_layer_prefill(const void *xq, const void *xk, const void *xv, const float *conv_w,
                      const float *a_logit, const float *b_logit, const void *conv_state_in,
                      void *conv_state_out, const float *state_in, float *state_out, const void *z,
                      const float *norm_w, void *y, const int32_t *cu_seqlens, int num_seqs,
                      int64_t total_tokens, int H, int d, int activation, int gate, float eps,
                      int dtype, void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------ sliding-window attention
 *
 * The hybrid block's other token mixer (InfiniteVL explainer page, "Step 2:
 * Process tokens with Hybrid Blocks" and the "Sliding Window Attention"
 * concept box): softmax attention restricted to a recent window of tokens
 * (8K), with rotary positions and grouped-query heads (16 query heads, 2
 * key/value heads).  Readings taken where the page is silent: the window
 * counts tokens and includes the query token itself; RoPE is the rotate-half
 * form at the token's position inside its sequence.
 */

/*
 * Rotate-half RoPE over rows of d values (rows = tokens x heads):
 *
 *   p = (position of the token inside its sequence) + pos_offset
 *   theta_i = base^(-2i/d),  a = p * theta_i,  for i < d/2:
 *   out[i]       = x[i] cos a - x[i + d/2] sin a
 *   out[i + d/2] = x[i + d/2] cos a + x[i] sin a
 *
 *   x, out       [total_tokens, H, d] dtype; out may equal x (in place), no
 *                other overlap
 *   cu_seqlens   as in gdn_prefill (NULL: num_seqs equal sequences)
 *   pos_offset   >= 0, added to every position (a stream's tokens seen so far)
 *   base         > 1 (10000 is the usual choice)
 * The angle is reduced in double precision before the fp32 sine and cosine.
 * Supported: d a multiple of 8 in [8, 256]; dtype GDN_F32 or GDN_BF16.
 */
int gdn_rope(const void *x, void *out, const int32_t *cu_seqlens, int num_seqs, int64_t total_tokens, int H, int d,
             int pos_offset, float base, int dtype, void *stream);

/*
 * Causal sliding-window attention with grouped key/value heads, per sequence:
 *
 *   o[t, h] = sum_s softmax_s(scale * q[t, h] . k[s, h / (Hq / Hkv)]) v[s, h / (Hq / Hkv)]
 *   over the keys s of t's sequence with t - window < s <= t
 *
 *   q        [total_tokens, Hq, d]   bf16 (already rotated)
 *   k, v     [total_tokens, Hkv, d]  bf16 (k already rotated)
 *   o        [total_tokens, Hq, d]   bf16 (written; may not overlap q, k, v)
 *   cu_seqlens  as in gdn_prefill (NULL: num_seqs equal sequences)
 *   window   >= 1 tokens;  scale > 0, or 0 for 1/sqrt(d)
 *   status   device int32 or NULL: set to a nonzero code (left as is
 *            otherwise; the caller clears it) when a wait inside the kernel
 *            gave up after 2 s, in which case o is not valid
 * Scores and the row sums are fp32; the probabilities enter the P V product
 * as bf16.  Supported: dtype GDN_BF16, d = 128, Hq a multiple of Hkv,
 * Hq <= 65535, total_tokens < 2^31 - 256.
 */
int gdn_swa_attention(const void *q, const void *k, const void *v, void *o, const int32_t *cu_seqlens,
                      int num_seqs, int64_t total_tokens, int Hq, int Hkv, int d, int window, float scale,
                      int dtype, int32_t *status, void *stream);

/* ------------------------------------------------------------------ streaming session
 *
 * One Gated DeltaNet layer step over a constant-size memory, captured as a
 * CUDA graph and replayed (InfiniteVL project page, "Advanced Usage: CUDA
 * Graph Acceleration" and "Accelerated Streaming Inference": the fixed-size
 * state lets the whole streaming-prefill computation, and the decode step,
 * be captured once and replayed without launch overhead; a video is fed
 * segment by segment while the state is carried).
 *
 * A step, for each of num_streams independent streams, with the convolution
 * and recurrent states carried in place:
 *   tokens > 0:  gdn_layer_prefill (pre-processing, recurrence and output
 *                gate; fused on the tensor-core path);
 *   one token:   gdn_preprocess -> gdn_decode_step -> gdn_output_gate.
 *
 * The caller owns every buffer and keeps it in place for the session's
 * lifetime (the graphs hold the addresses).  Sizes, with R = num_streams *
 * seg_tokens rows:
 *   xq, xk, xv, z, y, q, k, v, o   [R, H, d] dtype
 *   a, b, g, beta                  [R, H] fp32
 *   state                          [num_streams, H, d, d] fp32
 *   conv_state                     [num_streams, 3, 3, H, d] dtype
 *   conv_w [3, H, d, 4] fp32;  norm_w [d] fp32 or NULL (no RMS norm)
 *   workspace                      gdn_session_workspace_size() bytes
 * Per step the caller writes xq, xk, xv, a, b, z for `tokens` tokens of every
 * stream, stream-major ([num_streams][tokens] at the start of each buffer),
 * and reads y in the same layout; q, k, v, o, g, beta are scratch.  The
 * decode step uses one row per stream.
 *
 * gdn_session_create allocates no device memory: it checks the buffers, runs
 * the kernels' one-time per-device set-up and creates a capture stream.  The
 * first step for a token count captures its graph (up to 8 counts are kept;
 * capturing synchronises nothing); later steps only launch it on `stream`.
 * Calls on one session are serialised by a host lock.  Steps share the
 * buffers, so the caller orders them on the device (one stream, or events).
 */
typedef struct gdn_session gdn_session;

typedef struct gdn_session_buffers_t {
    void *xq, *xk, *xv;       /* raw projections of the next step (caller writes) */
    float *a, *b;             /* gate logits of the next step (caller writes) */
    void *z;                  /* output-gate input of the next step (caller writes) */
    void *y;                  /* gated output of the last step (caller reads) */
    void *q, *k, *v, *o;      /* scratch */
    float *g, *beta;          /* scratch */
    float *state;             /* recurrent state, carried */
    void *conv_state;         /* convolution state, carried */
    const float *conv_w;      /* convolution taps */
    const float *norm_w;      /* RMS-norm weights, or NULL */
    void *workspace;          /* prefill workspace */
    size_t workspace_bytes;
} gdn_session_buffers_t;

size_t gdn_session_workspace_size(int num_streams, int H, int d, int seg_tokens, int dtype);
int gdn_session_create(int num_streams, int H, int d, int seg_tokens, int dtype, int activation, int gate,
                       float eps, const gdn_session_buffers_t *buffers, gdn_session **out);
/* a step of `tokens` in [1, seg_tokens] per stream, as a graph replay */
int gdn_session_prefill(gdn_session *s, int tokens, void *stream);
/* one token per stream, as a graph replay */
int gdn_session_decode(gdn_session *s, void *stream);
/* the same step launched kernel by kernel, without a graph (tokens = 0: decode) */
int gdn_session_step_eager(gdn_session *s, int tokens, void *stream);
/* number of instantiated graphs */
int gdn_session_graph_count(const gdn_session *s);
void gdn_session_destroy(gdn_session *s);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
