/*
 * bimamba.h -- C ABI of the B200 (sm_100a) bidirectional Mamba-2 mixer core.
 *
 * The operation (sources by page title and section):
 *  - "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone"
 *    (Japanese technical summary, section 2 "Proposed method"; Portuguese
 *    technical summary, section 2 "Metodologia"): each mixer is a
 *    bidirectional Mamba-2 mixer whose forward and reverse streams are
 *    combined by addition.
 *  - "DiffuMamba" blog post, network-architecture listing: d_state = 128,
 *    d_conv = 4, expand = 2.
 *  - Mamba-2 selective state space recurrence, per head h (A_h < 0 scalar):
 *        h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T     (P x N state)
 *        y_t = h_t C_t + D_h x_t
 *    preceded by a depthwise causal conv1d (K = 4 taps) + SiLU over the
 *    x, B and C channels.  The reverse stream is the same computation on the
 *    reversed sequence (mirrored conv taps, zero padding past the end, zero
 *    initial state), flipped back.  y = forward stream + reverse stream.
 *  - "Fixed state, long reach: constant-size caches in large-scale block
 *    diffusion" (abstract, section 1): a finished prefix is cached as the
 *    forward SSM state (O(1) in the context length) plus the conv history;
 *    the reverse scan covers only the active block.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller.  Nothing is
 *    allocated or freed inside the library.  Every call is asynchronous on
 *    `stream` (the handle is a cudaStream_t; NULL = legacy default stream).
 *  - Tensors are dense, row-major (last index fastest), and 16-byte aligned.
 *  - Activations (xbc, dt, y, conv tails) have the element type `dtype`
 *    (BIMAMBA_F32 or BIMAMBA_BF16).  A, D, conv weights/bias and SSM states
 *    are always fp32.  Internal accumulation is fp32.
 *  - xbc channel order per token is [x (H*P, head-major) | B (G*N) | C (G*N)],
 *    ch = H*P + 2*G*N.
 *  - Return value: BIMAMBA_OK, or an error code.  Argument errors are found
 *    on the host before anything is launched (nothing is written).  Errors a
 *    kernel detects (a bounded wait that gave up) are recorded in a per-device
 *    status word; read and clear it with bimamba_get_error after the stream
 *    has been synchronised.  No C++ exception crosses this boundary.
 *  - Supported shapes: ngroups = 1, d_conv = 4, headdim a multiple of 8 up
 *    to 128, d_state a power of two from 8 to 256, batch <= 65535.  Others
 *    return BIMAMBA_ERR_UNSUPPORTED.
 */
#ifndef BIMAMBA_H
#define BIMAMBA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *bimamba_stream_t; /* == cudaStream_t */

typedef enum {
    BIMAMBA_OK = 0,
    BIMAMBA_ERR_INVALID = 1,      /* null pointer, bad size, misaligned      */
    BIMAMBA_ERR_UNSUPPORTED = 2,  /* valid but not implemented shape/dtype   */
    BIMAMBA_ERR_CUDA = 3,         /* a CUDA runtime call failed              */
    BIMAMBA_ERR_TIMEOUT = 4,      /* a kernel's bounded wait gave up         */
    BIMAMBA_ERR_WORKSPACE = 5     /* workspace missing or too small          */
} bimamba_status;

typedef enum { BIMAMBA_F32 = 0, BIMAMBA_BF16 = 1 } bimamba_dtype;

/* How bimamba_ssd_fwd_rev_untied combines its two streams. */
typedef enum { BIMAMBA_FUSE_SUM = 0, BIMAMBA_FUSE_CONCAT = 1 } bimamba_fusion;

typedef struct {
    int batch;    /* independent sequences (decode: streams)                */
    int len;      /* tokens per sequence (decode: active block length)      */
    int heads;    /* H                                                      */
    int headdim;  /* P                                                      */
    int d_state;  /* N                                                      */
    int ngroups;  /* G, B/C groups shared by H/G heads each (must be 1)     */
    int d_conv;   /* K, conv taps (must be 4)                               */
    int dtype;    /* bimamba_dtype of xbc, dt, y and conv tails             */
} bimamba_dims;

/* Library version, (major << 16) | minor. */
int bimamba_version(void);

/* Number of kernels this library has launched in this process so far
 * (host-side counter, all devices and streams).  For accounting only. */
unsigned long long bimamba_launch_count(void);

/*
 * Timing hook for benchmarks.  When `start` and `stop` are non-NULL
 * cudaEvent_t handles, every later bimamba_ssd_fwd_rev / bimamba_block_decode
 * call on this host thread records `start` immediately before its main scan
 * kernel and `stop` immediately after it, on the call's stream, so that
 * cudaEventElapsedTime(start, stop) is that kernel's device time.  Pass NULL
 * for both to switch it off.  Returns BIMAMBA_ERR_INVALID if only one is NULL.
 */
int bimamba_set_timing_events(void *start, void *stop);

/* Human-readable name of a status code (static string, never NULL). */
const char *bimamba_strerror(int status);

/*
 * Reads and clears this device's kernel status word (the current device).
 * Synchronises `stream` first.  Returns BIMAMBA_OK when no kernel recorded
 * an error since the last call, BIMAMBA_ERR_TIMEOUT when a bounded wait gave
 * up, BIMAMBA_ERR_CUDA when the runtime reports an error.
 */
int bimamba_get_error(bimamba_stream_t stream);

/*
 * Depthwise conv1d with `d_conv` taps followed by SiLU (silu != 0) or the
 * identity (silu == 0).  Step "conv + SiLU" of the mixer: the blog post
 * "DiffuMamba", network-architecture listing, gives each Mamba mixer a
 * d_conv = 4 convolution; the reverse stream runs it on the reversed
 * sequence (same listing: the second module sees the flipped sequence, its
 * output flipped back), which is the mirrored form below.
 *   u    : (batch, len, ch)    input, dtype
 *   out  : (batch, len, ch)    output, dtype; must not overlap u
 *   w    : (ch, d_conv) fp32   tap j of channel c
 *   bias : (ch) fp32 or NULL
 *   tail : (batch, d_conv, ch) dtype or NULL -- the d_conv raw tokens that
 *          precede t = 0, oldest first (forward only; must be NULL when
 *          reverse != 0).  NULL means zeros.
 * Forward (reverse == 0): pre[t,c] = bias[c] + sum_j w[c,j] u[t-(K-1)+j, c]
 * Reverse (reverse != 0): pre[t,c] = bias[c] + sum_j w[c,j] u[t+(K-1)-j, c],
 *                         u past the end = 0   (= flip(conv(flip(u)))).
 * Requires ch % 8 == 0.  Sums are formed in fp32 in tap order j = 0..K-1.
 */
int bimamba_conv_silu(const void *u, void *out, const float *w, const float *bias,
                      const void *tail, int batch, int len, int ch, int d_conv,
                      int reverse, int silu, int dtype, bimamba_stream_t stream);

/*
 * Bytes of scratch workspace bimamba_ssd_fwd_rev / bimamba_block_decode need
 * for dims `d`.  The caller allocates it once (device memory, 256-byte
 * aligned), zero-fills it before first use, and may reuse it for any later
 * call whose workspace size is not larger.  A call that completes returns
 * the workspace's forward/reverse meeting counters to zero, so it needs no
 * clearing between calls (the rest holds per-call intermediates that every
 * call rewrites).  After a call whose kernels reported BIMAMBA_ERR_TIMEOUT
 * (bimamba_get_error), the counters may be left set: zero-fill the workspace
 * again before reusing it.  Calls that share one workspace must not run
 * concurrently.  Returns 0 for invalid dims.  This scratch is the library's
 * own; the pages describe no such buffer.
 */
size_t bimamba_workspace_bytes(const bimamba_dims *d);

/*
 * How a bimamba_ssd_fwd_rev / bimamba_block_decode call with dims `d` is
 * launched; host only, no device work.  The chunked scan ("Mamba-2" state
 * space duality, chunkwise form: intra-chunk contraction, chunk states,
 * state passing) parallelises over (sequence, head pair, direction); when
 * that gives fewer than two CTAs per 148 SMs each direction's walk is cut
 * into segments, and a state-only pass first reduces the walk before each
 * segment to end states that the segment chains from.
 *   out[0] : 1 chunked tensor-core path, 0 sequential fp32 path
 *   out[1] : segments per direction (1: no segmentation)
 *   out[2] : 128-token chunks per segment
 *   out[3] : state-only items per (sequence, head pair, direction)
 *            (0: no state-only pass)
 * out must point to 4 writable ints.  Returns BIMAMBA_ERR_INVALID for
 * invalid dims or a NULL out, else BIMAMBA_OK (the same shape checks as the
 * compute calls, so UNSUPPORTED dims are reported too).
 */
int bimamba_launch_plan(const bimamba_dims *d, int *out);

/*
 * Full bidirectional mixer core (steps: load, conv+SiLU both ways, decay,
 * intra-chunk contraction, chunk states, state passing, off-diagonal term,
 * fused forward+reverse sum).  Defined by "DiffuMamba: High-Throughput
 * Diffusion LMs with Mamba Backbone", Japanese technical summary section 2
 * "Proposed method" and Portuguese technical summary section 2
 * "Metodologia" (bidirectional Mamba-2 mixer, forward and reverse streams
 * added), with the Mamba-2 recurrence written at the top of this file and
 * the blog's network-architecture listing for d_state = 128, d_conv = 4.
 *   xbc         : (batch, len, ch) raw xBC, dtype.  If conv_w == NULL the
 *                 conv and SiLU are skipped and xbc is taken as activated.
 *   dt          : (batch, len, H) dtype, already positive (post-softplus)
 *   A, D        : (H) fp32
 *   conv_w      : (ch, 4) fp32 or NULL;  conv_b : (ch) fp32 or NULL
 *   init_state  : (batch, H, P, N) fp32 or NULL -- forward initial state
 *   final_state : (batch, H, P, N) fp32 or NULL -- forward state after the
 *                 last token (written); may alias init_state
 *   y           : (batch, len, H*P) dtype, written (not accumulated)
 *   workspace   : bimamba_workspace_bytes(d) bytes, see above
 */
int bimamba_ssd_fwd_rev(const bimamba_dims *d, const void *xbc, const void *dt,
                        const float *A, const float *D, const float *conv_w,
                        const float *conv_b, const float *init_state,
                        float *final_state, void *y, void *workspace,
                        size_t workspace_bytes, bimamba_stream_t stream);

/*
 * Bidirectional mixer core with UNTIED directions: the forward stream and
 * the reverse stream each have their own inputs and parameters.  The blog
 * post "DiffuMamba", network-architecture listing, builds the mixer from two
 * separate Mamba modules (one on the sequence, one on the reversed
 * sequence, output reversed back), concatenates their outputs and maps 2d
 * back to d with a Linear layer; the technical summaries add the two
 * streams.  Both fusions are offered; the Linear after a concatenation is a
 * plain GEMM outside this call.
 *   xbc_f, xbc_r : (batch, len, ch) raw xBC of the forward / reverse stream
 *   dt_f, dt_r   : (batch, len, H) dtype, already positive
 *   A_f, A_r, D_f, D_r : (H) fp32
 *   conv_w_f, conv_w_r : (ch, 4) fp32 or NULL (that stream's xbc is taken as
 *                        activated); conv_b_f, conv_b_r : (ch) fp32 or NULL
 *                        (a bias needs its taps)
 *   init_state, final_state : the forward stream's, as in bimamba_ssd_fwd_rev
 *   fusion : BIMAMBA_FUSE_SUM    -> y (batch, len, H*P) = forward + reverse
 *            BIMAMBA_FUSE_CONCAT -> y (batch, len, 2*H*P), per token
 *                                   [forward (H*P) | reverse (H*P)]
 *   workspace : bimamba_workspace_bytes(d) bytes, as above
 * With every *_f pointer equal to its *_r pointer and BIMAMBA_FUSE_SUM this
 * is bimamba_ssd_fwd_rev.  Returns BIMAMBA_ERR_INVALID for an unknown
 * fusion, a missing input, a bias without taps or a misaligned pointer.
 */
int bimamba_ssd_fwd_rev_untied(const bimamba_dims *d, const void *xbc_f,
                               const void *xbc_r, const void *dt_f,
                               const void *dt_r, const float *A_f,
                               const float *A_r, const float *D_f,
                               const float *D_r, const float *conv_w_f,
                               const float *conv_w_r, const float *conv_b_f,
                               const float *conv_b_r, const float *init_state,
                               float *final_state, void *y, int fusion,
                               void *workspace, size_t workspace_bytes,
                               bimamba_stream_t stream);

/*
 * Sequence shards (one sequence split across ranks, e.g. one GPU each).
 * The pages describe no sharding; this is the same mixer core as
 * bimamba_ssd_fwd_rev (same sources), split along the sequence using the
 * recurrence's linearity in the state.
 * The recurrence is linear in the state, so a shard's effect on the state
 * that crosses it is h -> 2^dec h + S, where S is the state the shard leaves
 * when entered with zero and dec the log2 of the product of its per-token
 * decay factors exp(dt A).  Each rank computes (S, dec) of its shard for both
 * directions, the ranks exchange them (an all-gather: 2 x H x P x N fp32 plus
 * 2 x H per sequence and rank), and each rank then computes its outputs
 * entering its shard with the states the other shards hand on.  This is the
 * exchange step of the scan on a sharded sequence dimension.  The tokens next
 * to a shard that its conv reads (3 before for the forward stream, 3 after
 * for the reverse stream) come from the neighbouring shards as halos.
 * Tensor-core path only (bf16, headdim 64, d_state 128, even H); other
 * shapes return BIMAMBA_ERR_UNSUPPORTED.
 *
 * bimamba_shard_states: this rank's (S, dec), no outputs.
 *   d      : the shard's dims (len = shard length)
 *   xbc, dt, A, conv_w, conv_b : as in bimamba_ssd_fwd_rev, for the shard
 *   tail   : (batch, 4, ch) dtype or NULL -- the 4 raw tokens before the shard
 *            (oldest first; NULL or zeros for the first shard)
 *   head   : (batch, 4, ch) dtype or NULL -- the 4 raw tokens after the shard
 *            (in order; NULL or zeros for the last shard)
 *   states : (2, batch, H, P, N) fp32, written: [0] the forward stream's state
 *            after the shard, [1] the reverse stream's state after walking the
 *            shard from its last token to its first, both from zero
 *   decays : (2, batch, H) fp32, written: dec per direction (equal up to the
 *            rounding of the two summation orders)
 *   workspace : bimamba_workspace_bytes(d) bytes
 */
int bimamba_shard_states(const bimamba_dims *d, const void *xbc, const void *dt,
                         const float *A, const float *conv_w, const float *conv_b,
                         const void *tail, const void *head, float *states,
                         float *decays, void *workspace, size_t workspace_bytes,
                         bimamba_stream_t stream);

/*
 * bimamba_ssd_fwd_rev_shard: this rank's outputs.  The forward stream enters
 * the shard with init_state carried through shards 0 .. rank-1; the reverse
 * stream enters with zero carried through shards nranks-1 .. rank+1.
 *   xbc, dt, A, D, conv_w, conv_b, tail, head : as above
 *   init_state : (batch, H, P, N) fp32 or NULL -- forward state before shard 0
 *   all_states : (nranks, 2, batch, H, P, N) fp32 -- every rank's `states`,
 *                in rank order (may be NULL when nranks == 1)
 *   all_decays : (nranks, 2, batch, H) fp32 -- every rank's `decays`
 *   rank, nranks : this shard's position, 0 <= rank < nranks
 *   final_state : (batch, H, P, N) fp32 or NULL -- the forward state after
 *                this shard (the sequence's final state on the last rank)
 *   y          : (batch, len, H*P) dtype -- the shard's outputs
 * Concatenating every rank's y gives bimamba_ssd_fwd_rev on the whole sequence.
 * A shard must hold at least one token (an empty shard returns
 * BIMAMBA_ERR_INVALID here; bimamba_shard_states reports it as zero states
 * and zero decay, which leave the crossing state unchanged).
 */
int bimamba_ssd_fwd_rev_shard(const bimamba_dims *d, const void *xbc,
                              const void *dt, const float *A, const float *D,
                              const float *conv_w, const float *conv_b,
                              const void *tail, const void *head,
                              const float *init_state, const float *all_states,
                              const float *all_decays, int rank, int nranks,
                              float *final_state, void *y, void *workspace,
                              size_t workspace_bytes, bimamba_stream_t stream);

/*
 * Cached block decode for block diffusion: d->batch independent streams,
 * each with an active block of d->len tokens.  The forward stream resumes
 * from `state` with the conv history `tail`; the reverse stream covers the
 * block only (zero padding past the block end, zero state).  y = sum.
 * Defined by "Fixed state, long reach: constant-size caches in large-scale
 * block diffusion", abstract and section 1 (the finished prefix cached as the
 * forward SSM state, O(1) in the context length; the reverse scan restricted
 * to the active block; block-causal training makes the cached decode equal
 * to a full recompute).
 * Result equals a full recompute over prefix + block (forward stream at the
 * block positions) plus the reverse stream over the block alone.
 *   xbc_block : (streams, len, ch) raw xBC of the active block, dtype
 *   dt_block  : (streams, len, H) dtype
 *   A, D, conv_w (required), conv_b (nullable): as above
 *   state     : (streams, H, P, N) fp32 forward state after the prefix
 *   tail      : (streams, 4, ch) dtype, last 4 raw prefix tokens, oldest
 *               first (zeros where the prefix is shorter)
 *   y         : (streams, len, H*P) dtype
 *   state_out : (streams, H, P, N) fp32 or NULL -- commit: forward state
 *               after the block; may alias `state`
 *   tail_out  : (streams, 4, ch) dtype or NULL -- commit: last 4 raw tokens
 *               of prefix + block; must not overlap `tail`
 *   workspace : bimamba_workspace_bytes(d) bytes
 */
int bimamba_block_decode(const bimamba_dims *d, const void *xbc_block,
                         const void *dt_block, const float *A, const float *D,
                         const float *conv_w, const float *conv_b,
                         const float *state, const void *tail, void *y,
                         float *state_out, void *tail_out, void *workspace,
                         size_t workspace_bytes, bimamba_stream_t stream);

/*
 * Cached block decode over a pool of cached streams, with a commit per row:
 * the batch form a serving loop drives.  Block diffusion keeps one cache
 * entry per stream -- the forward SSM state after its finished prefix and
 * its last 4 raw tokens ("Fixed state, long reach: constant-size caches in
 * large-scale block diffusion", abstract and section 1: an O(1) state per
 * stream, many streams decoded together, a block committed once finished) --
 * and each step decodes the active blocks of a batch of streams whose
 * prefixes may all have different lengths.
 *   d          : batch = rows decoded in this call, len = block length
 *                (1..64); bf16, headdim 64, d_state 128 (else
 *                BIMAMBA_ERR_UNSUPPORTED)
 *   xbc_block, dt_block, A, D, conv_w, conv_b, y : as in bimamba_block_decode,
 *                row s of the batch
 *   state_pool : (pool_size, H, P, N) fp32 -- the cached forward states
 *   tail_pool  : (pool_size, 4, ch) dtype -- the cached conv tails
 *   slots      : (batch) int32, device -- the pool entry of each row; entries
 *                of one call must be distinct.  A slot outside
 *                [0, pool_size) skips its row and makes bimamba_get_error
 *                report BIMAMBA_ERR_INVALID.
 *   commit     : (batch) int32, device, or NULL -- rows with commit[s] != 0
 *                (every row when NULL) write their state after the block and
 *                their new conv tail back into their pool entry, in place
 *   workspace  : bimamba_workspace_bytes(d) bytes
 * Row s's output equals bimamba_block_decode on state_pool[slots[s]] and
 * tail_pool[slots[s]].
 */
int bimamba_block_decode_pool(const bimamba_dims *d, const void *xbc_block,
                              const void *dt_block, const float *A, const float *D,
                              const float *conv_w, const float *conv_b,
                              float *state_pool, void *tail_pool, int pool_size,
                              const int *slots, const int *commit, void *y,
                              void *workspace, size_t workspace_bytes,
                              bimamba_stream_t stream);

/*
 * Backward pass of the bidirectional mixer core (training): the gradients of
 * L = sum(dy * y), y = bimamba_ssd_fwd_rev(xbc, dt, A, D, conv_w, conv_b,
 * init_state), with respect to every input.  "DiffuMamba: High-Throughput
 * Diffusion LMs with Mamba Backbone" trains this mixer with the
 * masked-diffusion objective (Portuguese technical summary, section 2
 * "Metodologia"); the gradients are those of the recurrence and conv written
 * at the top of this file, run back through both streams.
 *   xbc, dt, A, D, conv_w (required), conv_b, init_state : the forward call's
 *                inputs (init_state NULL = zero)
 *   dy         : (batch, len, H*P) dtype
 *   outputs, fp32, written (not accumulated):
 *   dxbc (batch, len, ch), ddt (batch, len, H), dA (H), dD (H),
 *   dconv_w (ch, 4), dconv_b (ch) or NULL, dinit (batch, H, P, N) or NULL
 *   workspace  : bimamba_backward_workspace_bytes(d) bytes (no clearing
 *                needed); it holds both streams' activations, their fp32
 *                gradients and the state entering every chunk
 * Shapes: headdim <= 64 and d_state <= 128, both multiples of 4 (else
 * BIMAMBA_ERR_UNSUPPORTED); fp32 or bf16 activations.  For bf16 with
 * headdim 64 and d_state 128 the chunked backward (128-token chunks) runs
 * every matrix product on the tensor cores (bf16 operands, fp32
 * accumulation); otherwise (64-token chunks) its small products run on the
 * CUDA cores in fp32.  The conv passes read 64-token x 64-channel tiles by
 * TMA and evaluate SiLU and its derivative in fp32, through the hardware
 * tanh for bf16 activations.  Errors: as bimamba_ssd_fwd_rev (a bounded wait
 * that gave up is reported by bimamba_get_error as BIMAMBA_ERR_TIMEOUT).
 */
size_t bimamba_backward_workspace_bytes(const bimamba_dims *d);

int bimamba_ssd_fwd_rev_backward(const bimamba_dims *d, const void *xbc, const void *dt,
                                 const float *A, const float *D, const float *conv_w,
                                 const float *conv_b, const float *init_state,
                                 const void *dy, float *dxbc, float *ddt, float *dA,
                                 float *dD, float *dconv_w, float *dconv_b, float *dinit,
                                 void *workspace, size_t workspace_bytes,
                                 bimamba_stream_t stream);

/*
 * The projections on either side of the mixer, on the tensor cores (bf16
 * operands, fp32 accumulation, bf16 results).  "DiffuMamba" blog post,
 * network-architecture listing: d_model = 2048 with expand = 2, so each
 * mixer maps d_model to its inner width H*P and back, and the bidirectional
 * block maps the concatenation of its two streams (2 d) back to d with a
 * Linear.  Weights are row-major (out_features, in_features), as a Linear
 * layer stores them.
 *
 * bimamba_in_proj: u (tokens, d_model) -> the mixer's inputs, written in the
 * layouts bimamba_ssd_fwd_rev reads:
 *   xbc (tokens, ch)  = u . W_in[0:ch]^T              ch = H*P + 2*N
 *   dt  (tokens, H)   = softplus(u . W_in[ch:ch+H]^T + dt_bias)
 *   w_in : (ch + H, d_model) bf16;  dt_bias : (H) fp32 or NULL (zero)
 * Requires d_model % 8 == 0.
 *
 * bimamba_out_proj: out (tokens, d_model) = y . W_out^T
 *   y     : (tokens, d_inner) bf16 -- the mixer's output; with untied
 *           directions and concatenated streams d_inner = 2*H*P and W_out is
 *           the block's fusion Linear (applied after each stream's own output
 *           map, which composes into one (d_model, 2*H*P) matrix)
 *   w_out : (d_model, d_inner) bf16
 * Requires d_inner % 8 == 0.
 * Both: pointers 16-byte aligned, outputs must not overlap inputs; a kernel
 * wait that gives up is reported by bimamba_get_error as BIMAMBA_ERR_TIMEOUT.
 */
int bimamba_in_proj(int tokens, int d_model, int heads, int headdim, int d_state,
                    const void *u, const void *w_in, const float *dt_bias, void *xbc,
                    void *dt, bimamba_stream_t stream);

int bimamba_out_proj(int tokens, int d_inner, int d_model, const void *y,
                     const void *w_out, void *out, bimamba_stream_t stream);

/*
 * Cached block decode without a caller workspace.  The paper has no
 * counterpart to this entry point; it exists for callers that cannot
 * allocate device memory: a serving process whose memory pool already holds
 * the whole device (an allocation by the library would fail or fight that
 * pool), or a decode loop whose rules forbid allocating once it serves.
 * Arguments, layouts and result are those of bimamba_block_decode, minus the
 * workspace.  The scratch comes from one fixed array of
 * bimamba_noalloc_scratch_bytes() bytes (16 MiB) inside this library, which
 * every GPU that loads the library holds until the process exits.
 *  - Returns BIMAMBA_ERR_WORKSPACE when the call needs more scratch than the
 *    array holds (bimamba_workspace_bytes(d) > bimamba_noalloc_scratch_bytes();
 *    for bf16, headdim 64, d_state 128 that is about 16 000 tokens, i.e.
 *    streams x block length, per call).  Nothing is launched then.
 *  - The first call on a device looks up the array's device address, so make
 *    that first call before any stream capture.  The address is kept for the
 *    life of the process: do not use the library across cudaDeviceReset.
 *  - Arguments are checked as bimamba_block_decode checks them, before
 *    anything is queued.  Each accepted call then clears the array's meeting
 *    counters (an asynchronous memset on `stream`, so a call that stopped on
 *    a timeout cannot leave them set for the next) and runs the same kernels
 *    as bimamba_block_decode.
 *  - All calls share the one array: calls that overlap on the GPU (on
 *    different streams, or from several host threads without ordering) race
 *    and corrupt each other's results.  Serialise them.
 *  - It allocates and frees nothing.
 */
size_t bimamba_noalloc_scratch_bytes(void);

int bimamba_block_decode_noalloc(const bimamba_dims *d, const void *xbc_block,
                                 const void *dt_block, const float *A, const float *D,
                                 const float *conv_w, const float *conv_b,
                                 const float *state, const void *tail, void *y,
                                 float *state_out, void *tail_out,
                                 bimamba_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BIMAMBA_H */
