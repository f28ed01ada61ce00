/*
 * gdn2.h -- C ABI of the Gated DeltaNet-2 operator library (libgdn2.so).
 *
 * The operator is the gated delta rule with decoupled erase and write gates
 * ("Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention").  Per
 * (batch, head) it keeps a dk x dv state S and, for each token t,
 *
 *     Sbar = Diag(alpha_t) S_{t-1}          alpha_t = exp(log_alpha_t), per key channel
 *     e_t  = b_t (*) k_t                    erase gate b_t on the key axis
 *     z_t  = w_t (*) v_t                    write gate w_t on the value axis
 *     r_t  = Sbar^T e_t
 *     S_t  = Sbar + k_t (z_t - r_t)^T
 *     o_t  = S_t^T q_t                      the query reads the updated state
 *
 * as stated on the iplexlaw.co.kr page, section "Decisiones independientes en
 * dos ejes", and in product form S_t = (I - k_t (b_t (*) k_t)^T) D_t S_{t-1}
 * + k_t (w_t (*) v_t)^T in the zubnet.ai news item and the gist.science
 * summary (section 1, "Gated Delta Rule-2").  No scale is applied to q.
 *
 * Conventions shared by every entry point:
 *   - All tensor arguments are DEVICE pointers owned by the caller.  The
 *     library keeps no per-call state and never synchronises the stream; work
 *     is queued on `stream` (NULL = the legacy default stream) and the call
 *     returns once it is queued.  The bf16 path of gdn2_fwd_chunked needs a
 *     workspace, which it takes from a stream-ordered pool owned by the
 *     library (allocated and released on `stream`; the pool keeps freed
 *     blocks for reuse).  Nothing else allocates.
 *   - Layouts are dense row-major: q, k, b, log_alpha are [B][T][H][dk];
 *     v, w, o are [B][T][H][dv]; states are [B][H][dk][dv].  (The decode entry
 *     point drops the T axis.)
 *   - `dtype` is the element type of q, k, v, b, w and o.  log_alpha and
 *     every state are always fp32.  bf16 outputs are rounded to nearest even.
 *   - Every pointer must be 16-byte aligned.
 *   - Supported head sizes: dk and dv each 64 or 128.
 *   - The returned status covers argument checks and launch errors only.
 *     A condition found while the kernels run (a bounded wait that gave up) is
 *     recorded in a device-side error word and reported by
 *     gdn2_check_device_error().
 *   - Gates are used as given: values outside [0, 1] (the pages' ablation
 *     widens the erase range to [0, 2]) are not clamped.
 */
#ifndef GDN2_H
#define GDN2_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn2_status {
    GDN2_OK = 0,
    GDN2_ERR_NULL = 1,           /* a required pointer is NULL                        */
    GDN2_ERR_SHAPE = 2,          /* a size is out of range (negative, zero, too big)  */
    GDN2_ERR_DTYPE = 3,          /* unknown gdn2_dtype code                           */
    GDN2_ERR_ALIGN = 4,          /* a pointer is not 16-byte aligned                  */
    GDN2_ERR_UNSUPPORTED = 5,    /* valid request outside the implemented set         */
    GDN2_ERR_CUDA = 6,           /* a CUDA runtime call or launch failed              */
    GDN2_ERR_DEVICE_TIMEOUT = 7, /* a device-side bounded wait gave up                */
    GDN2_ERR_RANGE = 8,          /* reserved: no longer reported (every decay is computed) */
    GDN2_ERR_SCRATCH_LIMIT = 9   /* needs more than gdn2_fwd_chunked_noalloc's fixed buffer */
} gdn2_status;

typedef enum gdn2_dtype {
    GDN2_F32 = 0,
    GDN2_BF16 = 1
} gdn2_dtype;

/*
 * Gate layouts: which of b, w and log_alpha hold one value per (token, head)
 * instead of one per channel.  Bits of the `layout` argument of
 * gdn2_fwd_chunked_gates and gdn2_decode_tokens; 0 is the per-channel layout of
 * every other entry point.
 *
 * The pages derive the special cases of the operator from these shapes
 * (iplexlaw.co.kr, section "Decisiones independientes en dos ejes"; gist.science,
 * section 1): b = w = beta with beta a scalar per token gives Kimi Delta
 * Attention (pass the same pointer for b and w with GDN2_ERASE_SCALAR |
 * GDN2_WRITE_SCALAR); a scalar decay as well gives Gated DeltaNet (add
 * GDN2_DECAY_SCALAR).  A channel-averaged erase or write gate alone is
 * GDN2_ERASE_SCALAR or GDN2_WRITE_SCALAR.  A scalar tensor is [B][T][H]
 * ([B][H] for gdn2_decode_step's T-less layout), same dtype as the per-channel
 * one; it reads fewer bytes, which is what the bandwidth-bound kernels spend
 * their time on.
 */
typedef enum gdn2_gate_layout {
    GDN2_GATES_PER_CHANNEL = 0,  /* b [..][dk], w [..][dv], log_alpha [..][dk]     */
    GDN2_ERASE_SCALAR = 1,       /* b is [B][T][H]: one erase gate per token, head  */
    GDN2_WRITE_SCALAR = 2,       /* w is [B][T][H]: one write gate per token, head  */
    GDN2_DECAY_SCALAR = 4        /* log_alpha is [B][T][H]: one decay per token, head */
} gdn2_gate_layout;

/* Same type as cudaStream_t; declared here so this header needs no CUDA header. */
typedef struct CUstream_st *gdn2_stream_t;

/*
 * gdn2_fwd_chunked -- prefill / training forward over a whole sequence.
 *
 * Computes o_t for t = 0..T-1 and the final state S_T of the recurrence above,
 * chunkwise with chunks of 64 tokens: the per-channel decay is cumulated in
 * fp32 inside each chunk and folded into asymmetric decayed erase/key factors,
 * the strictly lower triangular 64 x 64 system is solved per chunk, and the
 * state is passed from chunk to chunk (iplexlaw.co.kr, section "Procesamiento
 * del token y entrenamiento paralelo"; gist.science, section 3 "Efficient
 * chunkwise parallel training").  The result equals the token recurrence up
 * to rounding.
 *
 *   q, k, b     [B][T][H][dk]  dtype   query, key, erase gate
 *   v, w        [B][T][H][dv]  dtype   value, write gate
 *   log_alpha   [B][T][H][dk]  fp32    log of the per-key-channel decay (<= 0)
 *   S0          [B][H][dk][dv] fp32    initial state; NULL means zero
 *   o           [B][T][H][dv]  dtype   output, written (never read)
 *   S_T         [B][H][dk][dv] fp32    final state; NULL means not written.
 *                                      May alias S0 (in-place advance).
 *   B, H >= 1; T >= 0 (T = 0 only copies S0, or zeros, into S_T).
 *
 * Decay: any log_alpha <= 0 is accepted, -inf included (alpha = 0: the
 * channel forgets everything before that token).  A chunk whose cumulative
 * decay is mild splits it into growing and shrinking factors around the chunk
 * midpoint; a chunk where that split would leave the fp32 range (strong
 * decay, e.g. log_alpha below about -2.5 held for 32 tokens) is computed in a
 * form whose factors are all decays, at a higher cost for that chunk.
 *
 * Execution (bf16, dk = 128): when the sequences' state chains take at most a
 * quarter of the SMs (see gdn2_fwd_chunked_launches) the call is one
 * cooperative kernel with one CTA on every SM, whose CTAs hand work to one
 * another (each such wait gives up after one second and reports
 * GDN2_ERR_DEVICE_TIMEOUT); it starts once every SM is free, so kernels of
 * other streams delay it or wait for it.  If the device cannot hold that grid
 * the call falls back to the windowed schedule.  There, when the chains take
 * more than half of the SMs, each window of chunks is two kernels on `stream`:
 * the prep, then the chains, which also compute the outputs.  Otherwise it is
 * three kernels per window, with the output kernels on a library-owned side
 * stream that forks from and joins back into `stream`.
 */
gdn2_status gdn2_fwd_chunked(const void *q, const void *k, const void *v,
                             const void *b, const void *w, const float *log_alpha,
                             const float *S0, void *o, float *S_T,
                             int B, int T, int H, int dk, int dv,
                             gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_fwd_chunked_noalloc -- gdn2_fwd_chunked without any device allocation.
 *
 * The pages have no counterpart to this entry point; it serves callers that
 * cannot let a library allocate device memory: a runtime that hands out all
 * device memory itself, a hot loop that must never enter the driver's
 * allocator (an allocation can block, or fail on a fragmented heap), or a
 * process that must know its whole device footprint before it starts.
 *
 * Same arguments, layouts, dtypes and results as gdn2_fwd_chunked.  Instead of
 * drawing its workspace from a memory pool, it uses one fixed 32 MiB buffer in
 * the library's device image (held on every GPU that loads the library, until
 * the process exits) and processes the sequence in as many windows as needed
 * to fit it.  A problem whose single chunk of records does not fit (about
 * 185 KiB per (batch, head) pair for dv = 128, so B*H up to 177) returns
 * GDN2_ERR_SCRATCH_LIMIT and launches nothing.
 *
 * The first call on a device looks the buffer's device address up
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls on one device share that device's
 * buffer: calls whose work overlaps on the GPU (for instance on two streams of
 * the same device) race and corrupt each other's results, so serialize them.
 * Each device has its own copy of the buffer; calls on different devices do
 * not share it.
 * Every byte of the buffer that a call reads, that call writes first, so its
 * leftover contents from earlier calls do not matter.
 */
gdn2_status gdn2_fwd_chunked_noalloc(const void *q, const void *k, const void *v,
                                     const void *b, const void *w, const float *log_alpha,
                                     const float *S0, void *o, float *S_T,
                                     int B, int T, int H, int dk, int dv,
                                     gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_decode_step -- one token of the recurrence with the state resident in
 * device memory (recurrent decoding with a fixed-size state instead of a
 * growing cache: gist.science, "Problem Statement"; iplexlaw.co.kr, "De una
 * caché creciente a un estado fijo").
 *
 *   q, k, b     [B][H][dk]      dtype
 *   v, w        [B][H][dv]      dtype
 *   log_alpha   [B][H][dk]      fp32
 *   S           [B][H][dk][dv]  fp32   read and updated in place
 *   o           [B][H][dv]      dtype  written
 *   B, H >= 1.
 *
 * Each state is streamed through the GPU once: read once, written once.
 */
gdn2_status gdn2_decode_step(const void *q, const void *k, const void *v,
                             const void *b, const void *w, const float *log_alpha,
                             float *S, void *o, int B, int H, int dk, int dv,
                             gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_decode_tokens -- T consecutive tokens of the recurrence on a state
 * resident in device memory (multi-token decode, or a short prefill into a
 * cached state: the recurrent form with a fixed-size state of gist.science,
 * "Problem Statement").  Equivalent to T calls of gdn2_decode_step, but each
 * state is read and written once per call instead of once per token; meant for
 * T up to a few dozen (longer sequences: gdn2_fwd_chunked).
 *
 *   q, k        [B][T][H][dk]  dtype
 *   v           [B][T][H][dv]  dtype
 *   b           [B][T][H][dk], or [B][T][H] with GDN2_ERASE_SCALAR   dtype
 *   w           [B][T][H][dv], or [B][T][H] with GDN2_WRITE_SCALAR   dtype
 *   log_alpha   [B][T][H][dk], or [B][T][H] with GDN2_DECAY_SCALAR   fp32
 *   S           [B][H][dk][dv] fp32   read and updated in place
 *   o           [B][T][H][dv]  dtype  written
 *   B, H, T >= 1; layout: a combination of gdn2_gate_layout bits.
 */
gdn2_status gdn2_decode_tokens(const void *q, const void *k, const void *v,
                               const void *b, const void *w, const float *log_alpha,
                               float *S, void *o, int B, int T, int H, int dk, int dv,
                               gdn2_dtype dtype, unsigned int layout, gdn2_stream_t stream);

/*
 * gdn2_fwd_chunked_gates -- gdn2_fwd_chunked with a gate layout: b, w and/or
 * log_alpha may be one value per (token, head) ([B][T][H]) as `layout` says.
 * Everything else (arguments, results, execution) is as for gdn2_fwd_chunked,
 * which is this function with layout 0.
 */
gdn2_status gdn2_fwd_chunked_gates(const void *q, const void *k, const void *v,
                                   const void *b, const void *w, const float *log_alpha,
                                   const float *S0, void *o, float *S_T,
                                   int B, int T, int H, int dk, int dv,
                                   gdn2_dtype dtype, unsigned int layout, gdn2_stream_t stream);

/*
 * gdn2_layer_fwd -- the chunked forward with the layer's processing around the
 * operator fused into its kernels ("Gated DeltaNet-2", iplexlaw.co.kr, section
 * "Procesamiento del token y entrenamiento paralelo": queries and keys are
 * L2-normalised, the gates come through sigmoids, and the recurrent output
 * receives RMS normalisation and an independent output gate before the output
 * projection).  The projections, the short convolution and the SiLU stay with
 * the caller.  Per (batch, token, head):
 *
 *     q_hat = q / sqrt(|q|^2 + 1e-6),  k_hat = k / sqrt(|k|^2 + 1e-6)
 *     b = sigmoid(b_logit),  w = sigmoid(w_logit),  log_alpha = log sigmoid(decay_logit)
 *     o, S_T = the operator of gdn2_fwd_chunked on (q_hat, k_hat, v, b, w, log_alpha, S0)
 *     y = o / sqrt(mean_j o_j^2 + eps) * norm_weight * sigmoid(g_logit)
 *
 * The pages name neither the decay's activation nor the output gate's, nor the
 * epsilons: this library reads both activations as the sigmoid the pages give
 * for the erase and write gates.  o never reaches device memory: y is formed
 * from the fp32 accumulators (bf16 inputs, dk = 128) or by a row kernel after
 * the operator (other inputs).
 *
 *   q, k                 [B][T][H][dk]  dtype   before the L2 norm
 *   v                    [B][T][H][dv]  dtype
 *   b_logit              [B][T][H][dk]  dtype
 *   w_logit, g_logit     [B][T][H][dv]  dtype
 *   decay_logit          [B][T][H][dk]  fp32
 *   norm_weight          [dv]           fp32   RMS-norm weight
 *   eps                  >= 0                  RMS-norm epsilon
 *   S0, S_T, B, T, H, dk, dv, dtype, stream    as for gdn2_fwd_chunked
 *   y                    [B][T][H][dv]  dtype   written
 */
gdn2_status gdn2_layer_fwd(const void *q, const void *k, const void *v,
                           const void *b_logit, const void *w_logit, const float *decay_logit,
                           const void *g_logit, const float *norm_weight, float eps,
                           const float *S0, void *y, float *S_T,
                           int B, int T, int H, int dk, int dv,
                           gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_bwd_chunked -- the backward of gdn2_fwd_chunked: gradients of
 * L = sum(o * dO) + sum(S_T * dS_T) with respect to every input, chunkwise
 * over 64-token chunks in reverse ("Gated DeltaNet-2", iplexlaw.co.kr, section
 * "Procesamiento del token y entrenamiento paralelo": the WY form's backward
 * must use the modulated keys and values, the per-channel gates staying inside
 * the gradient aggregation).  b and w get gradients of their own, per channel.
 * The forward is recomputed first (its chunk-entry states are the backward's
 * checkpoints, held in a workspace from the library's pool), then the gradient
 * of every chunk's exit state by a reverse pass over the chunks, then the
 * gradients of each chunk, all chunks at once.  Any log_alpha <= 0 is handled:
 * pairwise decays that a split around the chunk midpoint cannot hold are
 * running products of alpha.
 *   bf16 inputs with dk = 128: tensor cores (bf16 operands, fp32 accumulation
 *     and state), within the bf16 tolerance of the forward.  A chunk whose
 *     T = (I + A)^{-1} has an entry off the identity by more than 0.5 (nearly
 *     collinear keys with erase gates near 2) is computed a second time by the
 *     same CTA, with T and X = Z - Ebar S (the chunk's written values less what
 *     its erases read from the entry state) as bf16 pairs (hi + lo), over its
 *     plain gradients; three launches a call;
 *   fp32 inputs, and dk = 64: fp32 on the CUDA cores.
 *
 *   q, k, v, b, w, log_alpha, S0, B, T, H, dk, dv, dtype   as for gdn2_fwd_chunked
 *   dO          [B][T][H][dv]  dtype   incoming gradient of o
 *   dS_T        [B][H][dk][dv] fp32    incoming gradient of S_T; NULL means zero
 *   dq, dk, db, dlog_alpha  [B][T][H][dk]  fp32   written
 *   dv, dw                  [B][T][H][dv]  fp32   written
 *   dS0         [B][H][dk][dv] fp32    written; NULL means not wanted
 *
 * The key-axis gradients are sums over the value columns; one CTA per chunk and
 * head forms each of them in a fixed order, without atomics, so repeated calls
 * give identical bits.
 */
gdn2_status gdn2_bwd_chunked(const void *q, const void *k, const void *v,
                             const void *b, const void *w, const float *log_alpha,
                             const float *S0, const void *dO, const float *dS_T,
                             float *dq, float *dk, float *dv, float *db, float *dw,
                             float *dlog_alpha, float *dS0,
                             int B, int T, int H, int dk_, int dv_,
                             gdn2_dtype dtype, gdn2_stream_t stream);

/*
 * gdn2_check_device_error -- wait for `stream`, then read and clear the
 * device error word of the current device.  Returns GDN2_OK,
 * GDN2_ERR_DEVICE_TIMEOUT or GDN2_ERR_CUDA.
 */
gdn2_status gdn2_check_device_error(gdn2_stream_t stream);

/*
 * gdn2_fwd_chunked_launches -- number of kernel launches one gdn2_fwd_chunked
 * call on the current device makes for this problem (-1 for arguments
 * gdn2_fwd_chunked would reject).  The bf16 path launches one persistent
 * kernel when the sequences' chains (batch * heads * dv / 64 CTAs) take at
 * most a quarter of the SMs, else
 * per window of chunks two kernels (chains on more than half of the SMs) or
 * three, the window size depending on the device's SM count, which is the only thing this
 * queries (without a device it plans for 148 SMs); the fp32 path launches one
 * kernel.  A zeroing memset of a few kilobytes of flags precedes the persistent
 * kernel and is not counted.
 */
int gdn2_fwd_chunked_launches(int B, int T, int H, int dk, int dv, gdn2_dtype dtype);

/*
 * gdn2_selftest_bounded_wait -- queue on `stream` a one-warp kernel that waits
 * for a device flag nothing sets, with the bounded wait the persistent forward
 * uses between its CTAs.  The wait gives up after one second and records
 * GDN2_ERR_DEVICE_TIMEOUT in the device error word, so the next
 * gdn2_check_device_error(stream) returns it, and the context stays usable.
 * Returns GDN2_OK once queued (GDN2_ERR_CUDA if queuing failed).
 */
gdn2_status gdn2_selftest_bounded_wait(gdn2_stream_t stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char *gdn2_status_string(gdn2_status status);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
