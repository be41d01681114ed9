/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated delta-rule library (libgdn.so).
 *
 * The library computes the causal gated delta-rule recurrence
 *
 *     S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,            alpha_t = exp(g_t),
 *
 * with the state S in R^{dv x dk} stored row-major as [B,H,dv,dk] (the column
 * convention; the pages write the transposed row-vector form S_t = S_{t-1} +
 * k_t^T v_t, o_t = q_t S_t, which is the same map).  Sources, all on the page
 * "Linear Attention, Visualized": "Naive linear attention" (additive write),
 * "RetNet: scalar decay" and "Mamba-2: input-dependent scalar decay" (scalar
 * gate), "DeltaNet: correcting memory collisions" / "Recurrent form" (delta
 * write), "Gated DeltaNet (GDN)" (scalar gate + delta), "Gated Linear
 * Attention (GLA)" and "Kimi Delta Attention (KDA)" (per-channel gate along
 * the key dimension).  The three write rules are also listed in "Beyond
 * attention", section "Linear attention: a running sum".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is a DEVICE pointer (cudaMalloc'd or torch CUDA
 *    storage) on the current CUDA device, 16-byte aligned, contiguous in the
 *    layout stated.  The caller owns every buffer; the library allocates no
 *    device memory and keeps no state between calls except one device status
 *    word (see gdn_device_status).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it; a return value of GDN_OK means the
 *    launch was accepted, not that it finished.
 *  - q, k, v, o element type is given by desc->dtype / desc->out_dtype
 *    (GDN_F32 = float, GDN_BF16 = bfloat16).  g, beta and the state are float.
 *  - g holds the log-gate log(alpha) (normally <= 0):  [B,H,T] for
 *    GDN_GATE_SCALAR, [B,H,T,dk] for GDN_GATE_CHANNEL, and must be NULL for
 *    GDN_GATE_NONE.  beta [B,H,T] is read only for GDN_DELTA (else may be NULL).
 *  - NaN or Inf in the inputs propagate to the outputs; nothing traps.
 *  - Errors are negative return codes; nothing is launched when a call fails
 *    validation.  gdn_strerror() names them.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_VERSION 7

/* Return codes. */
#define GDN_OK 0
#define GDN_ERR_ARG (-1)         /* null pointer, bad enum, bad size or overlap */
#define GDN_ERR_ALIGN (-2)       /* a pointer is not 16-byte aligned */
#define GDN_ERR_UNSUPPORTED (-3) /* valid request this build does not implement */
#define GDN_ERR_CUDA (-4)        /* the CUDA runtime refused the launch */
#define GDN_ERR_TIMEOUT (-5)     /* device status: a bounded wait in a kernel ran out */
#define GDN_ERR_RANGE (-6)       /* device status: an fp16 tensor-core operand overflowed */

/* Largest token count of one gdn_decode_step call (longer runs: gdn_chunk_fwd). */
#define GDN_DECODE_MAX_T 16

/* Largest number of substeps per token of gdn_product_fwd. */
#define GDN_PRODUCT_MAX_NH 16

/* Write rule.  ADDITIVE: S += v k^T, no gate ("Naive linear attention").
 * DECAY: S = S Diag(alpha) + v k^T, gate required (RetNet / Mamba-2 / GLA).
 * DELTA: the gated delta rule above; any gate (DeltaNet / GDN / KDA). */
typedef enum { GDN_ADDITIVE = 0, GDN_DECAY = 1, GDN_DELTA = 2 } gdn_update_t;

/* Gate: none (alpha = 1), one scalar per token and head, or one value per key
 * channel per token and head. */
typedef enum { GDN_GATE_NONE = 0, GDN_GATE_SCALAR = 1, GDN_GATE_CHANNEL = 2 } gdn_gate_t;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype_t;

/* Kernel choice for gdn_chunk_fwd.  AUTO picks, for the additive update without
 * gate and without input prologue (bf16, dk = 128, dv in {64, 128}), the
 * linear-attention tensor-core kernel (state kept fp32 in tensor memory); else
 * the tensor-core kernel below when it supports the request (bf16 inputs,
 * dk = 128) and the fp32 SIMT kernel otherwise.  TC is the warp-specialised
 * tensor-core kernel for every mode (prep of the next chunk overlapping the
 * state update of the current one).  An explicit value
 * forces that kernel (GDN_ERR_UNSUPPORTED if it cannot serve the request); any
 * other value is GDN_ERR_ARG. */
typedef enum { GDN_ALGO_AUTO = 0, GDN_ALGO_SIMT = 1, GDN_ALGO_TC = 2 } gdn_algo_t;

/* Input prologue (bits of gdn_desc_t.prologue): maps the kernels apply to their
 * inputs as they load them, so that raw projections can be passed directly.
 *   QK_ELU1        q, k <- elu(x) + 1 elementwise, the feature map of linear
 *                  attention ("Linear attention: a running sum" code; "Beyond
 *                  attention" linear-attention forward)
 *   QK_L2          each q and k row <- x / |x|_2 (after QK_ELU1 when both are
 *                  set; a zero row stays zero), the normalised keys and queries
 *                  of the DeltaNet forward
 *   BETA_SIGMOID   beta <- 1 / (1 + e^{-beta}) (write strength from a logit)
 *   G_NEG_SOFTPLUS g <- -softplus(g) = -log(1 + e^{g}) (log-gate from a logit,
 *                  the softplus step of "Optional: Constructing the decay gate")
 * The oracle applies the same maps in float64 before the recurrence. */
#define GDN_PRO_QK_ELU1 1
#define GDN_PRO_QK_L2 2
#define GDN_PRO_BETA_SIGMOID 4
#define GDN_PRO_G_NEG_SOFTPLUS 8

typedef struct {
    int B, H;      /* batch and heads; B*H >= 0 */
    int T;         /* tokens per sequence (gdn_chunk_fwd: T >= 0; decode: 0..GDN_DECODE_MAX_T) */
    int dk, dv;    /* key and value head dims, each 64 or 128 */
    int update;    /* gdn_update_t */
    int gate;      /* gdn_gate_t */
    int dtype;     /* gdn_dtype_t of q, k, v */
    int out_dtype; /* gdn_dtype_t of o */
    int chunk;     /* chunk length C of the chunkwise form; 0 or 64 (others rejected) */
    int algo;      /* gdn_algo_t (gdn_chunk_fwd only; ignored by decode) */
    int prologue;  /* GDN_PRO_* bits, 0 = inputs used as given */
} gdn_desc_t;

/*
 * gdn_chunk_fwd -- prefill: the recurrence over T tokens for every (b,h), in
 * chunkwise-parallel form with chunk length C = 64.
 *
 * Defined by "Linear Attention, Visualized", section "Chunkwise algorithm"
 * (history read plus masked local block, then the state update), with the
 * decayed operands of "Mamba-2 ... Chunkwise form" / the GLA section and the
 * correction rows Z of "Optional: Use UT to share the triangular transform"
 * and "Correct the incoming state" (the GDN and KDA tables).  Every chunk
 * length gives the token recurrence exactly ("Cost").
 *
 *   q, k  [B,H,T,dk]   dtype          v  [B,H,T,dv]  dtype
 *   g     see above    float          beta [B,H,T]   float (DELTA)
 *   S0    [B,H,dv,dk]  float, or NULL for a zero initial state
 *   o     [B,H,T,dv]   out_dtype      (written)
 *   S_T   [B,H,dv,dk]  float, or NULL to skip; may alias S0 (in-place carry)
 *
 * o must not overlap any input.  T == 0 is valid (o is empty, S_T <- S0).
 * Returns GDN_OK or a negative code.
 */
int gdn_chunk_fwd(const gdn_desc_t *desc, const void *q, const void *k, const void *v,
                  const float *g, const float *beta, const float *S0, void *o, float *S_T,
                  void *stream);

/*
 * gdn_chunk_fwd_host -- gdn_chunk_fwd on HOST buffers: the same arguments and
 * results, with q, k, v, g, beta, S0, o and S_T in host memory (page-locked
 * for the copies to overlap; pageable memory works, serialised).  The heads are
 * cut into n_slices contiguous slices; slice i is copied host -> device on an
 * internal stream, computed by gdn_chunk_fwd on the caller's stream, and copied
 * device -> host on a second internal stream, alternating between two slots of
 * the device workspace, so the copies of one slice overlap the kernel of
 * another and the two copy directions overlap each other.  The call returns
 * once all work is enqueued; the caller's stream waits for the last copy, so
 * o and S_T are complete (and the host inputs free) when that stream has
 * synchronised.  (The pages' prefill has no transfer step; this is the
 * host-resident use of the same prefill.)
 *
 *   workspace  device buffer of gdn_host_workspace_bytes(desc, n_slices)
 *              bytes, 256-byte aligned, owned by the caller, on the calling
 *              thread's current device (where the two internal streams are
 *              created; `stream` must belong to that device too)
 *
 * n_slices >= 1 (more slices than heads act as one head per slice).  On a
 * non-zero return some copies may already be in flight: synchronise the device
 * before reusing the buffers.
 */
size_t gdn_host_workspace_bytes(const gdn_desc_t *desc, int n_slices);
int gdn_chunk_fwd_host(const gdn_desc_t *desc, int n_slices, const void *q, const void *k, const void *v,
                       const float *g, const float *beta, const float *S0, void *o, float *S_T, void *workspace,
                       size_t workspace_bytes, void *stream);

/*
 * gdn_product_fwd -- prefill of Gated DeltaProduct: every real token applies
 * nh delta-rule transitions in order, each with its own key, value and write
 * strength, after one decay by the token's gate, and is read after the last
 * ("Linear Attention, Visualized", "Gated Delta Product (GDP)").  Computed, as
 * "GDP as GDN over a virtual sequence" describes, by the chunkwise GDN path over
 * T * nh virtual steps: substep j of token t is step t * nh + j, the gate sits on
 * the first substep and the query on the last, and every nh-th output is kept.
 *
 *   q     [B,H,T,dk]      dtype       k  [B,H,T,nh,dk]  dtype
 *   v     [B,H,T,nh,dv]   dtype       beta [B,H,T,nh]   float
 *   g     [B,H,T] (scalar) or [B,H,T,dk] (channel) or NULL        float
 *   S0, S_T, o            as in gdn_chunk_fwd (o is [B,H,T,dv])
 *
 * desc->update must be GDN_DELTA and desc->T counts real tokens.  nh == 1 is
 * gdn_chunk_fwd.  For nh > 1, GDN_ALGO_AUTO takes the pipelined tensor-core
 * kernel when it serves the shape (bf16, dk = 128, dv in {64, 128}, any gate; a
 * chunk holds floor(64 / nh) whole tokens and identity steps fill its remaining
 * rows) and the fp32 SIMT kernel otherwise; GDN_ALGO_TC demands the former,
 * GDN_ALGO_SIMT the latter.
 * The caller owns every buffer; nothing is allocated.
 */
int gdn_product_fwd(const gdn_desc_t *desc, int nh, const void *q, const void *k, const void *v,
                    const float *g, const float *beta, const float *S0, void *o, float *S_T,
                    void *stream);

/*
 * gdn_chunk_fwd_segmented -- the prefill of gdn_chunk_fwd with each sequence
 * cut into nseg segments of T / nseg tokens that run in parallel (more CTAs
 * when B*H alone would leave the GPU idle).  A segment acts on its incoming
 * state as an affine map, S_out = S_in Lambda + H ("One chunk as an affine
 * recurrence", "Update the state"), so the call runs: every segment from a zero
 * state (H), every segment's transition (zero values from the identity state;
 * skipped for the additive write, whose transition is the identity), an
 * in-order composition S_{i+1} = S_i Lambda_i + H_i, and every segment again
 * from its true incoming state S_i for the outputs.  Same arguments and results
 * as gdn_chunk_fwd, about three times its arithmetic; T must be a multiple of
 * nseg (nseg == 1 is gdn_chunk_fwd).
 *
 *   workspace  device buffer of at least gdn_segmented_workspace_bytes(desc,
 *              nseg) bytes, 16-byte aligned, owned by the caller; it must not
 *              overlap any input (q, k, v, g, beta, S0) or output (o, S_T):
 *              the first pass writes it and later passes re-read the inputs,
 *              so an overlap returns GDN_ERR_ARG.  Its contents on return are
 *              unspecified.  gdn_segmented_workspace_bytes returns 0 for a
 *              request it cannot size (null desc, nseg < 1, more than 2^30
 *              segment-heads).
 */
size_t gdn_segmented_workspace_bytes(const gdn_desc_t *desc, int nseg);
int gdn_chunk_fwd_segmented(const gdn_desc_t *desc, int nseg, const void *q, const void *k, const void *v,
                            const float *g, const float *beta, const float *S0, void *o, float *S_T,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_segmented_noalloc -- gdn_chunk_fwd_segmented with the
 * workspace taken from a fixed device array of the library
 * (GDN_NOALLOC_SCRATCH_BYTES per device; with lazy module loading, the CUDA
 * default, it is mapped on first use) instead of the
 * caller, so the call allocates nothing and takes no workspace argument.  The
 * pages have no counterpart: it is a calling convenience for callers that
 * cannot allocate on the call path.  A malformed request returns the code
 * gdn_chunk_fwd_segmented returns for it (checked first); a well-formed one
 * whose workspace (gdn_segmented_workspace_bytes) exceeds the array returns
 * GDN_ERR_UNSUPPORTED; other arguments and results as gdn_chunk_fwd_segmented.
 * Concurrent calls on one device share the array and must be ordered (one
 * stream, or events).
 */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
size_t gdn_noalloc_scratch_bytes(void);
int gdn_chunk_fwd_segmented_noalloc(const gdn_desc_t *desc, int nseg, const void *q, const void *k, const void *v,
                                    const float *g, const float *beta, const float *S0, void *o, float *S_T,
                                    void *stream);

/*
 * gdn_segment_maps -- the affine map of a run of tokens taken as one segment
 * ("One chunk as an affine recurrence", "Update the state"): for every (b,h),
 * the T tokens send an incoming state S_in to S_in Lambda + H, where
 *     H       [B,H,dv,dk] float  the state after the T tokens from S = 0,
 *     Lambda  [B,H,dk,dk] float  the product of the tokens' transitions
 *                                (Diag(alpha_t)(I - beta_t k_t k_t^T) for DELTA,
 *                                Diag(alpha_t) for DECAY, I for ADDITIVE),
 * both written (no outputs o).  Used when the segments of one sequence live on
 * different devices: each device computes its segment's maps, the maps are
 * gathered, gdn_compose_segments gives every segment its incoming state, and
 * gdn_chunk_fwd from that state gives the outputs.  Inputs and their rules as in
 * gdn_chunk_fwd (q is read though no output is formed); H and Lambda must be
 * 16-byte aligned and overlap neither each other nor any input.  T == 0 gives
 * H = 0, Lambda = I.
 */
int gdn_segment_maps(const gdn_desc_t *desc, const void *q, const void *k, const void *v, const float *g,
                     const float *beta, float *H, float *Lambda, void *stream);

/*
 * gdn_compose_segments -- thread a state through nseg consecutive segments of
 * BH sequences given their maps:  S_0 = S0 (zero when NULL),
 * S_{i+1} = S_i Lambda_i + H_i; fp32 throughout.  Segment-major layouts:
 *     H      [nseg][BH][dv][dk] float   (from gdn_segment_maps, segment by segment)
 *     Lambda [nseg][BH][dk][dk] float   (NULL: every transition is the identity)
 *     S_in   [nseg][BH][dv][dk] float   written: S_i, the state entering segment i (or NULL)
 *     S_T    [BH][dv][dk]       float   written: S_nseg, the final state (or NULL; may be S0)
 * dk, dv in {64, 128}; pointers 16-byte aligned; outputs overlap no input
 * except S_T == S0 exactly.
 */
int gdn_compose_segments(int BH, int nseg, int dk, int dv, const float *S0, const float *H, const float *Lambda,
                         float *S_in, float *S_T, void *stream);

/*
 * gdn_decode_step -- decode: T recurrent steps (1 <= T <= GDN_DECODE_MAX_T,
 * usually 1) for every (b,h), with the state updated in place ("Optional:
 * Linear attention as an RNN": fixed state, constant work per token; the
 * per-token recurrences of the RetNet, Mamba-2, DeltaNet, GDN, GLA and KDA
 * sections).  A bandwidth-bound rank-1 update per token: per state row i,
 * with a = alpha_t,
 *     p_i = sum_j S_ij a_j k_j,  r_i = sum_j S_ij a_j q_j,
 *     u_i = beta (v_i - p_i)  (DELTA)  or  v_i  (ADDITIVE / DECAY),
 *     S_ij <- S_ij a_j + u_i k_j,   o_i = r_i + u_i (k . q).
 * The T tokens are applied in order with the state held on chip, so the state
 * is read and written once per call, not once per token.
 *
 *   q, k  [B,H,T,dk]   dtype          v  [B,H,T,dv]  dtype
 *   g     [B,H,T] (scalar) or [B,H,T,dk] (channel) or NULL     float
 *   beta  [B,H,T]      float (DELTA)
 *   S     [B,H,dv,dk]  float, read and overwritten in place
 *   o     [B,H,T,dv]   out_dtype      (written)
 *
 * T == 0 is a no-op; T > GDN_DECODE_MAX_T returns GDN_ERR_UNSUPPORTED.
 * desc->chunk and desc->algo are ignored.
 */
int gdn_decode_step(const gdn_desc_t *desc, const void *q, const void *k, const void *v,
                    const float *g, const float *beta, float *S, void *o, void *stream);

/* Static string naming a return code (never NULL). */
const char *gdn_strerror(int code);

/*
 * gdn_chunk_fwd_checked -- gdn_chunk_fwd with recovery from an fp16 overflow.
 * The tensor-core kernels hand fp16 operands to the tensor cores, and a value
 * beyond fp16's range there is reported as GDN_ERR_RANGE in the device status
 * word, with unspecified results.  This call synchronises `stream`, reads the
 * word, and after a GDN_ERR_RANGE clears it and runs the request again on the
 * fp32 SIMT kernel (fp32 range, fp32 arithmetic; "Linear Attention,
 * Visualized": the same recurrence).
 *
 *   arguments   as for gdn_chunk_fwd; S_T may not overlap S0 (GDN_ERR_ARG):
 *               the second run reads S0.
 *   returns     GDN_OK, 1 when the fp32 kernel ran again (the results are
 *               its), a negative code otherwise.  If the status word already
 *               holds an error on entry, that code is returned and nothing
 *               runs (clear it with gdn_device_status(1) first).
 *
 * Blocks the host until `stream` is idle.  The status word is shared by the
 * library's kernels on the device: a range error of another call running at
 * the same time also triggers the second run.
 */
int gdn_chunk_fwd_checked(const gdn_desc_t *desc, const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *S0, void *o, float *S_T, void *stream);

/*
 * gdn_chunk_bwd -- the gradients of gdn_chunk_fwd (training backward).  For the
 * scalar loss L = sum(dO (.) o) + sum(dS_T (.) S_T) of gdn_chunk_fwd on the same
 * desc and inputs, writes dq = dL/dq, dk, dv, dg (dL/d log alpha), dbeta and
 * dS0.  Reverse mode through the recurrence of "Linear Attention, Visualized"
 * ("Recurrent form" of DeltaNet, "Gated DeltaNet (GDN)", "Kimi Delta
 * Attention (KDA)", "Mamba-2", "Gated Linear Attention (GLA)"; the additive
 * and decay writes as in gdn_chunk_fwd): the state entering every chunk of 64
 * tokens is kept ("Update the state": training keeps the chunk-boundary
 * states) and each chunk is recomputed before its gradients are stepped back
 * through it.  fp32 arithmetic.
 *
 *   desc        as for gdn_chunk_fwd (update, gate, dtype of q, k, v; dk, dv
 *               in {64, 128}; chunk 0 or 64); out_dtype is not read.  algo
 *               GDN_ALGO_TC: the tensor-core path -- the tensor-core forward
 *               writes the chunk-entry states into the workspace, then the
 *               chunkwise backward of gdn_chunk_bwd_tc runs from them (its
 *               requests only, GDN_ERR_UNSUPPORTED otherwise; results at the
 *               rounding of those two kernels).  Any other algo: the fp32 token
 *               backward described here.
 *               With prologue bits the inputs are the raw q, k, beta, g the
 *               forward mapped, and dq, dk, dbeta, dg are the gradients with
 *               respect to them (the chain rule through each map follows the
 *               recurrence's backward).
 *   q, k, v, g, beta, S0   the forward inputs, laid out as in gdn_chunk_fwd
 *               (S0 may be NULL = 0).
 *   dO          [B,H,T,dv] float, the gradient of o (NULL = 0).
 *   dS_T        [B,H,dv,dk] float, the gradient of S_T (NULL = 0).
 *   dq, dk      [B,H,T,dk] float;  dv [B,H,T,dv] float (required when B*H*T > 0)
 *   dg          [B,H,T] (scalar) or [B,H,T,dk] (channel) float; non-NULL iff
 *               gate != NONE
 *   dbeta       [B,H,T] float; non-NULL iff update == DELTA
 *   dS0         [B,H,dv,dk] float, or NULL (not written)
 *   workspace   device buffer of at least gdn_bwd_workspace_bytes(desc) bytes
 *               (B*H*ceil(T/64)*dv*dk*4: the chunk-boundary states; with prologue
 *               bits also the mapped q, k, v, beta, g in fp32; with GDN_ALGO_TC
 *               also gdn_bwd_tc_workspace_bytes(desc)), 16-byte aligned, owned by
 *               the caller; contents on return unspecified.  0 for a GDN_ALGO_TC
 *               request the tensor-core path does not serve.
 *
 * Every pointer 16-byte aligned; no output may overlap another output, an
 * input or the workspace (GDN_ERR_ARG).  dq, dk, dg and dbeta are sums over the
 * value rows of the state, accumulated across slices of 32 rows with float
 * atomics after being zeroed by the call, so they can differ from run to run
 * in the last bits; dv and dS0 are written once.  T == 0 writes dS0 = dS_T (or
 * zeros) and nothing else.  Asynchronous on `stream`; allocates nothing.
 */
size_t gdn_bwd_workspace_bytes(const gdn_desc_t *desc);
int gdn_chunk_bwd(const gdn_desc_t *desc, const void *q, const void *k, const void *v, const float *g,
                  const float *beta, const float *S0, const float *dO, const float *dS_T, float *dq, float *dk,
                  float *dv, float *dg, float *dbeta, float *dS0, void *workspace, size_t workspace_bytes,
                  void *stream);

/*
 * gdn_chunk_fwd_states -- gdn_chunk_fwd for training: the same o and S_T, and
 * in `states` the state entering every chunk of 64 tokens (before that chunk's
 * first decay; chunk 0's is S0), the chunk-boundary states that training keeps
 * ("Linear Attention, Visualized", "Update the state").  Runs the pipelined
 * tensor-core kernel, so the request must be one it serves: bf16 inputs,
 * dk = 128, dv in {64, 128}, prologue 0, algo AUTO or TC (GDN_ERR_UNSUPPORTED
 * otherwise).  The states carry that kernel's rounding (fp16 operands, fp32
 * accumulation).
 *
 *   states   [B,H,ceil(T/64),dv,dk] float, gdn_bwd_workspace_bytes(desc) bytes,
 *            16-byte aligned, owned by the caller; overlaps no other argument
 *            (GDN_ERR_ARG).  Not written when T == 0.
 *   others   as for gdn_chunk_fwd.
 *
 * gdn_chunk_bwd_states -- gdn_chunk_bwd from those saved states: the backward's
 * own forward pass over the sequence is skipped (each chunk is still recomputed
 * from its saved state).  Arguments as for gdn_chunk_bwd, with `states` (read
 * only; required when B*H*T > 0) in place of S0 and the workspace; prologue 0;
 * always the fp32 token backward (algo is not read: gdn_chunk_bwd_tc is the
 * tensor-core form from saved states).
 */
int gdn_chunk_fwd_states(const gdn_desc_t *desc, const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const float *S0, void *o, float *S_T, float *states, void *stream);
int gdn_chunk_bwd_states(const gdn_desc_t *desc, const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const float *states, const float *dO, const float *dS_T, float *dq,
                         float *dk, float *dv, float *dg, float *dbeta, float *dS0, void *stream);

/*
 * gdn_chunk_bwd_tc -- the same gradients as gdn_chunk_bwd_states, computed at
 * chunk granularity on tensor cores: reverse mode through the chunkwise form
 * ("Linear Attention, Visualized": "The triangular correction system",
 * "Optional: Use UT...", "Correct the incoming state", "Update the state"),
 * not through the token loop.  Three passes: every chunk's T = (I + L)^-1, W,
 * A and Q~ = diag(b) q - A W (all chunks in parallel); the gradient of the state
 * entering each chunk, dS_r = b_C dS_{r+1} - (dS_{r+1} K>^T) W + dO^T Q~ (the one
 * sequential pass, chunks last to first); every chunk-local gradient (all
 * chunks in parallel).  Products on tf32 tensor cores with fp32 accumulation,
 * so the results carry tf32 rounding (10-bit significand) on top of the saved
 * states'.  dq, dk, dv, dg, dbeta are written once per token (deterministic).
 *
 *   desc        update any, gate NONE or SCALAR, dk = 128, dv in {64, 128},
 *               dtype bf16 or f32, prologue 0, chunk 0 or 64, B*H <= 65535
 *               (GDN_ERR_UNSUPPORTED otherwise).
 *   states      [B,H,ceil(T/64),dv,dk] float, the chunk-entry states
 *               (gdn_chunk_fwd_states); required when B*H*T > 0.
 *   workspace   device buffer of at least gdn_bwd_tc_workspace_bytes(desc)
 *               bytes, 16-byte aligned, owned by the caller; contents on
 *               return unspecified.  Per chunk and head: T, A, P (.) Gamma
 *               (64 x 64), W, K>, Q~ (64 x dk), the state gradient (dv x dk)
 *               and b_C, in fp32 (T, P (.) Gamma, W, K> only for the delta rule).
 *   others      as for gdn_chunk_bwd_states.
 * gdn_bwd_tc_workspace_bytes returns 0 for a request the call does not serve.
 */
size_t gdn_bwd_tc_workspace_bytes(const gdn_desc_t *desc);
int gdn_chunk_bwd_tc(const gdn_desc_t *desc, const void *q, const void *k, const void *v, const float *g,
                     const float *beta, const float *states, const float *dO, const float *dS_T, float *dq,
                     float *dk, float *dv, float *dg, float *dbeta, float *dS0, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * gdn_device_status -- synchronises the current device, then returns the
 * library's device status word: GDN_OK, GDN_ERR_TIMEOUT or GDN_ERR_RANGE (the
 * first error any kernel of this library recorded since the last clear), or
 * GDN_ERR_CUDA if the synchronisation itself failed.  With clear != 0 the word
 * is reset to GDN_OK afterwards.  Kernels never trap: a kernel that records an
 * error finishes (possibly with partial results) and leaves the context usable.
 */
int gdn_device_status(int clear);

/*
 * gdn_device_diag -- synchronises the current device and returns where the
 * first recorded timeout happened: 0 if none, else 1 + site * 1000000 + chunk,
 * where site names the wait (1 input tiles, 2 chunk Gram product, 3 W/U
 * products, 4 history read, 5 output and state update) and chunk is the chunk
 * index.  Cleared together with the status word by gdn_device_status(1).
 */
int gdn_device_diag(void);

/*
 * gdn_set_wait_limit_ns -- the bound, in ns, of the waits by which a kernel's
 * warps hand work to one another (the mbarrier phases of TMA loads, MMAs and
 * producer / consumer steps of the tensor-core prefill, linear-attention and
 * multi-token decode kernels); 0 restores the default of 1 s.  A wait that
 * runs out records GDN_ERR_TIMEOUT in the status word (the tensor-core prefill
 * also its site in the diagnostic word); the kernel then lets every copy and
 * MMA it issued land
 * (each of those waits bounded at 1 s whatever this setting) and returns,
 * with o and S_T unspecified.  For tests of that path: a process-wide setting
 * read when a call launches, not thread-safe.  Returns GDN_OK.
 */
int gdn_set_wait_limit_ns(unsigned long long ns);

/* GDN_VERSION of the built library. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
