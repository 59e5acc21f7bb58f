/*
 * libssd -- Mamba-2 SSD (structured state-space duality) layer core on one
 * NVIDIA B200 (sm_100a).  C ABI: plain pointers, sizes and status codes; no
 * C++ or framework types cross this boundary.
 *
 * The operation (per batch element b and head h; the state is N x P):
 *
 *   dt_t = softplus(dt_raw[t,h] + dt_bias[h])
 *   h_t  = exp(dt_t * A[h]) * h_{t-1} + dt_t * B_t x_t^T
 *   y_t  = C_t^T h_t + D[h] * x_t
 *
 * Where it is defined (page titles and sections; the pages print no formula,
 * these are the statements the formula above follows):
 *  - transition = a scalar times the identity: "Mamba3" (Telegram post,
 *    ai_machinelearning_big_data), first paragraph; "Mamba-3 : SSM optimise
 *    inference", section "Du training-first a l'inference-first".
 *  - ZOH on the state, Euler on the input: "Mamba3", section "New
 *    discretisation scheme" (Mamba-1 and Mamba-2 mix ZOH and Euler).
 *  - two paths: the blocked (chunked) contraction of the semiseparable matrix
 *    for a whole sequence, and the O(1) recurrent step at generation time:
 *    "Mamba-2 vs Transformers / SSD", sections "Mamba-2 and the SSD paper:
 *    what changed in practice" and "How to decide..." (table: streaming
 *    inference, O(1) recurrent step).
 *
 * Readings where the pages are silent:
 *  - y_t reads the state after the token-t update.
 *  - head h uses group g = h / (nheads / ngroups) of B and C.
 *  - dt_bias, A and D are one fp32 scalar per head; a NULL dt_bias or D means 0.
 *  - no clamp and no threshold on dt (softplus is exact up to fp32 rounding).
 *
 * Layouts (row-major, last index fastest, every tensor densely packed):
 *   prefill: x, y [batch][seqlen][nheads][headdim]; dt_raw [batch][seqlen][nheads];
 *            B, C [batch][seqlen][ngroups][dstate];
 *            init_state, final_state [batch][nheads][dstate][headdim].
 *   decode:  x, y [batch][nheads][headdim]; dt_raw [batch][nheads];
 *            B, C [batch][ngroups][dstate]; state [batch][nheads][dstate][headdim].
 *
 * Conventions shared by every call:
 *  - Ownership: the caller owns every pointer, all device memory and the
 *    stream.  The library allocates no device memory; the prefill takes a
 *    caller-owned workspace of at least ssd_chunk_scan_workspace_size() bytes.
 *  - All tensor pointers are device pointers.  dt_bias, A and D are device
 *    pointers too.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *  - Asynchrony: the compute calls only enqueue work on `stream` and never
 *    synchronise; SSD_OK means "enqueued".  Results are ready when the stream
 *    is.
 *  - Validation happens on the host before anything is enqueued; on any error
 *    nothing is launched and no memory is touched.
 *  - Alignment: every tensor base pointer must be 16-byte aligned
 *    (SSD_ERR_ALIGNMENT otherwise).
 *  - Reentrancy: the library keeps no per-call host state; concurrent calls on
 *    different streams must use different workspaces.
 */
#ifndef LIBSSD_SSD_H
#define LIBSSD_SSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,     /* NULL required pointer, bad dimension, bad dtype, aliasing */
    SSD_ERR_UNSUPPORTED = 2,     /* valid request this build does not implement */
    SSD_ERR_ALIGNMENT = 3,       /* a tensor base pointer is not 16-byte aligned */
    SSD_ERR_WORKSPACE = 4,       /* workspace NULL or smaller than required */
    SSD_ERR_CUDA = 5,            /* a CUDA runtime/driver call failed (launch, attribute, ...) */
    SSD_ERR_DEVICE_TIMEOUT = 6   /* a bounded device-side wait gave up (see ssd_get_device_error) */
} ssd_status_t;

typedef enum {
    SSD_F32 = 0,   /* IEEE binary32 */
    SSD_BF16 = 1   /* bfloat16 (stored as 16-bit patterns; results rounded to nearest even) */
} ssd_dtype_t;

/* Prefill problem description.  Enum fields are int32_t holding ssd_dtype_t. */
typedef struct {
    int64_t batch;      /* >= 0; 0 is a no-op */
    int64_t seqlen;     /* >= 0; 0 writes final_state = init_state (or zeros) */
    int64_t nheads;     /* H >= 1 */
    int64_t headdim;    /* P, multiple of 8, <= 256 */
    int64_t dstate;     /* N, multiple of 8, <= 256 */
    int64_t ngroups;    /* G >= 1, nheads % ngroups == 0 */
    int64_t chunk;      /* Q: power of two in [16, 256]; seqlen need not be a multiple */
    int32_t io_dtype;   /* dtype of x, dt_raw, B, C */
    int32_t y_dtype;    /* dtype of y */
    int32_t state_dtype;/* dtype of init_state and final_state */
} ssd_prefill_desc_t;

/* Decode (single-token state update) problem description. */
typedef struct {
    int64_t batch;      /* >= 0; 0 is a no-op */
    int64_t nheads;
    int64_t headdim;    /* P, multiple of 8, <= 256 */
    int64_t dstate;     /* N, multiple of 8, <= 256 */
    int64_t ngroups;
    int32_t io_dtype;   /* dtype of x, dt_raw, B, C */
    int32_t y_dtype;    /* dtype of y */
    int32_t state_dtype;/* dtype of the in-place state */
} ssd_decode_desc_t;

/* MIMO (rank-R) decode problem description. */
typedef struct {
    int64_t batch;      /* >= 0; 0 is a no-op */
    int64_t nheads;
    int64_t headdim;    /* P: 8, 16, 32, 64 or 128 */
    int64_t dstate;     /* N, multiple of 8, <= 256 */
    int64_t ngroups;
    int64_t rank;       /* R: 1, 2, 4 or 8 */
    int32_t io_dtype;   /* dtype of x, dt_raw, B, C */
    int32_t y_dtype;    /* dtype of y */
    int32_t state_dtype;/* dtype of the in-place state */
} ssd_mimo_desc_t;

/* Replayed decode (checkpoint + buffer of recent tokens) problem description. */
typedef struct {
    int64_t batch;      /* >= 0; 0 is a no-op */
    int64_t nheads;
    int64_t headdim;    /* P: 8, 16, 32, 64 or 128 */
    int64_t dstate;     /* N, multiple of 8, <= 256 */
    int64_t ngroups;
    int32_t io_dtype;   /* dtype of x, dt_raw, B, C (and of their buffered copies) */
    int32_t y_dtype;    /* dtype of y */
    int32_t state_dtype;/* dtype of the checkpoint */
    int32_t capacity;   /* K, 1..16: tokens after the checkpoint the buffer holds; the
                           step that brings it to K folds them into the checkpoint */
} ssd_replay_desc_t;

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int ssd_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* ssd_status_string(ssd_status_t status);

/*
 * Bytes of device workspace ssd_chunk_scan_fwd needs for `desc` (written to
 * *bytes).  Pure host function: touches no device.  The workspace holds the
 * per-token dt and chunk-local decay cumsum (fp32), the in-flight fp32 chunk
 * states of the inter-chunk state-passing scan, and its progress flags.
 * Errors: SSD_ERR_INVALID_ARG / SSD_ERR_UNSUPPORTED as for ssd_chunk_scan_fwd.
 */
ssd_status_t ssd_chunk_scan_workspace_size(const ssd_prefill_desc_t* desc, size_t* bytes);

/*
 * Which kernel path ssd_chunk_scan_fwd takes for `desc` (written to *path):
 *   0 = tensor-core path (bf16 inputs; tcgen05 MMAs with TMEM accumulators fed
 *       by TMA; fp32 accumulation and fp32 state passing): headdim 64,
 *       dstate 64, 128 or 256, chunk 128 or 256,
 *   1 = CUDA-core fp32 path (fp32 inputs, or shapes the tensor-core path does
 *       not cover),
 *   2 = the tensor-core path over pairs of heads of one group, which share
 *       B, C and C B^T: dstate 128 with an even number of heads per group and
 *       at least 148 (batch, head) sequences; same arithmetic as path 0.
 * Pure host function.
 */
ssd_status_t ssd_chunk_scan_path(const ssd_prefill_desc_t* desc, int32_t* path);

/*
 * Chunked prefill scan over whole sequences: the semiseparable matrix is
 * contracted chunk by chunk ("Mamba-2 vs Transformers / SSD", section "Mamba-2
 * and the SSD paper: what changed in practice": chunks processed in parallel,
 * then the per-chunk SSM states recombined).  Per chunk of Q tokens it
 * computes the chunk-local decay cumsum, the intra-chunk block
 * (C B^T o L)(dt x), the chunk state B^T(decay dt x) and the off-diagonal
 * term exp(cumsum) C h_in; an fp32 scan over chunks carries the state.
 *
 *  (x, dt_raw, B, C and y may be NULL when batch == 0 or seqlen == 0)
 *  x           [b][L][H][P]   io_dtype   required
 *  dt_raw      [b][L][H]      io_dtype   required
 *  dt_bias     [H]            fp32       nullable (= 0)
 *  A           [H]            fp32       required (taken as given; A <= 0 is the intended use)
 *  B, C        [b][L][G][N]   io_dtype   required
 *  D           [H]            fp32       nullable (= 0)
 *  init_state  [b][H][N][P]   state_dtype nullable (= zero state, not read)
 *  y           [b][L][H][P]   y_dtype    required, written; must not overlap x
 *  final_state [b][H][N][P]   state_dtype nullable (not written), else written
 *  workspace   >= ssd_chunk_scan_workspace_size bytes, 256-byte aligned; its
 *              contents on entry are irrelevant; clobbered
 * Errors: SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_ALIGNMENT,
 *         SSD_ERR_WORKSPACE (nothing launched), SSD_ERR_CUDA (launch failed;
 *         outputs undefined).
 */
ssd_status_t ssd_chunk_scan_fwd(const ssd_prefill_desc_t* desc,
                                const void* x, const void* dt_raw, const float* dt_bias,
                                const float* A, const void* B, const void* C, const float* D,
                                const void* init_state, void* y, void* final_state,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * ssd_chunk_scan_fwd for a batch of variable-length, left-padded sequences
 * (one of the adjacent steps the pages list with the Mamba-3 variants; the
 * Hugging Face integration they cite batches with left padding).  Sequence b
 * starts at token pad_left[b]: the tokens before it are absent from the
 * recurrence (dt = 0 there: no decay, no input), so final_state[b] and y[b]
 * from pad_left[b] on equal those of the unpadded sequence alone, started
 * from init_state[b].  y at the padding positions is computed as if dt = 0
 * (C_t^T h + D x_t with h the initial state); callers ignore it.
 *  pad_left  [b] int32, device, required when batch > 0, 4-byte aligned;
 *            values outside [0, seqlen] are clamped by their effect (a value
 *            >= seqlen pads the whole sequence, a negative one nothing)
 * All other arguments and errors as ssd_chunk_scan_fwd.
 */
ssd_status_t ssd_chunk_scan_fwd_varlen(const ssd_prefill_desc_t* desc,
                                       const void* x, const void* dt_raw, const float* dt_bias,
                                       const float* A, const void* B, const void* C, const float* D,
                                       const void* init_state, const int32_t* pad_left, void* y,
                                       void* final_state, void* workspace, size_t workspace_bytes,
                                       void* stream);

/*
 * Backward pass of ssd_chunk_scan_fwd (training).  The pages only state that
 * end-to-end training also needs it ("Mamba-3 : SSM optimise inference",
 * opening paragraph); it is the gradient of
 *     loss = sum_t <dy_t, y_t> + <dfinal_state, final_state>
 * with respect to every input of the forward call for the same descriptor.
 * The state adjoint G_t = C_t dy_t^T + exp(dt_{t+1} A) G_{t+1} is computed as
 * the forward's chunked scan run backwards in time; G_t x_t and h_t dy_t as
 * the same scan on transposed states; the decay gradients from the identity
 * d loss / d (cumulative log-decay at u) = dy_u.(y_u - D x_u) - dt_u x_u.(B_u^T G_u)
 * (+ <dfinal, h_{L-1}> at u = L-1), suffix-summed over the sequence.
 *
 *  inputs: exactly those of ssd_chunk_scan_fwd (same layouts and dtypes), plus
 *  dy           [b][L][H][P]   io_dtype    required (NULL allowed if empty)
 *  dfinal_state [b][H][N][P]   state_dtype nullable (= 0, final state not used)
 *  outputs (every one written, none may overlap an input or another output):
 *  dx           [b][L][H][P]   y_dtype     required
 *  ddt_raw      [b][L][H]      y_dtype     required
 *  dB, dC       [b][L][G][N]   y_dtype     required (summed over a group's heads)
 *  dA           [H]            fp32        required (summed over batch and tokens)
 *  ddt_bias, dD [H]            fp32        nullable (not written)
 *  dinit_state  [b][H][N][P]   state_dtype nullable (not written)
 *  workspace    >= ssd_chunk_scan_bwd_workspace_size bytes, 256-byte aligned,
 *               clobbered
 * The path (tensor-core or CUDA-core) follows ssd_chunk_scan_path for the
 * adjoint scan; the transposed scans (headdim N in 64-column slices, dstate
 * P) take the tensor-core path when bf16 inputs have headdim 64.
 * Empty problems (batch 0 or seqlen 0) launch one kernel: dA, ddt_bias and dD
 * are zeroed and dinit_state = dfinal_state (or zero); no workspace is needed.
 * Errors: as ssd_chunk_scan_fwd; the parameter gradients are plain fp32 sums
 * (deterministic: no atomics).
 */
ssd_status_t ssd_chunk_scan_bwd(const ssd_prefill_desc_t* desc,
                                const void* x, const void* dt_raw, const float* dt_bias,
                                const float* A, const void* B, const void* C, const float* D,
                                const void* init_state, const void* dy, const void* dfinal_state,
                                void* dx, void* ddt_raw, float* ddt_bias, float* dA, void* dB, void* dC,
                                float* dD, void* dinit_state, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Workspace bytes ssd_chunk_scan_bwd needs for `desc`.  Pure host function. */
ssd_status_t ssd_chunk_scan_bwd_workspace_size(const ssd_prefill_desc_t* desc, size_t* bytes);

/*
 * Number of kernels one ssd_chunk_scan_bwd call launches for `desc`
 * (has_states: dfinal_state or init_state given).  Pure host function.
 */
ssd_status_t ssd_chunk_scan_bwd_launches(const ssd_prefill_desc_t* desc, int32_t has_states,
                                         int32_t* launches);

/*
 * Mamba-3 prefill: the chunked scan of the Mamba-3 recurrence, with an
 * exponential-trapezoidal input ("Mamba3", section "New discretisation
 * scheme": both ends of each step's interval, mixed by a learned coefficient)
 * and a rotational (complex) state ("Mamba3", section on complex-valued SSMs;
 * "Mamba-3 : SSM optimise inference", "Etats complexes via RoPE").  Per batch
 * b and head h, with the state rows (2k, 2k+1) forming the rotating pair k:
 *   h_t = exp(dt_t A) R(theta_t) (h_{t-1} + (1 - lam_t) dt_t B_{t-1} x_{t-1}^T)
 *         + lam_t dt_t B_t x_t^T
 *   y_t = C_t^T h_t + D x_t
 * R(theta) turns (h[2k], h[2k+1]) counter-clockwise by theta[t][g][k]; there
 * is no input before the first token.  Computed, as the pages suggest, by
 * turning B and C with the cumulative angle and running the real chunked scan
 * with the trapezoid's weights (a token's own term weighted lam dt): with bf16
 * inputs and the head-pair shapes (N = 128, P = 64, an even number of heads per
 * group, batch * nheads >= 148) in one scan over the turned operands' bf16
 * hi/lo pairs, otherwise as three scans and a combination.
 *
 *  arguments as ssd_chunk_scan_fwd, plus
 *  lam    [b][L][H]      fp32  nullable (= 1: Euler input, Mamba-2's)
 *  theta  [b][L][G][N/2] fp32  nullable (= 0: real state)
 *  With both NULL this is ssd_chunk_scan_fwd.
 *  workspace >= ssd_chunk_scan_mamba3_workspace_size bytes, 256-byte aligned.
 * Errors: as ssd_chunk_scan_fwd.
 */
ssd_status_t ssd_chunk_scan_fwd_mamba3(const ssd_prefill_desc_t* desc,
                                       const void* x, const void* dt_raw, const float* dt_bias,
                                       const float* A, const void* B, const void* C, const float* D,
                                       const float* lam, const float* theta, const void* init_state,
                                       void* y, void* final_state, void* workspace, size_t workspace_bytes,
                                       void* stream);

/* Workspace bytes ssd_chunk_scan_fwd_mamba3 needs for `desc`.  Pure host function. */
ssd_status_t ssd_chunk_scan_mamba3_workspace_size(const ssd_prefill_desc_t* desc, size_t* bytes);

/* Kernels one ssd_chunk_scan_fwd_mamba3 call launches (flags: lam given,
 * theta given, final_state given).  Pure host function. */
ssd_status_t ssd_chunk_scan_mamba3_launches(const ssd_prefill_desc_t* desc, int32_t has_lam, int32_t has_theta,
                                            int32_t has_final_state, int32_t* launches);

/* Size of the scratch array ssd_chunk_scan_fwd_noalloc uses (32 MiB per GPU). */
#define SSD_NOALLOC_WORKSPACE_BYTES ((size_t)32 << 20)

/*
 * ssd_chunk_scan_fwd without a caller workspace, for callers that cannot
 * allocate device memory: code that may only touch the input and output
 * buffers it is given (for example a plugin inside a framework that owns all
 * device memory), or a path where cudaMalloc -- which can synchronise the
 * device -- is not allowed.  The pages describe no such variant; this is a
 * convenience of the library.
 *
 * Arguments and results are exactly those of ssd_chunk_scan_fwd minus the
 * workspace.  The scratch is a fixed array of SSD_NOALLOC_WORKSPACE_BYTES in
 * the library's own device memory; nothing is allocated per call (no
 * cudaMalloc, cudaFree or allocating library routine).
 *  - Problems whose ssd_chunk_scan_workspace_size exceeds the scratch are
 *    rejected with SSD_ERR_WORKSPACE before anything is launched (the 1.3B-
 *    shaped layer, batch 4 x 2048 tokens, needs about 12.6 MiB).
 *  - The first call with a given device current looks up the scratch's device
 *    address on that device.  With the CUDA runtime's lazy module loading
 *    (its default), that first lookup is also when the library's device code
 *    is loaded on the device and the scratch is reserved, which may allocate
 *    device memory and synchronise.  Make one warm-up call per device outside
 *    any latency-critical region and before any stream capture; from then on
 *    the scratch stays reserved on that device until the process exits.
 *  - The address is kept for the life of the process: after cudaDeviceReset
 *    (or anything else that destroys the device's primary context) it is
 *    stale, so do not call this entry point again in that process.
 *  - Every call on a device shares the one scratch array, which keeps the last
 *    call's contents (the kernels reset what must start at zero themselves).
 *    Calls that overlap on the GPU -- on different streams, or from different
 *    threads -- race on it: serialise them.
 * Errors: as ssd_chunk_scan_fwd, plus SSD_ERR_WORKSPACE for a problem too
 * large for the scratch, SSD_ERR_CUDA if the scratch cannot be located.
 */
ssd_status_t ssd_chunk_scan_fwd_noalloc(const ssd_prefill_desc_t* desc,
                                        const void* x, const void* dt_raw, const float* dt_bias,
                                        const float* A, const void* B, const void* C, const float* D,
                                        const void* init_state, void* y, void* final_state, void* stream);

/*
 * Single-token decode step, in place on the state ("Mamba-2 vs Transformers /
 * SSD", section "How to decide...": O(1) recurrent step; "Mamba3", section on
 * Mamba-2: decoding moves the state between memory levels rather than
 * computing -- the step is one streaming read-modify-write of the state):
 *
 *   state[b,h] <- exp(dt A) state[b,h] + dt B x^T;  y = C^T state[b,h] + D x
 *
 *  state  [b][H][N][P]  state_dtype  required, read and written in place
 *                                     (bf16 state is rounded to nearest even)
 *  x      [b][H][P]     io_dtype     required
 *  dt_raw [b][H]        io_dtype     required
 *  dt_bias, A, D [H]    fp32         dt_bias, D nullable
 *  B, C   [b][G][N]     io_dtype     required
 *  y      [b][H][P]     y_dtype      required; must not overlap state or x
 * Errors: as ssd_chunk_scan_fwd (no workspace).
 */
ssd_status_t ssd_state_update(const ssd_decode_desc_t* desc, void* state, const void* x,
                              const void* dt_raw, const float* dt_bias, const float* A,
                              const void* B, const void* C, const float* D, void* y,
                              void* stream);

/*
 * MIMO decode step, in place on the state: B and C widened to rank R, the
 * state keeps its N x P size ("Mamba3" (Telegram post), section on the switch
 * from SISO to MIMO: the outer products become matrix products; "Mamba-3 :
 * SSM optimise inference", section "Mode MIMO": several SSMs in parallel with
 * extended B and C, more arithmetic for the same decode memory traffic).
 * Per (b, h), with the R inputs x_r and outputs y_r of a token:
 *
 *   state <- exp(dt A) state + dt sum_r B_r x_r^T;   y_r = C_r^T state + D x_r
 *
 * rank 1 is ssd_state_update.
 *  state  [b][H][N][P]     state_dtype  required, read and written in place
 *                                        (bf16 state is rounded to nearest even)
 *  x      [b][H][R][P]     io_dtype     required
 *  dt_raw [b][H]           io_dtype     required (one dt per head and token)
 *  dt_bias, A, D [H]       fp32         dt_bias, D nullable
 *  B, C   [b][G][R][N]     io_dtype     required
 *  y      [b][H][R][P]     y_dtype      required; must not overlap state or x
 * Errors: SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED (headdim not 8/16/32/64/128,
 * rank not 1/2/4/8, dstate), SSD_ERR_ALIGNMENT, SSD_ERR_CUDA; nothing is
 * launched on a host-side error.
 */
ssd_status_t ssd_state_update_mimo(const ssd_mimo_desc_t* desc, void* state, const void* x,
                                   const void* dt_raw, const float* dt_bias, const float* A,
                                   const void* B, const void* C, const float* D, void* y,
                                   void* stream);

/*
 * Mamba-3 decode step, in place on the state: the exponential-trapezoidal
 * input ("Mamba3" Telegram post, section "New discretisation scheme": the
 * input is taken at both ends of the step and mixed by a learned weight) and
 * the rotational state ("Mamba3", section on the complex-valued SSM; "Mamba-3 :
 * SSM optimise inference", section "Etats complexes via RoPE": state pairs turn
 * by data-dependent angles).  With dt = softplus(dt_raw + dt_bias), lam the mix
 * and R(theta) turning state rows (2k, 2k+1) by theta[k]:
 *
 *   h <- exp(dt A) R(theta) (h + (1 - lam) dt B_prev x_prev^T) + lam dt B x^T
 *   y  = C^T h + D x
 *
 * lam = 1 and theta = 0 give ssd_state_update.  The trapezoid reaches one token
 * back, so the decode state is the SSM state plus the previous token's B and x;
 * the caller passes those (its previous call's B and x) and keeps them: the call
 * writes only the state and y.  The prefill's form is ssd_chunk_scan_fwd_mamba3.
 *
 *  desc   as ssd_state_update (io_dtype for x, x_prev, dt_raw, B, B_prev, C)
 *  state  [b][H][N][P]  state_dtype  required, read and written in place
 *  x      [b][H][P]     io_dtype     required
 *  x_prev [b][H][P]     io_dtype     the previous token's x; NULL (with B_prev)
 *                                     before the first token: no left end
 *  dt_raw [b][H]        io_dtype     required
 *  dt_bias, A, D [H]    fp32         dt_bias, D nullable
 *  B, C   [b][G][N]     io_dtype     required
 *  B_prev [b][G][N]     io_dtype     the previous token's B; NULL with x_prev
 *  lam    [b][H]        fp32         nullable (= 1: Mamba-2's input)
 *  theta  [b][G][N/2]   fp32         radians; nullable (= 0: no rotation)
 *  y      [b][H][P]     y_dtype      required; must not overlap state, x or x_prev
 * dstate must be even; headdim a power-of-two count of 16-byte state vectors
 * that divides 32 (P <= 128 for fp32 states, <= 256 for bf16).
 * Errors: SSD_ERR_INVALID_ARG (bad descriptor, NULL required pointer, only one
 * of x_prev / B_prev, overlapping outputs), SSD_ERR_UNSUPPORTED (shape),
 * SSD_ERR_ALIGNMENT, SSD_ERR_CUDA; nothing is launched on a host-side error.
 */
ssd_status_t ssd_state_update_mamba3(const ssd_decode_desc_t* desc, void* state, const void* x,
                                     const void* x_prev, const void* dt_raw, const float* dt_bias,
                                     const float* A, const void* B, const void* B_prev, const void* C,
                                     const float* D, const float* lam, const float* theta, void* y,
                                     void* stream);

/*
 * Bytes of the replay buffer ssd_replay_step needs for `desc` (written to
 * *bytes).  Pure host function.  Errors: SSD_ERR_INVALID_ARG /
 * SSD_ERR_UNSUPPORTED as for ssd_replay_step.
 */
ssd_status_t ssd_replay_buffer_size(const ssd_replay_desc_t* desc, size_t* bytes);

/*
 * One decode step on a state held as a checkpoint plus a buffer of the tokens
 * after it ("Mamba3" (Telegram post) and "Mamba-3 : SSM optimise inference",
 * ReplaySSM: outputs are computed from the checkpoint and the buffered inputs
 * on most steps; the state is written back only when the buffer fills).
 *
 * Before the call the state of sequence (b, h) is the checkpoint advanced by
 * the `fill` buffered tokens; the call takes token t and returns
 *   y_t = C_t^T h_t + D x_t,   h_t = exp(dt_t A) h_{t-1} + dt_t B_t x_t^T
 * (the decode step of ssd_state_update, up to rounding).  If fill + 1 <
 * capacity, token t is appended to the buffer and the checkpoint is only read
 * (the caller's next fill is fill + 1); if fill + 1 == capacity, all buffered
 * tokens and t are folded into the checkpoint, which then holds h_t (the
 * caller's next fill is 0).  A bf16 checkpoint is rounded (to nearest even) at
 * those folds only.  Averaged over capacity steps, the state is read once per
 * step and written once per capacity steps.
 *
 *  checkpoint [b][H][N][P]  state_dtype  required; read every step, written
 *                                        on the folding step
 *  buffer     ssd_replay_buffer_size bytes, 256-byte aligned, caller-owned;
 *             its layout is the library's; its contents are irrelevant when
 *             fill == 0 and must be left as the previous call left them otherwise
 *  fill       0 <= fill < capacity: tokens currently buffered (host value);
 *             start a sequence with the initial state in the checkpoint and fill 0
 *  x [b][H][P], dt_raw [b][H], B, C [b][G][N]: io_dtype, required
 *  dt_bias, A, D [H] fp32 (dt_bias, D nullable); y [b][H][P] y_dtype, required
 * Calls on one buffer must be ordered on one stream (each step reads what the
 * previous one appended).  Rollback (speculative decoding, which the pages name
 * as a use): until the buffer is folded the checkpoint is only read, so the
 * last k buffered tokens are dropped by calling again with fill - k; tokens
 * already folded into the checkpoint cannot be dropped.
 * Errors: SSD_ERR_INVALID_ARG (bad descriptor, fill out of range, NULL
 * pointers, y/x/checkpoint/buffer overlapping), SSD_ERR_UNSUPPORTED
 * (headdim not 8/16/32/64/128, dstate, capacity > 16), SSD_ERR_ALIGNMENT,
 * SSD_ERR_CUDA; nothing is launched on a host-side error.
 */
ssd_status_t ssd_replay_step(const ssd_replay_desc_t* desc, void* checkpoint, void* buffer, int32_t fill,
                             const void* x, const void* dt_raw, const float* dt_bias, const float* A,
                             const void* B, const void* C, const float* D, void* y, void* stream);

/*
 * Synchronises `stream`, then reports (and clears) the device-side error word
 * of the current device.  Kernels never trap: a bounded wait that gives up
 * (the inter-chunk state hand-off of the prefill waits for the previous
 * chunk's state with an iteration limit) records it there and returns.
 * Returns SSD_OK, SSD_ERR_DEVICE_TIMEOUT, or SSD_ERR_CUDA if synchronisation
 * itself failed.  If `detail` is not NULL it receives the raw error bits.
 * The word is shared by all streams of the device: call it when no other
 * libssd work is in flight.
 */
ssd_status_t ssd_get_device_error(void* stream, uint32_t* detail);

/* Fault-injection bits for ssd_debug_inject. */
#define SSD_FAULT_DROP_RUN_PUBLISH 0x1u

/*
 * Test hook for the device-side failure path; never needed in normal use.
 * Sets the faults injected into every following launch until called again
 * with 0 (process-wide, all devices).
 *  SSD_FAULT_DROP_RUN_PUBLISH: on the tensor-core prefill path, the state
 *    item that computes the entry state of a run of chunks never signals it.
 *    The bounded waits (2 s) of the items that need it then expire: the
 *    launch still completes (its outputs are undefined), and
 *    ssd_get_device_error reports SSD_ERR_DEVICE_TIMEOUT with bit 0x1 (a
 *    hand-off wait timed out) and possibly 0x2 (other waits cut short) in
 *    *detail.  Nothing traps and the CUDA context stays usable.  Sequences
 *    are cut into runs only when a prefill has fewer (batch x head) sequences
 *    than half the block pipelines (148 on a 148-SM part, 74 at dstate 256).
 * Errors: SSD_ERR_INVALID_ARG for unknown bits (nothing changed).
 */
ssd_status_t ssd_debug_inject(uint32_t faults);

#ifdef __cplusplus
}
#endif

#endif /* LIBSSD_SSD_H */
