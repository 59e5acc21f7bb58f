// Host-side declarations shared by the libssd translation units (not part of
// the public C ABI in include/ssd.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ssd {

struct DecodeArgs {
    int64_t batch, H, P, N, G;
    bool io_bf16, y_bf16, state_bf16;
    void* state;
    const void *x, *dt_raw, *B, *C;
    const float *dt_bias, *A, *D;
    void* y;
};

cudaError_t launch_state_update(const DecodeArgs& a, cudaStream_t stream);

// Mamba-3 decode step: trapezoidal input, rotational state (ssd_mamba3_decode.cu).
struct Mamba3StepArgs {
    int64_t batch, H, P, N, G;
    bool io_bf16, y_bf16, state_bf16;
    void* state;
    const void *x, *x_prev, *dt_raw, *B, *B_prev, *C;   // x, x_prev [b][H][P]; B, B_prev, C [b][G][N]
    const float *dt_bias, *A, *D, *lam, *theta;         // lam [b][H]; theta [b][G][N/2]
    void* y;
};

bool mamba3_step_supports(int64_t P, int64_t N, bool state_bf16);
cudaError_t launch_mamba3_step(const Mamba3StepArgs& a, cudaStream_t stream);

// Replayed decode step: checkpoint + buffer of the last tokens (ssd_replay.cu).
struct ReplayArgs {
    int64_t batch, H, P, N, G, K, fill;
    bool io_bf16, y_bf16, state_bf16;
    void* ckpt;
    void *xb, *Bb;                 // buffered x [b][H][K][P], B [b][G][K][N] (io dtype)
    float *dtb, *cumb;             // buffered dt, log-decay cumsum [b][H][K]
    float* cb;                     // the step's C_t . B_s [b][G][16]
    const void *x, *dt_raw, *B, *C;
    const float *dt_bias, *A, *D;
    void* y;
};

// Byte offsets of the replay buffer's parts (all 256-byte aligned) and its size.
struct ReplayLayout {
    size_t off_x, off_B, off_dt, off_cum, off_cb, total;
};

cudaError_t launch_replay_step(const ReplayArgs& a, cudaStream_t stream);

// MIMO (rank-R) decode step (ssd_mimo.cu).
struct MimoArgs {
    int64_t batch, H, P, N, G, R;
    bool io_bf16, y_bf16, state_bf16;
    void* state;
    const void *x, *dt_raw, *B, *C;   // x [b][H][R][P]; B, C [b][G][R][N]
    const float *dt_bias, *A, *D;
    void* y;                          // [b][H][R][P]
};

cudaError_t launch_mimo_step(const MimoArgs& a, cudaStream_t stream);

// Workspace carve-up of the prefill (all offsets 256-byte aligned).
struct PrefillLayout {
    int64_t nchunks;       // ceil(L / Q)
    int64_t Lpad;          // nchunks * Q
    size_t off_dt, off_acs;        // fp32 [b][H][Lpad] each; acs is the hi part of the cumsum
    size_t off_acs_lo;             // fp32 [b][H][Lpad]: its lo part (when has_lo)
    bool has_lo;                   // layouts of scans whose decays are written by other kernels have none
    size_t off_states;             // fp32 chunk states (CUDA-core path) or run-entry states
    size_t off_flags;              // int32 [b][H] run-entry states published + 64 control words
    size_t total;
};

struct PrefillArgs {
    int64_t batch, L, H, P, N, G, Q;
    bool io_bf16, y_bf16, state_bf16;
    const void *x, *dt_raw, *B, *C;
    const float *dt_bias, *A, *D;
    const void* init_state;
    void* y;
    void* final_state;
    char* ws;
    PrefillLayout lay;
    const int32_t* pad_left;  // [batch] leading tokens to treat as absent (dt = 0), or NULL
    unsigned* dev_err;     // device error word of the current device
    int drop_publish;      // fault injection (ssd_debug_inject): run-entry states are never published
};

// chunk-local dt / decay cumsum (shared by both prefill paths)
cudaError_t launch_dt_cumsum(const PrefillArgs& a, cudaStream_t s);
// CUDA-core fp32 prefill path (chunk states, state passing, chunk outputs)
cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s);
// tensor-core prefill path; returns cudaErrorNotSupported when the shape is not covered
bool tc_path_supports(int64_t P, int64_t N, int64_t Q, bool io_bf16);
// runs per sequence of the tensor-core path (1 = every work item is a whole sequence)
int64_t tc_runs(int64_t BH, int64_t nchunks, int64_t N);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s);
// tensor-core prefill over pairs of heads of one group (ssd_prefill_pair.cu);
// launch_prefill_tc takes it for the shapes it covers
bool pair_path_supports(int64_t batch, int64_t H, int64_t P, int64_t N, int64_t G, int64_t Q, bool io_bf16);
cudaError_t launch_prefill_pair(const PrefillArgs& a, cudaStream_t s);
// its Mamba-3 form: B, C are the turned operands as [b][L][G][2][N] bf16 (hi, lo),
// dt and the cumsum slots of the workspace hold the trapezoid's weights and the
// decay cumsum, dgw [BH][Lpad] the weight of each token's own term (or NULL: the
// scan weight), rot [b][G][N/2] cos, sin of the last token's angle (the final
// state is turned back by it as it is written); the initial state is read as
// bf16 when init_bf16, the final one written per a.state_bf16
cudaError_t launch_prefill_pair_mamba3(const PrefillArgs& a, const float* dgw, const float2* rot, bool init_bf16,
                                       cudaStream_t s);

// Backward pass of the prefill (ssd_backward.cu).  Workspace carve-up, all
// offsets 256-byte aligned; "slice" strides separate the column slices of the
// transposed scans.
struct BackwardLayout {
    // 0: three chunked scans on rearranged operands; 1: block form on CUDA cores
    // (ssd_backward_blocks.cu); 2: block form on tensor cores (ssd_backward_tc.cu)
    int mode;
    int64_t qb, nb;                // block form: tokens per block, blocks per sequence
    size_t off_h0, off_ge;         // block form: entry states, end adjoints [b*H][nb][N] x
                                   // (mode 1: fp32 [P]; mode 2: bf16 [2 (hi, lo)][P])
    size_t off_dbc;                // mode 2: fp32 dB, dC partials [grid * smax][2][128][128]
    int64_t nchunks, Lpad;
    int64_t pw, nblk;              // column-slice width of the transposed scans, slices
    bool tc_main, tc_t;            // tensor-core path for the adjoint scan / transposed scans
    size_t off_dtf, off_acsf, off_dtr, off_acsr;   // fp32 [b*H][Lpad]: forward and reversed
    size_t off_states, off_flags;                  // shared by the scans (run one after another)
    size_t off_dyr, off_xr, off_Cr, off_Br;        // io dtype, reversed in time
    size_t off_Cer, off_Be, slice_io;              // io dtype [slice][b][L][H][pw]
    size_t off_dfin, off_G0;                       // fp32 [b][H][N][P]
    size_t off_dfinT, off_h0T, off_hfT, slice_st;  // fp32 [slice][b][H][P][pw]
    size_t off_y1, off_y2, off_y3, slice_y;        // fp32 scan outputs
    size_t off_tok, off_part;                      // fp32 per-token and per-sequence scalars
    size_t total;
};

BackwardLayout backward_layout(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, int64_t Q,
                               bool io_bf16);

struct BackwardArgs {
    int64_t batch, L, H, P, N, G, Q;
    bool io_bf16, grad_bf16, state_bf16;
    const void *x, *dt_raw, *B, *C, *dy;
    const float *dt_bias, *A, *D;
    const void *init_state, *dfinal;
    void *dx, *ddt_raw, *dB, *dC, *dinit;
    float *ddt_bias, *dA, *dD;
    char* ws;
    BackwardLayout lay;
    unsigned* dev_err;
};

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s);
cudaError_t launch_backward_blocks_cc(const BackwardArgs& a, cudaStream_t s);
// the tensor-core block form: shapes it covers, its CTAs and partial slots per CTA
bool bwd_tc_supports(int64_t H, int64_t P, int64_t N, int64_t G, bool io_bf16);
void bwd_tc_grid(int64_t batch, int64_t L, int64_t H, int64_t G, int64_t* grid, int64_t* smax);
cudaError_t launch_backward_tc(const BackwardArgs& a, cudaStream_t s);
// tokens per block of the CUDA-core block form, and its shared memory per block
int blk_block_size(int P, int N);
size_t blk_smem_bytes(int qb, int P, int N);
// dA, d dt_bias, dD: part [nseg][H][3] summed over its nseg segments in order
cudaError_t launch_backward_params(const float* part, float* dA, float* ddt_bias, float* dD, int64_t nseg, int H,
                                   cudaStream_t s);
// seqlen 0 (or batch 0): zero parameter gradients, d init_state = dfinal
cudaError_t launch_backward_empty(const BackwardArgs& a, cudaStream_t s);
// kernels one ssd_chunk_scan_bwd call launches
int backward_launches(const BackwardLayout& l, bool has_states);

// Mamba-3 prefill (ssd_mamba3.cu): the forward's scan workspace plus the
// rotated operands, angle sums, the diagonal correction and staging buffers.
struct Mamba3Layout {
    PrefillLayout scan;
    size_t off_corr;               // fp32 [b*H][Lpad]
    size_t off_Bt, off_Ct;         // io dtype [b][L][G][N], rotated by -Theta_t (bf16: the hi part;
                                   // fused: [b][L][G][2][N], hi then lo per group)
    size_t off_Btl, off_Ctl;       // bf16 inputs: the lo part of the same (unused when fused)
    size_t off_csum;               // fp64 [b][G][nchunks][N/2] angle sums per chunk
    size_t off_rotL;               // float2 [b][G][N/2] cos, sin of the angle at the last token
    size_t off_y32[3];             // fp32 [b][L][H][P] scan outputs before the combination
    size_t off_fsr;                // state dtype [b][H][N][P] rotated-frame final state (scan 1)
    size_t off_fsr2;               // fp32 [b][H][N][P] the same of the B_lo scan
    size_t total;
    bool fused;                    // bf16 with the head-pair kernel: one scan of the turned hi/lo operands
};

Mamba3Layout mamba3_layout(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, int64_t Q,
                           bool io_bf16, bool tc);

struct Mamba3Args {
    int64_t batch, L, H, P, N, G, Q;
    bool io_bf16, y_bf16, state_bf16, tc;
    const void *x, *dt_raw, *B, *C;
    const float *dt_bias, *A, *D, *lam, *theta;
    const void* init_state;
    void *y, *final_state;
    char* ws;
    Mamba3Layout lay;
    unsigned* dev_err;
};

cudaError_t launch_mamba3(const Mamba3Args& a, cudaStream_t s);
int mamba3_launches(bool tc, bool io_bf16, bool has_lam, bool has_theta, bool has_final, bool fused);

// fault-injection bits set by ssd_debug_inject (read at every launch)
uint32_t debug_faults();

}  // namespace ssd
