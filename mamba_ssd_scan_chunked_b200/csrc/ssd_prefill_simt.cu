// Prefill kernels on CUDA cores, fp32 arithmetic throughout.
//
// The chunked ("blocked two-pass") contraction of the semiseparable matrix
// ("Mamba-2 vs Transformers / SSD", section "Mamba-2 and the SSD paper: what
// changed in practice": chunks processed in parallel, per-chunk states
// recombined), per (batch b, head h), chunk c of Q tokens, l, s in [0, Q):
//
//   dt_cumsum   : dt_s = softplus(dt_raw_s + dt_bias), acs_l = sum_{k<=l} dt_k A
//                 (chunk-local, inclusive), summed in fp64 and stored as an fp32
//                 pair hi + lo.  Shared with the tensor-core path.
//
// Decay factors are exponentials of cumsum differences, exp(acs_l - acs_s).
// With strong decays the cumsum of a chunk reaches magnitudes of 10^4, where
// one fp32 rounding of acs is worth 1e-3 in the exponent; differences are
// therefore formed as (hi_l - hi_s) + (lo_l - lo_s), which is exact in its
// first term whenever the difference is small next to the values (the only
// case where the factor is not negligibly small).
//   chunk_state : S_c[n,p] = sum_s B_s[n] exp(acs_{Q-1} - acs_s) dt_s x_s[p]
//   state_pass  : h_in[0] = init_state, h_in[c+1] = exp(acs_{Q-1}) h_in[c] + S_c
//                 (sequential fp32 scan over chunks); final_state = h_in[nc]
//   chunk_scan  : y_l = sum_{s<=l} (C_l . B_s) exp(acs_l - acs_s) dt_s x_s
//                       + exp(acs_l) C_l^T h_in[c] + D x_l
//
// This is the fp32 path: TF32 tensor cores (about 2^-11 relative rounding of
// every operand) cannot meet a 1e-4 max-error bound, so fp32 inputs run here.
// Tokens past seqlen in the last chunk get dt = 0 and a = 0, so they neither
// feed the state nor decay it; their outputs are not stored.
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

// --------------------------------------------------------------------------
// dt and chunk-local decay cumsum.  One block per (batch b, chunk c, group of
// DT_HG consecutive heads); thread l = token l of the chunk.  A thread reads
// its token's DT_HG heads (contiguous in dt_raw [b][L][H]; independent loads,
// all in flight at once), applies softplus and dt * A, and the block scans the
// DT_HG columns over its tokens at once: warp shuffles, then the warp totals
// through shared memory.  dt and the cumsum go out as coalesced rows of
// [b*H][Lpad] (a warp writes 32 consecutive tokens of one head).
// --------------------------------------------------------------------------
constexpr int DT_HG = 8;         // heads per block

template <typename IoT>
__global__ void __launch_bounds__(256)
dt_cumsum_kernel(const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                 const float* __restrict__ A, float* __restrict__ dt_out,
                 float* __restrict__ acs_out, float* __restrict__ acs_lo_out, int* __restrict__ flags,
                 const int32_t* __restrict__ pad_left,
                 int64_t L, int64_t Lpad, int H, int Q, int nflags, int nchunks, int hgroups) {
    __shared__ double warp_tot[8][DT_HG];      // Q <= 256: at most 8 warps
    const int hg = (int)(blockIdx.x % (unsigned)hgroups);
    const int c = (int)((blockIdx.x / (unsigned)hgroups) % (unsigned)nchunks);
    const int b = (int)(blockIdx.x / ((unsigned)hgroups * (unsigned)nchunks));
    const int h0 = hg * DT_HG;
    // the tensor-core kernel launched after this one may start now: it waits for
    // this grid to complete before it reads anything written here
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int l = threadIdx.x;                 // token within the chunk (blockDim = max(Q, 32))
    const int lane = l & 31, warp = l >> 5;
    const int64_t t = (int64_t)c * Q + l;
    // tokens before pad_left[b] are absent: dt = 0 (no decay, no input)
    const bool live = l < Q && t < L && (!pad_left || t >= (int64_t)pad_left[b]);
    float raw[DT_HG];
#pragma unroll
    for (int k = 0; k < DT_HG; ++k)
        raw[k] = (live && h0 + k < H) ? to_f32(dt_raw[((int64_t)b * L + t) * H + h0 + k]) : 0.f;
    float dt[DT_HG];
    double v[DT_HG];
#pragma unroll
    for (int k = 0; k < DT_HG; ++k) {
        const int h = h0 + k;
        dt[k] = (live && h < H) ? softplus_f32(raw[k] + (dt_bias ? dt_bias[h] : 0.f)) : 0.f;
        v[k] = h < H ? (double)dt[k] * (double)A[h] : 0.0;   // the product of two fp32 values is exact
    }
    // inclusive scan over the tokens in fp64, DT_HG columns at once
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int k = 0; k < DT_HG; ++k) {
            const double u = __shfl_up_sync(0xffffffffu, v[k], o);
            if (lane >= o) v[k] += u;
        }
    }
    if (lane == 31)
#pragma unroll
        for (int k = 0; k < DT_HG; ++k) warp_tot[warp][k] = v[k];
    __syncthreads();
    for (int w = 0; w < warp; ++w)
#pragma unroll
        for (int k = 0; k < DT_HG; ++k) v[k] += warp_tot[w][k];
    if (l < Q) {
#pragma unroll
        for (int k = 0; k < DT_HG; ++k) {
            if (h0 + k >= H) break;
            const int64_t o = ((int64_t)b * H + h0 + k) * Lpad + t;
            dt_out[o] = dt[k];
            const float hi = (float)v[k];
            acs_out[o] = hi;
            if (acs_lo_out) acs_lo_out[o] = (float)(v[k] - (double)hi);
        }
    }
    // reset the run hand-off flags and control words of this launch (a slice per block)
    const int per = (int)((nflags + gridDim.x - 1) / gridDim.x);
    const int f0 = (int)blockIdx.x * per;
    for (int i = f0 + l; i < nflags && i < f0 + per; i += blockDim.x) flags[i] = 0;
}

template <typename IoT>
static cudaError_t launch_dt_t(const PrefillArgs& a, cudaStream_t s) {
    float* dt = (float*)(a.ws + a.lay.off_dt);
    float* acs = (float*)(a.ws + a.lay.off_acs);
    float* acs_lo = a.lay.has_lo ? (float*)(a.ws + a.lay.off_acs_lo) : nullptr;
    int* flags = (int*)(a.ws + a.lay.off_flags);
    const int nflags = (int)(a.batch * a.H + 64);
    const int hgroups = (int)((a.H + DT_HG - 1) / DT_HG);
    const long long blocks = a.lay.nchunks * a.batch * hgroups;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    const unsigned threads = (unsigned)(a.Q < 32 ? 32 : a.Q);   // whole warps for the shuffles
    dt_cumsum_kernel<IoT><<<(unsigned)blocks, threads, 0, s>>>(
        (const IoT*)a.dt_raw, a.dt_bias, a.A, dt, acs, acs_lo, flags, a.pad_left, a.L, a.lay.Lpad, (int)a.H, (int)a.Q,
        nflags,
        (int)a.lay.nchunks, hgroups);
    return cudaGetLastError();
}

cudaError_t launch_dt_cumsum(const PrefillArgs& a, cudaStream_t s) {
    return a.io_bf16 ? launch_dt_t<bf16>(a, s) : launch_dt_t<float>(a, s);
}

// --------------------------------------------------------------------------
// 64x64 register-tiled fp32 product from shared memory, both operands stored
// k-major: acc[i][j] += sum_k At[k][ty*4+i] * Bt[k][tx*4+j], 256 threads.
// --------------------------------------------------------------------------
constexpr int TM = 64, TK = 16, TPAD = 4;

__device__ __forceinline__ void tile_fma(const float (*At)[TM + TPAD], const float (*Bt)[TM + TPAD],
                                         float acc[4][4], int ty, int tx, int kmax) {
    for (int k = 0; k < kmax; ++k) {
        const float4 a4 = *reinterpret_cast<const float4*>(&At[k][ty * 4]);
        const float4 b4 = *reinterpret_cast<const float4*>(&Bt[k][tx * 4]);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
}

// --------------------------------------------------------------------------
// chunk_state.  1-D grid over nchunks x (b*H) x ceil(N/64)*ceil(P/64), block 256.
// states[(bh*nchunks + c)][n][p] (fp32).
// --------------------------------------------------------------------------
template <typename IoT>
__global__ void __launch_bounds__(256)
chunk_state_kernel(const IoT* __restrict__ x, const IoT* __restrict__ Bm, const float* __restrict__ dtw,
                   const float* __restrict__ acsw, const float* __restrict__ acslo, float* __restrict__ states,
                   int64_t L, int64_t Lpad, int H, int P, int N, int G, int Q, int nchunks, int ntiles) {
    __shared__ __align__(16) float At[TK][TM + TPAD];   // [s][n]
    __shared__ __align__(16) float Bt[TK][TM + TPAD];   // [s][p] scaled by w_s
    __shared__ float ws[256];
    const int tile = (int)(blockIdx.x % (unsigned)ntiles);
    const int c = (int)((blockIdx.x / (unsigned)ntiles) % (unsigned)nchunks);
    const int bh = (int)(blockIdx.x / ((unsigned)ntiles * (unsigned)nchunks));
    const int b = bh / H, h = bh % H, g = h / (H / G);
    const int ptiles = (P + TM - 1) / TM;
    const int n0 = (tile / ptiles) * TM, p0 = (tile % ptiles) * TM;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int64_t base_t = (int64_t)c * Q;
    const float* dtc = dtw + (int64_t)bh * Lpad + base_t;
    const float* acc_c = acsw + (int64_t)bh * Lpad + base_t;
    const float* acl_c = acslo ? acslo + (int64_t)bh * Lpad + base_t : nullptr;
    const float a_last = acc_c[Q - 1], a_last_lo = acl_c ? acl_c[Q - 1] : 0.f;
    for (int s = tid; s < Q; s += 256)
        ws[s] = expf((a_last - acc_c[s]) + (a_last_lo - (acl_c ? acl_c[s] : 0.f))) * dtc[s];
    float acc[4][4] = {};
    for (int k0 = 0; k0 < Q; k0 += TK) {
        __syncthreads();
        for (int i = tid; i < TK * TM; i += 256) {
            const int kk = i / TM, m = i % TM;
            const int64_t t = base_t + k0 + kk;
            float bv = 0.f, xv = 0.f;
            if (t < L) {
                if (n0 + m < N) bv = to_f32(Bm[((int64_t)b * L + t) * G * N + (int64_t)g * N + n0 + m]);
                if (p0 + m < P) xv = to_f32(x[(((int64_t)b * L + t) * H + h) * P + p0 + m]) * ws[k0 + kk];
            }
            At[kk][m] = bv;
            Bt[kk][m] = xv;
        }
        __syncthreads();
        tile_fma(At, Bt, acc, ty, tx, TK);
    }
    float* out = states + ((int64_t)bh * nchunks + c) * N * P;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + ty * 4 + i, p = p0 + tx * 4 + j;
            if (n < N && p < P) out[(int64_t)n * P + p] = acc[i][j];
        }
}

// --------------------------------------------------------------------------
// state_pass: sequential fp32 scan over chunks, one thread per 4 state
// elements.  Overwrites states[c] (= S_c) with h_in[c].  grid (b*H, ceil(NP/1024)).
// --------------------------------------------------------------------------
template <typename StateT>
__global__ void __launch_bounds__(256)
state_pass_kernel(float* __restrict__ states, const float* __restrict__ acsw,
                  const StateT* __restrict__ init_state, StateT* __restrict__ final_state,
                  int64_t Lpad, int NP, int Q, int nchunks) {
    const int bh = blockIdx.x;
    const int e = (blockIdx.y * 256 + threadIdx.x) * 4;
    if (e >= NP) return;
    float h[4] = {0.f, 0.f, 0.f, 0.f};
    if (init_state) {
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j] = to_f32(init_state[(int64_t)bh * NP + e + j]);
    }
    const float* acs = acsw + (int64_t)bh * Lpad;
    float* st = states + (int64_t)bh * nchunks * NP + e;
    for (int c = 0; c < nchunks; ++c) {
        const float decay = expf(acs[(int64_t)c * Q + Q - 1]);
        float4 sc = *reinterpret_cast<float4*>(st + (int64_t)c * NP);
        *reinterpret_cast<float4*>(st + (int64_t)c * NP) = make_float4(h[0], h[1], h[2], h[3]);
        h[0] = fmaf(decay, h[0], sc.x);
        h[1] = fmaf(decay, h[1], sc.y);
        h[2] = fmaf(decay, h[2], sc.z);
        h[3] = fmaf(decay, h[3], sc.w);
    }
    if (final_state) {
#pragma unroll
        for (int j = 0; j < 4; ++j) final_state[(int64_t)bh * NP + e + j] = from_f32<StateT>(h[j]);
    }
}

// --------------------------------------------------------------------------
// chunk_scan.  1-D grid over nchunks*ceil(Q/64) x (b*H) x ceil(P/64), block 256.
// --------------------------------------------------------------------------
template <typename IoT, typename YT>
__global__ void __launch_bounds__(256)
chunk_scan_kernel(const IoT* __restrict__ x, const IoT* __restrict__ Bm, const IoT* __restrict__ Cm,
                  const float* __restrict__ Dv, const float* __restrict__ dtw,
                  const float* __restrict__ acsw, const float* __restrict__ acslo,
                  const float* __restrict__ states, YT* __restrict__ y, int64_t L, int64_t Lpad, int H, int P,
                  int N, int G, int Q, int nchunks, int ptiles) {
    __shared__ __align__(16) float At[TK][TM + TPAD];
    __shared__ __align__(16) float Bt[TK][TM + TPAD];
    __shared__ __align__(16) float Mt[TM][TM + TPAD];   // [s][l] masked decay matrix
    __shared__ __align__(16) float Xs[TM][TM + TPAD];   // [s][p]
    __shared__ float acs_l[TM], acs_s[TM], dt_s[TM], lo_l[TM], lo_s[TM];
    const int rtiles = (Q + TM - 1) / TM;
    const unsigned crt = (unsigned)(nchunks * rtiles);
    const int cr = (int)((blockIdx.x / (unsigned)ptiles) % crt);
    const int c = cr / rtiles, rt = cr % rtiles;
    const int bh = (int)(blockIdx.x / ((unsigned)ptiles * crt)), b = bh / H, h = bh % H, g = h / (H / G);
    const int p0 = (int)(blockIdx.x % (unsigned)ptiles) * TM;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int l0 = rt * TM;                       // chunk-local first row of the tile
    const int64_t base_t = (int64_t)c * Q;
    const float* acs = acsw + (int64_t)bh * Lpad + base_t;
    const float* acl = acslo ? acslo + (int64_t)bh * Lpad + base_t : nullptr;
    const float* dtc = dtw + (int64_t)bh * Lpad + base_t;
    const float* hin = states + ((int64_t)bh * nchunks + c) * N * P;
    const int rows = min(TM, Q - l0);
    if (tid < TM) {
        acs_l[tid] = tid < rows ? acs[l0 + tid] : 0.f;
        lo_l[tid] = tid < rows && acl ? acl[l0 + tid] : 0.f;
    }

    // off-diagonal term: acc = C_l^T h_in
    float acc[4][4] = {};
    for (int k0 = 0; k0 < N; k0 += TK) {
        __syncthreads();
        for (int i = tid; i < TK * TM; i += 256) {
            const int kk = i / TM, m = i % TM;
            const int64_t t = base_t + l0 + m;
            const int n = k0 + kk;
            At[kk][m] = (m < rows && t < L && n < N)
                            ? to_f32(Cm[((int64_t)b * L + t) * G * N + (int64_t)g * N + n]) : 0.f;
            Bt[kk][m] = (n < N && p0 + m < P) ? hin[(int64_t)n * P + p0 + m] : 0.f;
        }
        __syncthreads();
        tile_fma(At, Bt, acc, ty, tx, TK);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float e = expf(acs_l[ty * 4 + i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] *= e;
    }

    // intra-chunk term over column blocks s0 <= l0
    for (int s0 = 0; s0 <= l0; s0 += TM) {
        const int cols = min(TM, Q - s0);
        __syncthreads();
        if (tid < TM) {
            acs_s[tid] = tid < cols ? acs[s0 + tid] : 0.f;
            lo_s[tid] = tid < cols && acl ? acl[s0 + tid] : 0.f;
            dt_s[tid] = tid < cols ? dtc[s0 + tid] : 0.f;
        }
        float sc[4][4] = {};
        for (int k0 = 0; k0 < N; k0 += TK) {
            __syncthreads();
            for (int i = tid; i < TK * TM; i += 256) {
                const int kk = i / TM, m = i % TM;
                const int n = k0 + kk;
                const int64_t tl = base_t + l0 + m, ts = base_t + s0 + m;
                At[kk][m] = (m < rows && tl < L && n < N)
                                ? to_f32(Cm[((int64_t)b * L + tl) * G * N + (int64_t)g * N + n]) : 0.f;
                Bt[kk][m] = (m < cols && ts < L && n < N)
                                ? to_f32(Bm[((int64_t)b * L + ts) * G * N + (int64_t)g * N + n]) : 0.f;
            }
            __syncthreads();
            tile_fma(At, Bt, sc, ty, tx, TK);
        }
        // masked decay: M[l][s] = sc * exp(acs_l - acs_s) * dt_s for s <= l
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int li = ty * 4 + i, sj = tx * 4 + j;
                const bool keep = (s0 + sj) <= (l0 + li) && sj < cols && li < rows;
                Mt[sj][li] = keep ? sc[i][j] * expf((acs_l[li] - acs_s[sj]) + (lo_l[li] - lo_s[sj])) * dt_s[sj]
                                  : 0.f;
            }
        for (int i = tid; i < TM * TM; i += 256) {
            const int sj = i / TM, pp = i % TM;
            const int64_t ts = base_t + s0 + sj;
            Xs[sj][pp] = (sj < cols && ts < L && p0 + pp < P)
                             ? to_f32(x[(((int64_t)b * L + ts) * H + h) * P + p0 + pp]) : 0.f;
        }
        __syncthreads();
        tile_fma(Mt, Xs, acc, ty, tx, TM);
    }

    const float d_skip = Dv ? Dv[h] : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int li = ty * 4 + i;
        const int64_t t = base_t + l0 + li;
        if (li >= rows || t >= L) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = p0 + tx * 4 + j;
            if (p >= P) continue;
            const int64_t o = (((int64_t)b * L + t) * H + h) * P + p;
            y[o] = from_f32<YT>(acc[i][j] + d_skip * to_f32(x[o]));
        }
    }
}

template <typename IoT, typename YT, typename StateT>
static cudaError_t launch_simt_t(const PrefillArgs& a, cudaStream_t s) {
    const float* dt = (const float*)(a.ws + a.lay.off_dt);
    const float* acs = (const float*)(a.ws + a.lay.off_acs);
    const float* acslo = a.lay.has_lo ? (const float*)(a.ws + a.lay.off_acs_lo) : nullptr;
    float* states = (float*)(a.ws + a.lay.off_states);
    const int nc = (int)a.lay.nchunks;
    const int H = (int)a.H, P = (int)a.P, N = (int)a.N, G = (int)a.G, Q = (int)a.Q;
    const unsigned BH = (unsigned)(a.batch * a.H);
    const unsigned tiles_np = (unsigned)(((N + TM - 1) / TM) * ((P + TM - 1) / TM));
    chunk_state_kernel<IoT><<<(unsigned)(nc * BH * tiles_np), 256, 0, s>>>(
        (const IoT*)a.x, (const IoT*)a.B, dt, acs, acslo, states, a.L, a.lay.Lpad, H, P, N, G, Q, nc, (int)tiles_np);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int NP = N * P;
    state_pass_kernel<StateT><<<dim3(BH, (unsigned)((NP / 4 + 255) / 256)), 256, 0, s>>>(
        states, acs, (const StateT*)a.init_state, (StateT*)a.final_state, a.lay.Lpad, NP, Q, nc);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const unsigned rtiles = (unsigned)((Q + TM - 1) / TM);
    const unsigned ptiles = (unsigned)((P + TM - 1) / TM);
    chunk_scan_kernel<IoT, YT><<<nc * rtiles * BH * ptiles, 256, 0, s>>>(
        (const IoT*)a.x, (const IoT*)a.B, (const IoT*)a.C, a.D, dt, acs, acslo, states, (YT*)a.y, a.L,
        a.lay.Lpad, H, P, N, G, Q, nc, (int)ptiles);
    return cudaGetLastError();
}

template <typename IoT, typename YT>
static cudaError_t launch_simt_s(const PrefillArgs& a, cudaStream_t s) {
    return a.state_bf16 ? launch_simt_t<IoT, YT, bf16>(a, s) : launch_simt_t<IoT, YT, float>(a, s);
}

template <typename IoT>
static cudaError_t launch_simt_y(const PrefillArgs& a, cudaStream_t s) {
    return a.y_bf16 ? launch_simt_s<IoT, bf16>(a, s) : launch_simt_s<IoT, float>(a, s);
}

cudaError_t launch_prefill_simt(const PrefillArgs& a, cudaStream_t s) {
    return a.io_bf16 ? launch_simt_y<bf16>(a, s) : launch_simt_y<float>(a, s);
}

}  // namespace ssd
