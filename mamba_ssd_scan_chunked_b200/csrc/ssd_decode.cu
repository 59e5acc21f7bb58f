// Single-token decode step of the SSD layer core: a streaming, memory-bound
// read-modify-write of the recurrent state.
//
//   dt = softplus(dt_raw + dt_bias); dA = exp(dt * A)
//   h[n,p] <- dA * h[n,p] + (dt * B[n]) * x[p]
//   y[p]    = sum_n C[n] * h[n,p] + D * x[p]        (updated state)
//
// "Mamba3" (Telegram post), first paragraph: with a scalar-times-identity
// transition, decoding spends its time moving the state between memory levels;
// "Mamba-3 : SSM optimise inference", section "Du training-first a
// l'inference-first": token-by-token decoding is almost entirely memory-bound.
// Roughly 0.6 flop per state byte, so the kernel is built for HBM bandwidth:
// no tensor cores, every state byte is read once and written once with 16-byte
// vector accesses, coalesced 512 bytes per warp instruction.
//
// Mapping: one CTA per (batch, head).  Thread t owns the 16-byte column vector
// `vc = t % VPR` of every row it visits (VPR = vectors per state row) and rows
// r = t / VPR + k * (THREADS / VPR).  All of a thread's state loads are issued
// before any is used.  Partial y sums are reduced over rows through shared
// memory.
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

template <typename StateT, typename IoT, typename YT, int THREADS>
__global__ void __launch_bounds__(THREADS, 3)
state_update_kernel(StateT* __restrict__ state, const IoT* __restrict__ x,
                    const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                    const float* __restrict__ A, const IoT* __restrict__ Bm,
                    const IoT* __restrict__ Cm, const float* __restrict__ Dv,
                    YT* __restrict__ y, int H, int P, int N, int heads_per_group) {
    using SV = Vec16<StateT>;
    constexpr int VEC = SV::N;                 // state elements per 16-byte vector
    constexpr int UNROLL = 32 / VEC;           // 32 state values in flight per thread
    extern __shared__ float smem[];            // [THREADS / VPR][P] partial y, then x, B, C

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H, g = h / heads_per_group;
    const int vpr = P / VEC;                   // vectors per row (P multiple of 8)
    const int row_groups = THREADS / vpr;
    const int tid = threadIdx.x;
    const int vc = tid % vpr;
    const int rg = tid / vpr;
    const bool active = rg < row_groups;       // THREADS may not be a multiple of vpr

    float* red = smem;                              // row_groups * P
    float* xs = red + row_groups * P;               // P
    float* bs = xs + P;                             // N
    float* cs = bs + N;                             // N

    // stage x, B, C (fp32) in shared memory
    const IoT* xg = x + (size_t)bh * P;
    const IoT* bg = Bm + ((size_t)b * (H / heads_per_group) + g) * N;
    const IoT* cg = Cm + ((size_t)b * (H / heads_per_group) + g) * N;
    for (int i = tid; i < P; i += THREADS) xs[i] = to_f32(xg[i]);
    for (int i = tid; i < N; i += THREADS) { bs[i] = to_f32(bg[i]); cs[i] = to_f32(cg[i]); }

    const float dt = softplus_f32(to_f32(dt_raw[bh]) + (dt_bias ? dt_bias[h] : 0.f));
    const float dA = expf(dt * A[h]);
    __syncthreads();

    float acc[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] = 0.f;

    if (active) {
        float xv[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) xv[j] = xs[vc * VEC + j];
        StateT* base = state + (size_t)bh * N * P + vc * VEC;
        // rows handled by this thread: rg, rg + row_groups, ... (< N)
        for (int r0 = rg; r0 < N; r0 += UNROLL * row_groups) {
            float hv[UNROLL][VEC];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int r = r0 + u * row_groups;
                if (r < N) SV::load_stream(base + (size_t)r * P, hv[u]);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int r = r0 + u * row_groups;
                if (r < N) {
                    const float coef = dt * bs[r];
                    const float c = cs[r];
#pragma unroll
                    for (int j = 0; j < VEC; ++j) {
                        const float v = fmaf(dA, hv[u][j], coef * xv[j]);
                        hv[u][j] = v;
                        acc[j] = fmaf(c, v, acc[j]);
                    }
                    SV::store_stream(base + (size_t)r * P, hv[u]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < VEC; ++j) red[rg * P + vc * VEC + j] = acc[j];
    }
    __syncthreads();
    const float d_skip = Dv ? Dv[h] : 0.f;
    for (int p = tid; p < P; p += THREADS) {
        float s = 0.f;
        for (int k = 0; k < row_groups; ++k) s += red[k * P + p];
        y[(size_t)bh * P + p] = from_f32<YT>(s + d_skip * xs[p]);
    }
}

template <typename StateT, typename IoT, typename YT>
static cudaError_t launch_t(const DecodeArgs& a, cudaStream_t stream) {
    constexpr int THREADS = 256;
    const int vpr = (int)a.P / Vec16<StateT>::N;
    const int row_groups = THREADS / vpr;
    const size_t smem = sizeof(float) * ((size_t)row_groups * a.P + a.P + 2 * a.N);
    const dim3 grid((unsigned)(a.batch * a.H));
    state_update_kernel<StateT, IoT, YT, THREADS><<<grid, THREADS, smem, stream>>>(
        (StateT*)a.state, (const IoT*)a.x, (const IoT*)a.dt_raw, a.dt_bias, a.A, (const IoT*)a.B,
        (const IoT*)a.C, a.D, (YT*)a.y, (int)a.H, (int)a.P, (int)a.N, (int)(a.H / a.G));
    return cudaGetLastError();
}

template <typename StateT, typename IoT>
static cudaError_t launch_y(const DecodeArgs& a, cudaStream_t s) {
    return a.y_bf16 ? launch_t<StateT, IoT, bf16>(a, s) : launch_t<StateT, IoT, float>(a, s);
}

template <typename StateT>
static cudaError_t launch_io(const DecodeArgs& a, cudaStream_t s) {
    return a.io_bf16 ? launch_y<StateT, bf16>(a, s) : launch_y<StateT, float>(a, s);
}

cudaError_t launch_state_update(const DecodeArgs& a, cudaStream_t stream) {
    if (a.batch == 0) return cudaSuccess;
    return a.state_bf16 ? launch_io<bf16>(a, stream) : launch_io<float>(a, stream);
}

}  // namespace ssd
