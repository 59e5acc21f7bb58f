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
// Mapping: one warp per (batch, head) when a state row is a power-of-two number
// of 16-byte vectors that divides 32 (headdim 8..128 for fp32 states, 8..256 for
// bf16), else one 256-thread CTA per (batch, head).  Either way a thread owns one
// 16-byte column vector of the rows it visits and issues all of a batch of state
// loads before using any.
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

// Warp-per-head variant: one warp streams one (batch, head) state.  Lane l
// owns the 16-byte column vector l % VPR of rows l / VPR + k * (32 / VPR).  A
// lane keeps U raw 16-byte state vectors in flight and widens each to fp32 only
// when it is used, so the registers held across the loads are 4 per vector
// whatever the state type.  The first batch of state loads is issued before
// dt, B, C and x are fetched, so their latency overlaps.  B and C of the head's
// group go to warp-private shared memory; the y partial sums of the lanes that
// share a column vector are reduced with shuffles, so the warps of a CTA never
// synchronise with each other.
template <typename StateT, typename IoT, typename YT, int WARPS, int U>
__global__ void __launch_bounds__(WARPS * 32)
state_update_warp_kernel(StateT* __restrict__ state, const IoT* __restrict__ x,
                         const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                         const float* __restrict__ A, const IoT* __restrict__ Bm,
                         const IoT* __restrict__ Cm, const float* __restrict__ Dv,
                         YT* __restrict__ y, int BH, int H, int P, int N, int heads_per_group) {
    using SV = Vec16<StateT>;
    constexpr int VEC = SV::N;                 // state elements per 16-byte vector
    extern __shared__ float smem[];            // per warp: dt * B[N], C[N]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x * WARPS + warp;
    if (bh >= BH) return;                      // whole warps only; no block barrier follows
    const int b = bh / H, h = bh % H, g = h / heads_per_group;
    const int vpr = P / VEC;                   // vectors per row; divides 32 on this path
    const int rstep = 32 / vpr;                // rows covered by one warp instruction
    const int vc = lane % vpr, r_off = lane / vpr;
    uint4* base = reinterpret_cast<uint4*>(state + (size_t)bh * N * P) + vc;   // row stride vpr

    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int r = r_off + u * rstep;
        if (r < N) raw[u] = __ldcs(base + (size_t)r * vpr);
    }

    float* bs = smem + warp * 2 * N;
    float* cs = bs + N;
    const IoT* bg = Bm + ((size_t)b * (H / heads_per_group) + g) * N;
    const IoT* cg = Cm + ((size_t)b * (H / heads_per_group) + g) * N;
    const float dt = softplus_f32(to_f32(dt_raw[bh]) + (dt_bias ? dt_bias[h] : 0.f));
    for (int i = lane; i < N; i += 32) {
        bs[i] = dt * to_f32(bg[i]);
        cs[i] = to_f32(cg[i]);
    }
    const float dA = expf(dt * A[h]);
    float xv[VEC];
    {
        const IoT* xg = x + (size_t)bh * P + vc * VEC;
#pragma unroll
        for (int j = 0; j < VEC; ++j) xv[j] = to_f32(xg[j]);
    }
    __syncwarp();
    float acc[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
    for (int r0 = r_off; r0 < N; r0 += U * rstep) {
        if (r0 != r_off) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u * rstep;
                if (r < N) raw[u] = __ldcs(base + (size_t)r * vpr);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int r = r0 + u * rstep;
            if (r < N) {
                float hv[VEC];
                SV::unpack(raw[u], hv);
                const float coef = bs[r], c = cs[r];
#pragma unroll
                for (int j = 0; j < VEC; ++j) {
                    const float v = fmaf(dA, hv[j], coef * xv[j]);
                    hv[j] = v;
                    acc[j] = fmaf(c, v, acc[j]);
                }
                __stcs(base + (size_t)r * vpr, SV::pack(hv));
            }
        }
    }
    // reduce over the lanes that share column vector vc (lane = vc + k * vpr)
    for (int o = vpr; o < 32; o <<= 1) {
#pragma unroll
        for (int j = 0; j < VEC; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
    if (r_off == 0) {
        const float d_skip = Dv ? Dv[h] : 0.f;
        YT* yg = y + (size_t)bh * P + vc * VEC;
#pragma unroll
        for (int j = 0; j < VEC; ++j) yg[j] = from_f32<YT>(acc[j] + d_skip * xv[j]);
    }
}

template <typename StateT, typename IoT, typename YT>
static cudaError_t launch_t(const DecodeArgs& a, cudaStream_t stream) {
    constexpr int VEC = Vec16<StateT>::N;
    if (32 % (a.P / VEC) == 0) {
        // warp per head (P / VEC divides 32: P <= 128 for fp32, <= 256 for bf16)
        // 16-byte state vectors in flight per lane: 16 for fp32 (96 registers), 8 for
        // bf16, where 16 cost registers (128) and so warps on short states (N = 64)
        constexpr int WARPS = 4, U = sizeof(StateT) == 4 ? 16 : 8;
        const long long bh = a.batch * a.H;
        const size_t smem = sizeof(float) * WARPS * 2 * (size_t)a.N;
        const dim3 grid((unsigned)((bh + WARPS - 1) / WARPS));
        state_update_warp_kernel<StateT, IoT, YT, WARPS, U><<<grid, WARPS * 32, smem, stream>>>(
            (StateT*)a.state, (const IoT*)a.x, (const IoT*)a.dt_raw, a.dt_bias, a.A, (const IoT*)a.B,
            (const IoT*)a.C, a.D, (YT*)a.y, (int)bh, (int)a.H, (int)a.P, (int)a.N, (int)(a.H / a.G));
        return cudaGetLastError();
    }
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
