// Single-token decode step of the Mamba-3 recurrence: exponential-trapezoidal
// input and rotational (complex-valued) state, as a streaming, memory-bound
// read-modify-write of the state.
//
//   dt = softplus(dt_raw + dt_bias);  a = exp(dt A);  lam in [0, 1]
//   h  <- h + (1 - lam) dt B_prev x_prev^T          the interval's left end
//   h  <- a R(theta) h                              pairs (2k, 2k+1) turned by theta_k
//   h  <- h + lam dt B x^T                          its right end
//   y   = C^T h + D x
//
// "Mamba3" (Telegram post), section "New discretisation scheme": the input is
// taken at both ends of the step, mixed by a learned weight; section on the
// complex-valued SSM and "Mamba-3 : SSM optimise inference", section "Etats
// complexes via RoPE": the state's pairs turn by data-dependent angles.  The
// decode state is the SSM state plus the previous token's B and x ("Mamba3",
// the same section: the trapezoid reaches back one step); here the caller passes
// those as inputs -- they are the previous call's B and x -- so nothing but the
// state is written in place.
//
// Per element that is a few fused multiply-adds on top of the plain decode step,
// still far below one flop per byte: the kernel keeps the shape of the plain
// step's warp kernel (one warp per (batch, head), 16-byte state vectors streamed
// in and out once), with each lane owning both rows of the pairs it visits so
// that the rotation needs no data from other lanes.
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

template <typename StateT, typename IoT, typename YT, int WARPS, int UP>
__global__ void __launch_bounds__(WARPS * 32)
mamba3_step_kernel(StateT* __restrict__ state, const IoT* __restrict__ x, const IoT* __restrict__ x_prev,
                   const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias, const float* __restrict__ A,
                   const IoT* __restrict__ Bm, const IoT* __restrict__ B_prev, const IoT* __restrict__ Cm,
                   const float* __restrict__ Dv, const float* __restrict__ lam, const float* __restrict__ theta,
                   YT* __restrict__ y, int BH, int H, int P, int N, int heads_per_group) {
    using SV = Vec16<StateT>;
    constexpr int VEC = SV::N;                 // state elements per 16-byte vector
    // per warp, fp32: right-end coefficient lam dt B[n], left-end (1 - lam) dt B_prev[n],
    // C[n], then per pair a cos(theta_k), a sin(theta_k)
    extern __shared__ float smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x * WARPS + warp;
    if (bh >= BH) return;                      // whole warps only; no block barrier follows
    const int b = bh / H, h = bh % H, g = h / heads_per_group, G = H / heads_per_group;
    const int vpr = P / VEC;                   // vectors per row; divides 32 on this path
    const int pstep = 32 / vpr;                // pairs covered by one warp instruction
    const int vc = lane % vpr, p_off = lane / vpr;
    const int npairs = N / 2;
    uint4* base = reinterpret_cast<uint4*>(state + (size_t)bh * N * P) + vc;   // row stride vpr

    // the first batch of state loads goes out before the per-token terms are fetched
    uint4 raw[UP][2];
#pragma unroll
    for (int u = 0; u < UP; ++u) {
        const int k = p_off + u * pstep;
        if (k < npairs) {
            raw[u][0] = __ldcs(base + (size_t)(2 * k) * vpr);
            raw[u][1] = __ldcs(base + (size_t)(2 * k + 1) * vpr);
        }
    }

    float* br = smem + warp * (4 * N);         // lam dt B
    float* bl = br + N;                        // (1 - lam) dt B_prev
    float* cs = bl + N;                        // C
    float* rot = cs + N;                       // [npairs][2]: a cos, a sin
    const float dt = softplus_f32(to_f32(dt_raw[bh]) + (dt_bias ? dt_bias[h] : 0.f));
    const float mix = lam ? lam[bh] : 1.f;
    const float decay = expf(dt * A[h]);
    const size_t bg = ((size_t)b * G + g) * N;
    for (int i = lane; i < N; i += 32) {
        br[i] = mix * dt * to_f32(Bm[bg + i]);
        bl[i] = B_prev ? (1.f - mix) * dt * to_f32(B_prev[bg + i]) : 0.f;
        cs[i] = to_f32(Cm[bg + i]);
    }
    for (int k = lane; k < npairs; k += 32) {
        float sn = 0.f, cn = 1.f;
        if (theta) sincosf(theta[((size_t)b * G + g) * npairs + k], &sn, &cn);
        rot[2 * k] = decay * cn;
        rot[2 * k + 1] = decay * sn;
    }
    float xv[VEC], xp[VEC];
    {
        const IoT* xg = x + (size_t)bh * P + vc * VEC;
#pragma unroll
        for (int j = 0; j < VEC; ++j) xv[j] = to_f32(xg[j]);
        if (x_prev) {
            const IoT* xq = x_prev + (size_t)bh * P + vc * VEC;
#pragma unroll
            for (int j = 0; j < VEC; ++j) xp[j] = to_f32(xq[j]);
        } else {
#pragma unroll
            for (int j = 0; j < VEC; ++j) xp[j] = 0.f;
        }
    }
    __syncwarp();

    float acc[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
    for (int k0 = p_off; k0 < npairs; k0 += UP * pstep) {
        if (k0 != p_off) {
#pragma unroll
            for (int u = 0; u < UP; ++u) {
                const int k = k0 + u * pstep;
                if (k < npairs) {
                    raw[u][0] = __ldcs(base + (size_t)(2 * k) * vpr);
                    raw[u][1] = __ldcs(base + (size_t)(2 * k + 1) * vpr);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UP; ++u) {
            const int k = k0 + u * pstep;
            if (k < npairs) {
                const int n0 = 2 * k, n1 = n0 + 1;
                float hu[VEC], hv[VEC];
                SV::unpack(raw[u][0], hu);
                SV::unpack(raw[u][1], hv);
                const float l0 = bl[n0], l1 = bl[n1], r0 = br[n0], r1 = br[n1];
                const float ac = rot[2 * k], as = rot[2 * k + 1], c0 = cs[n0], c1 = cs[n1];
#pragma unroll
                for (int j = 0; j < VEC; ++j) {
                    const float uu = fmaf(l0, xp[j], hu[j]);        // + left end
                    const float vv = fmaf(l1, xp[j], hv[j]);
                    const float nu = fmaf(ac, uu, fmaf(-as, vv, r0 * xv[j]));   // turn, decay, + right end
                    const float nv = fmaf(as, uu, fmaf(ac, vv, r1 * xv[j]));
                    hu[j] = nu;
                    hv[j] = nv;
                    acc[j] = fmaf(c0, nu, fmaf(c1, nv, acc[j]));
                }
                __stcs(base + (size_t)n0 * vpr, SV::pack(hu));
                __stcs(base + (size_t)n1 * vpr, SV::pack(hv));
            }
        }
    }
    // reduce over the lanes that share column vector vc (lane = vc + k * vpr)
    for (int o = vpr; o < 32; o <<= 1) {
#pragma unroll
        for (int j = 0; j < VEC; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
    if (p_off == 0) {
        const float d_skip = Dv ? Dv[h] : 0.f;
        YT* yg = y + (size_t)bh * P + vc * VEC;
#pragma unroll
        for (int j = 0; j < VEC; ++j) yg[j] = from_f32<YT>(fmaf(d_skip, xv[j], acc[j]));
    }
}

bool mamba3_step_supports(int64_t P, int64_t N, bool state_bf16) {
    const int64_t vec = state_bf16 ? 8 : 4;
    return N % 2 == 0 && P % vec == 0 && 32 % (P / vec) == 0;
}

template <typename StateT, typename IoT, typename YT>
static cudaError_t launch_m3(const Mamba3StepArgs& a, cudaStream_t stream) {
    // 8 state vectors in flight per lane (4 pairs) for fp32 states, 4 pairs of bf16 vectors
    constexpr int WARPS = 4, UP = 4;
    const long long bh = a.batch * a.H;
    const size_t smem = sizeof(float) * WARPS * 4 * (size_t)a.N;
    const dim3 grid((unsigned)((bh + WARPS - 1) / WARPS));
    mamba3_step_kernel<StateT, IoT, YT, WARPS, UP><<<grid, WARPS * 32, smem, stream>>>(
        (StateT*)a.state, (const IoT*)a.x, (const IoT*)a.x_prev, (const IoT*)a.dt_raw, a.dt_bias, a.A,
        (const IoT*)a.B, (const IoT*)a.B_prev, (const IoT*)a.C, a.D, a.lam, a.theta, (YT*)a.y, (int)bh,
        (int)a.H, (int)a.P, (int)a.N, (int)(a.H / a.G));
    return cudaGetLastError();
}

template <typename StateT, typename IoT>
static cudaError_t launch_m3_y(const Mamba3StepArgs& a, cudaStream_t s) {
    return a.y_bf16 ? launch_m3<StateT, IoT, bf16>(a, s) : launch_m3<StateT, IoT, float>(a, s);
}

template <typename StateT>
static cudaError_t launch_m3_io(const Mamba3StepArgs& a, cudaStream_t s) {
    return a.io_bf16 ? launch_m3_y<StateT, bf16>(a, s) : launch_m3_y<StateT, float>(a, s);
}

cudaError_t launch_mamba3_step(const Mamba3StepArgs& a, cudaStream_t stream) {
    if (a.batch == 0) return cudaSuccess;
    if (!mamba3_step_supports(a.P, a.N, a.state_bf16)) return cudaErrorNotSupported;
    return a.state_bf16 ? launch_m3_io<bf16>(a, stream) : launch_m3_io<float>(a, stream);
}

}  // namespace ssd
