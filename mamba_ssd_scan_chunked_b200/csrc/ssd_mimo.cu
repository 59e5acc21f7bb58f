// MIMO decode step of the SSD layer core: B and C widened to rank R, so the
// rank-1 outer product of the decode step becomes a small matrix product while
// the state keeps its N x P size ("Mamba3" (Telegram post), section on the
// switch from SISO to MIMO; "Mamba-3 : SSM optimise inference", section "Mode
// MIMO": several SSMs in parallel with extended B and C, more arithmetic for
// the same memory traffic in decoding).  Per (batch, head), X = [x_0..x_{R-1}]:
//
//   h <- exp(dt A) h + dt sum_r B_r x_r^T;   y_r = C_r^T h + D x_r
//
// Mapping: one warp per (batch, head).  A lane owns a 4-element column vector
// of the state (16 bytes fp32, 8 bytes bf16) and keeps x_r of its columns for
// all R in registers; dt B_r[n] and C_r[n] are staged per warp in shared
// memory (a row of R floats per n, read as 16-byte vectors for R >= 4); the
// state moves once each way.
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

constexpr int MM_WARPS = 4;

// 4 consecutive elements of T as fp32 (one 16-byte fp32 / 8-byte bf16 access)
template <typename T> struct Quad;
template <> struct Quad<float> {
    __device__ __forceinline__ static void load(const float* p, float* o) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
    __device__ __forceinline__ static void load_stream(const float* p, float* o) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
    __device__ __forceinline__ static void store_stream(float* p, const float* i) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(i[0], i[1], i[2], i[3]));
    }
};
template <> struct Quad<bf16> {
    __device__ __forceinline__ static void unpack(uint2 v, float* o) {
        o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xffff0000u);
        o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xffff0000u);
    }
    __device__ __forceinline__ static uint2 pack(const float* i) {
        __nv_bfloat162 a = __floats2bfloat162_rn(i[0], i[1]), b = __floats2bfloat162_rn(i[2], i[3]);
        return make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
    }
    __device__ __forceinline__ static void load(const bf16* p, float* o) {
        unpack(*reinterpret_cast<const uint2*>(p), o);
    }
    __device__ __forceinline__ static void load_stream(const bf16* p, float* o) {
        unpack(__ldcs(reinterpret_cast<const uint2*>(p)), o);
    }
    __device__ __forceinline__ static void store_stream(bf16* p, const float* i) {
        __stcs(reinterpret_cast<uint2*>(p), pack(i));
    }
};

template <typename StateT, typename IoT, typename YT, int R>
__global__ void __launch_bounds__(MM_WARPS * 32)
mimo_step_kernel(StateT* __restrict__ state, const IoT* __restrict__ x, const IoT* __restrict__ dt_raw,
                 const float* __restrict__ dt_bias, const float* __restrict__ A, const IoT* __restrict__ Bm,
                 const IoT* __restrict__ Cm, const float* __restrict__ Dv, YT* __restrict__ y, int BH, int H,
                 int P, int N, int G) {
    // smem row stride: R for R >= 4 (rows read as 16-byte vectors), else R + 1
    constexpr int S = R >= 4 ? R : R + 1;
    constexpr int U = R <= 2 ? 16 : (R == 4 ? 8 : 4);   // state vectors in flight per lane
    extern __shared__ float mm_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x * MM_WARPS + warp;
    if (bh >= BH) return;                      // whole warps; no block barrier follows
    float* gt = mm_smem + (size_t)warp * 2 * S * N;   // dt B_r[n] at [n][r]
    float* ct = gt + S * N;                           // C_r[n] at [n][r]
    const int b = bh / H, h = bh % H, g = h / (H / G);
    const size_t bg = (size_t)b * G + g;
    const float dt = softplus_f32(to_f32(dt_raw[bh]) + (dt_bias ? dt_bias[h] : 0.f));
    const float alpha = expf(dt * A[h]);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const IoT* br = Bm + (bg * R + r) * N;
        const IoT* cr = Cm + (bg * R + r) * N;
        for (int n = lane; n < N; n += 32) {
            gt[n * S + r] = dt * to_f32(br[n]);
            ct[n * S + r] = to_f32(cr[n]);
        }
    }
    __syncwarp();

    const int vpr = P / 4;                     // vectors per state row; divides 32
    const int rstep = 32 / vpr;
    const int vc = lane % vpr, r_off = lane / vpr;
    const int p0 = vc * 4;
    float xs[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) Quad<IoT>::load(x + ((size_t)bh * R + r) * P + p0, xs[r]);
    float acc[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[r][j] = 0.f;
    StateT* base = state + (size_t)bh * N * P + p0;
    for (int r0 = r_off; r0 < N; r0 += U * rstep) {
        float hv[U][4];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int n = r0 + u * rstep;
            if (n < N) Quad<StateT>::load_stream(base + (size_t)n * P, hv[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int n = r0 + u * rstep;
            if (n < N) {
                float v[4], gr[R], cr[R];
                if (R >= 4) {
#pragma unroll
                    for (int q = 0; q < R / 4; ++q) {
                        const float4 g4 = reinterpret_cast<const float4*>(gt + n * S)[q];
                        const float4 c4 = reinterpret_cast<const float4*>(ct + n * S)[q];
                        gr[4 * q] = g4.x; gr[4 * q + 1] = g4.y; gr[4 * q + 2] = g4.z; gr[4 * q + 3] = g4.w;
                        cr[4 * q] = c4.x; cr[4 * q + 1] = c4.y; cr[4 * q + 2] = c4.z; cr[4 * q + 3] = c4.w;
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        gr[r] = gt[n * S + r];
                        cr[r] = ct[n * S + r];
                    }
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) v[j] = alpha * hv[u][j];
#pragma unroll
                for (int r = 0; r < R; ++r) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) v[j] = fmaf(gr[r], xs[r][j], v[j]);
                }
                Quad<StateT>::store_stream(base + (size_t)n * P, v);   // bf16: rounded to nearest even
#pragma unroll
                for (int r = 0; r < R; ++r) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[r][j] = fmaf(cr[r], v[j], acc[r][j]);
                }
            }
        }
    }
    // reduce over the lanes that share column vector vc (lane = vc + k * vpr)
    for (int o = vpr; o < 32; o <<= 1) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[r][j] += __shfl_xor_sync(0xffffffffu, acc[r][j], o);
    }
    if (r_off == 0) {
        const float d_skip = Dv ? Dv[h] : 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            YT* yr = y + ((size_t)bh * R + r) * P + p0;
#pragma unroll
            for (int j = 0; j < 4; ++j) yr[j] = from_f32<YT>(acc[r][j] + d_skip * xs[r][j]);
        }
    }
}

template <typename StateT, typename IoT, typename YT, int R>
static cudaError_t launch_mm(const MimoArgs& a, cudaStream_t s) {
    const long long bh = a.batch * a.H;
    const unsigned grid = (unsigned)((bh + MM_WARPS - 1) / MM_WARPS);
    const size_t smem = sizeof(float) * MM_WARPS * 2 * (R >= 4 ? R : R + 1) * (size_t)a.N;
    auto k = mimo_step_kernel<StateT, IoT, YT, R>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k<<<grid, MM_WARPS * 32, smem, s>>>((StateT*)a.state, (const IoT*)a.x, (const IoT*)a.dt_raw, a.dt_bias, a.A,
                                        (const IoT*)a.B, (const IoT*)a.C, a.D, (YT*)a.y, (int)bh, (int)a.H,
                                        (int)a.P, (int)a.N, (int)a.G);
    return cudaGetLastError();
}

template <typename StateT, typename IoT, typename YT>
static cudaError_t launch_mm_r(const MimoArgs& a, cudaStream_t s) {
    switch (a.R) {
        case 1: return launch_mm<StateT, IoT, YT, 1>(a, s);
        case 2: return launch_mm<StateT, IoT, YT, 2>(a, s);
        case 4: return launch_mm<StateT, IoT, YT, 4>(a, s);
        default: return launch_mm<StateT, IoT, YT, 8>(a, s);
    }
}

template <typename StateT, typename IoT>
static cudaError_t launch_mm_y(const MimoArgs& a, cudaStream_t s) {
    return a.y_bf16 ? launch_mm_r<StateT, IoT, bf16>(a, s) : launch_mm_r<StateT, IoT, float>(a, s);
}

template <typename StateT>
static cudaError_t launch_mm_io(const MimoArgs& a, cudaStream_t s) {
    return a.io_bf16 ? launch_mm_y<StateT, bf16>(a, s) : launch_mm_y<StateT, float>(a, s);
}

cudaError_t launch_mimo_step(const MimoArgs& a, cudaStream_t s) {
    if (a.batch == 0) return cudaSuccess;
    return a.state_bf16 ? launch_mm_io<bf16>(a, s) : launch_mm_io<float>(a, s);
}

}  // namespace ssd
