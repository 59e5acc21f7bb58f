// Replayed decode of the SSD layer core: the recurrent state of a sequence is
// a checkpoint h_c (the state after token c) plus a buffer of the tokens that
// came after it, and most steps compute their output from the two without
// writing any state back ("Mamba3" (Telegram post), ReplaySSM paragraph, and
// "Mamba-3 : SSM optimise inference", ReplaySSM: the state is a checkpoint
// plus a buffer of recent inputs; outputs are computed directly on most steps
// and the checkpoint is written only when the buffer fills).
//
// With cum_s = sum_{u=c+1..s} dt_u A (the log decay since the checkpoint) and
// the step's own token t = c + fill + 1,
//
//   h_t = exp(cum_t) h_c + sum_{s=c+1..t} exp(cum_t - cum_s) dt_s B_s x_s^T
//   y_t = C_t^T h_t + D x_t
//       = exp(cum_t) (C_t^T h_c) + sum_s exp(cum_t - cum_s) dt_s (C_t . B_s) x_s + D x_t
//
// An ordinary step reads h_c once (no write) and appends token t to the
// buffer; the step that fills the buffer folds all of it into the checkpoint
// (a rank-K update, one read-modify-write of the state) and computes y_t from
// the new state.  Averaged over K steps the state moves (1 + 1/K) times per
// step instead of twice.  Capacity 1 is the plain decode step.
//
// Mapping: one warp per (batch, head), as the decode kernel.  A lane owns a
// 4-element column vector of the state (16 bytes fp32, 8 bytes bf16) so that
// the fold can keep x_s of all K buffered tokens for its columns in registers
// (paired fp32 FMAs: two columns per instruction).  The dot products C_t . B_s
// of an ordinary step are per (batch, group) and come from a small kernel run
// before it.  The fold's coefficients beta_s B_s[n] are staged per warp in
// shared memory, rows of 17 floats (conflict-free writes and reads).
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

constexpr int RP_WARPS = 4;
constexpr int RP_VEC = 4;
// read-only pass: 8 checkpoint vectors in flight per lane and registers capped
// for 8 resident CTAs (32 warps per SM); measured best of 4/8/16 x 1/5/8
constexpr int RP_U = 8;
constexpr int RP_MINB = 8;
constexpr int RP_MINB_FOLD = 4;             // the fold: 4 resident CTAs (measured 1..4)
constexpr int RP_GS = 16;                   // floats per row of the fold's coefficient table

// 4 consecutive elements of T, converted to and from fp32 (16 B fp32, 8 B bf16)
template <typename T> struct Vec4;
template <> struct Vec4<float> {
    __device__ __forceinline__ static void load(const float* p, float* o) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    }
    __device__ __forceinline__ static void store(float* p, const float* i) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(i[0], i[1], i[2], i[3]));
    }
};
template <> struct Vec4<bf16> {
    __device__ __forceinline__ static void load(const bf16* p, float* o) {
        const uint2 v = __ldcs(reinterpret_cast<const uint2*>(p));
        o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xffff0000u);
        o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xffff0000u);
    }
    __device__ __forceinline__ static void store(bf16* p, const float* i) {
        __nv_bfloat162 a = __floats2bfloat162_rn(i[0], i[1]), b = __floats2bfloat162_rn(i[2], i[3]);
        __stcs(reinterpret_cast<uint2*>(p), make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b)));
    }
};

// 4 / 8 consecutive io elements as fp32 (one 8/16-byte load for bf16)
__device__ __forceinline__ void load4(const float* p, float* o) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load4(const bf16* p, float* o) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xffff0000u);
    o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xffff0000u);
}
template <typename IoT>
__device__ __forceinline__ void load8(const IoT* p, float* o) {
    load4(p, o);
    load4(p + 4, o + 4);
}

// The dot products C_t . B_s of an ordinary step depend on (batch, group)
// only: one warp per (b, g) writes them for s <= fill (s == fill: this step's
// B) to cb [b][G][16], and every head of the group reads them.  Lane l covers
// elements [8l, 8l + 8) of an N-vector (N <= 256); tokens go in batches of 4
// whose loads are all issued before any is used.
template <typename IoT>
__global__ void __launch_bounds__(RP_WARPS * 32)
replay_dots_kernel(const IoT* __restrict__ Bb, const IoT* __restrict__ Bm, const IoT* __restrict__ Cm,
                   float* __restrict__ cb, int BG, int N, int K, int fill) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bg = blockIdx.x * RP_WARPS + warp;
    if (bg >= BG) return;
    const bool nl = 8 * lane < N;
    float creg[8];
    if (nl) load8(Cm + (size_t)bg * N + 8 * lane, creg);
    for (int s0 = 0; s0 <= fill; s0 += 4) {
        float bv[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = s0 + u;
            if (s <= fill && nl)
                load8((s < fill ? Bb + ((size_t)bg * K + s) * N : Bm + (size_t)bg * N) + 8 * lane, bv[u]);
            else {
#pragma unroll
                for (int j = 0; j < 8; ++j) bv[u][j] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float d = 0.f;
            if (nl) {
#pragma unroll
                for (int j = 0; j < 8; ++j) d = fmaf(creg[j], bv[u][j], d);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (lane == 0 && s0 + u <= fill) cb[(size_t)bg * 16 + s0 + u] = d;
        }
    }
}

// Packed fp32 pairs (low half = first element) and the sm_100 paired FMA: one
// instruction adds two consecutive buffered tokens' terms to a state element.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float f2lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// FLUSH: this step fills the buffer (fill == K - 1) and is folded into the
// checkpoint.  Buffers: xb [b][H][K][P], Bb [b][G][K][N] (io dtype), dtb and
// cumb [b][H][K] fp32 (dt_s after softplus and cum_s).
template <typename StateT, typename IoT, typename YT, bool FLUSH>
__global__ void __launch_bounds__(RP_WARPS * 32, FLUSH ? RP_MINB_FOLD : RP_MINB)
replay_step_kernel(StateT* __restrict__ ckpt, IoT* __restrict__ xb, IoT* __restrict__ Bb,
                   float* __restrict__ dtb, float* __restrict__ cumb, const float* __restrict__ cb,
                   const IoT* __restrict__ x, const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                   const float* __restrict__ A, const IoT* __restrict__ Bm, const IoT* __restrict__ Cm,
                   const float* __restrict__ Dv, YT* __restrict__ y, int BH, int H, int P, int N, int G,
                   int K, int fill) {
    extern __shared__ float rp_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x * RP_WARPS + warp;
    if (bh >= BH) return;                      // whole warps; no block barrier follows
    // per warp: C_t [N], then (flush) g[n][s] = beta_s B_s[n] for the 16 slots,
    // rows of RP_GS floats (16-byte aligned rows, read as 4 float4; the two rows
    // a warp reads at once fall in different banks)
    float* cs = rp_smem + (size_t)warp * (N + (FLUSH ? RP_GS * N : 0));
    float* gs = cs + N;
    const int b = bh / H, h = bh % H, hpg = H / G, g = h / hpg;
    const size_t bg = (size_t)b * G + g;
    const int vpr = P / RP_VEC;                // vectors per state row; divides 32
    const int rstep = 32 / vpr;
    const int vc = lane % vpr, r_off = lane / vpr;
    const int p0 = vc * RP_VEC;
    StateT* base = ckpt + (size_t)bh * N * P + p0;
    // state vectors in flight per lane (the fold holds x_s of 16 tokens as well)
    constexpr int U = FLUSH ? 4 : RP_U;

    // the prologue's independent loads first, so that they are in flight together:
    // this step's dt_raw and head parameters, the buffered cumsum and dt of lane
    // s's slot, C_t . B_s, C_t (N <= 256: at most 8 elements a lane), x_t
    const IoT* cg = Cm + bg * N;
    const IoT* bcur = Bm + bg * N;
    const float draw = to_f32(dt_raw[bh]), bias = dt_bias ? dt_bias[h] : 0.f, Ah = A[h];
    const float cumf = fill > 0 ? cumb[(size_t)bh * K + fill - 1] : 0.f;
    float cum_l = 0.f, dt_l = 0.f;
    if (lane < fill) {
        cum_l = cumb[(size_t)bh * K + lane];
        dt_l = dtb[(size_t)bh * K + lane];
    }
    const float cbv = (!FLUSH && lane <= fill) ? cb[bg * 16 + lane] : 0.f;   // C_t . B_s (ordinary step)
    float cv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) cv[i] = lane + 32 * i < N ? to_f32(cg[lane + 32 * i]) : 0.f;
    float xt[RP_VEC];
    load4(x + (size_t)bh * P + p0, xt);
    const float dt = softplus_f32(draw + bias);
    const float cum_t = cumf + dt * Ah;
    const float alpha = expf(cum_t);
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < N) cs[lane + 32 * i] = cv[i];
    // lane s <= fill: token s of the buffer (s == fill: this step's token)
    float beta = 0.f;
    if (lane <= fill) {
        const float cum_s = lane < fill ? cum_l : cum_t;
        const float dt_s = lane < fill ? dt_l : dt;
        beta = expf(cum_t - cum_s) * dt_s;
    }
    __syncwarp();
    float w = 0.f;                             // lane s: beta_s (C_t . B_s)
    if (!FLUSH) w = beta * cbv;
    uint64_t xs2[8][RP_VEC];                   // the fold's x pairs (below), loaded before the B rows
    if (FLUSH) {
        // x of the 16 slots for this lane's 4 columns (slot fill: x_t; past it: zero), as
        // pairs of consecutive slots per column: the paired FMA below adds slots 2k and
        // 2k + 1 of one column at once, against the coefficient pair (g_2k, g_2k+1)
#pragma unroll
        for (int k2 = 0; k2 < 8; ++k2) {
            float xa[RP_VEC], xb2[RP_VEC];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                const int s = 2 * k2 + z;
                float* xv = z ? xb2 : xa;
                if (s < fill) load4(xb + ((size_t)bh * K + s) * P + p0, xv);
                else {
#pragma unroll
                    for (int j = 0; j < RP_VEC; ++j) xv[j] = s == fill ? xt[j] : 0.f;
                }
            }
#pragma unroll
            for (int j = 0; j < RP_VEC; ++j) xs2[k2][j] = f2pack(xa[j], xb2[j]);
        }
    }
    if (FLUSH) {
        // g[n][s] for the 16 slots (unused slots K..15 get zero coefficients), the B_s
        // rows read as 16-byte vectors, 8 per lane in flight at once
        using BV = Vec16<IoT>;
        constexpr int VE = BV::N;              // elements per vector
        const int nvr = N / VE, nv = 16 * nvr;
        for (int v0 = 0; v0 < nv; v0 += 8 * 32) {
            uint4 raw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int v = v0 + i * 32 + lane, s = v / nvr, c = v - s * nvr;
                if (v < nv && s < K) {
                    const IoT* bs = s < fill ? Bb + (bg * K + s) * N : bcur;
                    raw[i] = *reinterpret_cast<const uint4*>(bs + c * VE);
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int v = v0 + i * 32 + lane, s = v / nvr, c = v - s * nvr;
                const float bt = __shfl_sync(0xffffffffu, beta, s & 15);
                if (v < nv) {
                    float f[VE];
                    if (s < K) BV::unpack(raw[i], f);
#pragma unroll
                    for (int e = 0; e < VE; ++e) gs[(c * VE + e) * RP_GS + s] = s < K ? bt * f[e] : 0.f;
                }
            }
        }
        __syncwarp();
    }

    float acc[RP_VEC] = {0.f, 0.f, 0.f, 0.f};
    if (!FLUSH) {
        // read-only pass: acc = sum_n C[n] h_c[n][cols]
        for (int r0 = r_off; r0 < N; r0 += U * rstep) {
            float hv[U][RP_VEC];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u * rstep;
                if (r < N) Vec4<StateT>::load(base + (size_t)r * P, hv[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u * rstep;
                if (r < N) {
                    const float c = cs[r];
#pragma unroll
                    for (int j = 0; j < RP_VEC; ++j) acc[j] = fmaf(c, hv[u][j], acc[j]);
                }
            }
        }
    } else {
        // h <- alpha h + sum_s g[n][s] x_s[cols] (even and odd slots summed apart, then
        // added); acc = sum_n C[n] h_new[n][cols]
        for (int r0 = r_off; r0 < N; r0 += U * rstep) {
            float hv[U][RP_VEC];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u * rstep;
                if (r < N) Vec4<StateT>::load(base + (size_t)r * P, hv[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u * rstep;
                if (r < N) {
                    const float4* g4 = reinterpret_cast<const float4*>(gs + r * RP_GS);
                    uint64_t gp[8];
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const float4 q4 = g4[k4];
                        gp[2 * k4] = f2pack(q4.x, q4.y);
                        gp[2 * k4 + 1] = f2pack(q4.z, q4.w);
                    }
                    float v[RP_VEC];
#pragma unroll
                    for (int j = 0; j < RP_VEC; ++j) {
                        uint64_t a2 = f2pack(alpha * hv[u][j], 0.f);
#pragma unroll
                        for (int k2 = 0; k2 < 8; ++k2) a2 = ffma2(gp[k2], xs2[k2][j], a2);
                        v[j] = f2lo(a2) + f2hi(a2);
                    }
                    Vec4<StateT>::store(base + (size_t)r * P, v);   // bf16: rounded to nearest even
                    const float c = cs[r];
#pragma unroll
                    for (int j = 0; j < RP_VEC; ++j) acc[j] = fmaf(c, v[j], acc[j]);
                }
            }
        }
    }
    // reduce over the lanes that share column vector vc (lane = vc + k * vpr)
    for (int o = vpr; o < 32; o <<= 1) {
#pragma unroll
        for (int j = 0; j < RP_VEC; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
    float yv[RP_VEC];
    const float d_skip = Dv ? Dv[h] : 0.f;
#pragma unroll
    for (int j = 0; j < RP_VEC; ++j) yv[j] = (FLUSH ? acc[j] : alpha * acc[j]) + d_skip * xt[j];
    if (!FLUSH) {
        for (int s0 = 0; s0 <= fill; s0 += 4) {   // warp-uniform bounds: every lane shuffles
            float xv[4][RP_VEC];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int s = s0 + u;
                if (s < fill) load4(xb + ((size_t)bh * K + s) * P + p0, xv[u]);
                else {
#pragma unroll
                    for (int j = 0; j < RP_VEC; ++j) xv[u][j] = s == fill ? xt[j] : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float ws = __shfl_sync(0xffffffffu, w, (s0 + u) & 31);
#pragma unroll
                for (int j = 0; j < RP_VEC; ++j) yv[j] = fmaf(ws, xv[u][j], yv[j]);
            }
        }
    }
    if (r_off == 0) {
        YT* yg = y + (size_t)bh * P + p0;
#pragma unroll
        for (int j = 0; j < RP_VEC; ++j) yg[j] = from_f32<YT>(yv[j]);
    }
    if (!FLUSH) {
        // append token t to the buffer (the group's first head writes B_t)
        IoT* xd = xb + ((size_t)bh * K + fill) * P;
        const IoT* xs_ = x + (size_t)bh * P;
        for (int i = lane; i < P; i += 32) xd[i] = xs_[i];
        if (h % hpg == 0) {
            IoT* bd = Bb + (bg * K + fill) * N;
            for (int i = lane; i < N; i += 32) bd[i] = bcur[i];
        }
        if (lane == 0) {
            dtb[(size_t)bh * K + fill] = dt;
            cumb[(size_t)bh * K + fill] = cum_t;
        }
    }
}

template <typename StateT, typename IoT, typename YT>
static cudaError_t launch_rp(const ReplayArgs& a, cudaStream_t s) {
    const long long bh = a.batch * a.H;
    const unsigned grid = (unsigned)((bh + RP_WARPS - 1) / RP_WARPS);
    const bool flush = a.fill == a.K - 1;
    const size_t smem = sizeof(float) * RP_WARPS * (size_t)a.N * (flush ? 1 + RP_GS : 1);
    if (flush) {
        auto k = replay_step_kernel<StateT, IoT, YT, true>;
        if (smem > 48 * 1024) {
            const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        k<<<grid, RP_WARPS * 32, smem, s>>>((StateT*)a.ckpt, (IoT*)a.xb, (IoT*)a.Bb, a.dtb, a.cumb, a.cb, (const IoT*)a.x,
                                            (const IoT*)a.dt_raw, a.dt_bias, a.A, (const IoT*)a.B, (const IoT*)a.C,
                                            a.D, (YT*)a.y, (int)bh, (int)a.H, (int)a.P, (int)a.N, (int)a.G,
                                            (int)a.K, (int)a.fill);
    } else {
        const long long bgs = a.batch * a.G;
        replay_dots_kernel<IoT><<<(unsigned)((bgs + RP_WARPS - 1) / RP_WARPS), RP_WARPS * 32, 0, s>>>(
            (const IoT*)a.Bb, (const IoT*)a.B, (const IoT*)a.C, a.cb, (int)bgs, (int)a.N, (int)a.K, (int)a.fill);
        replay_step_kernel<StateT, IoT, YT, false><<<grid, RP_WARPS * 32, smem, s>>>(
            (StateT*)a.ckpt, (IoT*)a.xb, (IoT*)a.Bb, a.dtb, a.cumb, a.cb, (const IoT*)a.x, (const IoT*)a.dt_raw,
            a.dt_bias, a.A, (const IoT*)a.B, (const IoT*)a.C, a.D, (YT*)a.y, (int)bh, (int)a.H, (int)a.P,
            (int)a.N, (int)a.G, (int)a.K, (int)a.fill);
    }
    return cudaGetLastError();
}

template <typename StateT, typename IoT>
static cudaError_t launch_rp_y(const ReplayArgs& a, cudaStream_t s) {
    return a.y_bf16 ? launch_rp<StateT, IoT, bf16>(a, s) : launch_rp<StateT, IoT, float>(a, s);
}

template <typename StateT>
static cudaError_t launch_rp_io(const ReplayArgs& a, cudaStream_t s) {
    return a.io_bf16 ? launch_rp_y<StateT, bf16>(a, s) : launch_rp_y<StateT, float>(a, s);
}

cudaError_t launch_replay_step(const ReplayArgs& a, cudaStream_t s) {
    if (a.batch == 0) return cudaSuccess;
    return a.state_bf16 ? launch_rp_io<bf16>(a, s) : launch_rp_io<float>(a, s);
}

}  // namespace ssd
