// Mamba-3 prefill: exponential-trapezoidal input and rotational state, run on
// the forward's chunked scan.
//
// The recurrence ("Mamba3", sections "New discretisation scheme" and on
// complex-valued SSMs; "Mamba-3 : SSM optimise inference", "Etats complexes
// via RoPE"), with the state rows (2k, 2k+1) a rotating pair:
//   h_t = a_t R(theta_t) (h_{t-1} + (1 - lam_t) dt_t B_{t-1} x_{t-1}^T) + lam_t dt_t B_t x_t^T
//   y_t = C_t^T h_t + D x_t,            a_t = exp(dt_t A)
// The pages' own remark that the rotations go into the matrices through a
// cumulative sum of angles is what makes the existing kernels reusable: with
// Theta_t = sum_{s<=t} theta_s and the rotated frame ~h_t = R(-Theta_t) h_t,
//   ~h_t = a_t ~h_{t-1} + a_t (1 - lam_t) dt_t ~B_{t-1} x_{t-1}^T + lam_t dt_t ~B_t x_t^T,
// ~B_t = R(-Theta_t) B_t, ~C_t = R(-Theta_t) C_t, and y_t = ~C_t^T ~h_t + D x_t.
// Expanding the sum, token s enters every later state with weight
//   w_s = lam_s dt_s + (1 - lam_{s+1}) dt_{s+1}      (w_{L-1} = lam_{L-1} dt_{L-1})
// and its own state with lam_s dt_s only, so
//   y_t = [scan with weights w, decays dt A, operands x, ~B, ~C] - c_t (C_t . B_t) x_t,
//   c_t = (1 - lam_{t+1}) dt_{t+1} (0 at t = L-1),
// and h_{L-1} = R(Theta_{L-1}) ~S_{L-1}.  (C_t . B_t is rotation invariant.)
// bf16 inputs: the turned operands are not bf16 numbers any more, and rounding
// them once costs 0.067 x rms(y) on the test shapes (float64 model), so each is
// stored as a bf16 pair hi + lo and, the scan being bilinear in (B, C), run as
// scan(B_hi, C_hi) + scan(B_lo, C_hi) + scan(B_hi, C_lo) (the lo x lo term, about
// 2^-18 relative, is dropped; the model then gives 9.8e-5).  Where the head-pair
// kernel covers the shape, its Mamba-3 form takes all three products and the
// correction in one scan (the turned operands then interleaved as
// [b][L][G][2][N], hi then lo).  fp32 inputs take one scan.
#include "../../include/ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

static inline size_t al256m(size_t v) { return (v + 255) & ~(size_t)255; }

Mamba3Layout mamba3_layout(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, int64_t Q,
                           bool io_bf16, bool tc) {
    Mamba3Layout l{};
    const int64_t BH = batch * H;
    PrefillLayout& s = l.scan;
    s.nchunks = (L + Q - 1) / Q;
    s.Lpad = s.nchunks * Q;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t o = off; off = al256m(off + bytes); return o; };
    s.off_dt = take(sizeof(float) * BH * s.Lpad);
    s.off_acs = take(sizeof(float) * BH * s.Lpad);
    const int64_t nstates = tc ? tc_runs(BH, s.nchunks, N) - 1 : s.nchunks;
    s.off_states = take(sizeof(float) * (size_t)N * P * BH * nstates);
    s.off_flags = take(sizeof(int) * ((size_t)BH + 64));
    const size_t e = io_bf16 ? 2 : 4, tok = (size_t)batch * L;
    const size_t opb = e * tok * G * N;        // one turned operand
    l.fused = io_bf16 && tc && pair_path_supports(batch, H, P, N, G, Q, io_bf16);
    l.off_corr = take(sizeof(float) * BH * s.Lpad);
    // bf16: hi and lo of each turned operand in one region (lo after hi, or
    // interleaved per group in the fused form)
    l.off_Bt = take(opb * (io_bf16 ? 2 : 1));
    l.off_Ct = take(opb * (io_bf16 ? 2 : 1));
    l.off_Btl = io_bf16 ? l.off_Bt + opb : 0;
    l.off_Ctl = io_bf16 ? l.off_Ct + opb : 0;
    l.off_csum = take(sizeof(double) * (size_t)batch * G * s.nchunks * (N / 2));
    l.off_rotL = take(sizeof(float2) * (size_t)batch * G * (N / 2));
    // fp32 scan outputs before the combination: three for the split scans, one
    // otherwise (the fused form writes y itself; lam without theta still combines)
    for (int i = 0; i < 3; ++i) l.off_y32[i] = (i == 0 || !l.fused) ? take(sizeof(float) * tok * H * P) : 0;
    l.off_fsr = take(sizeof(float) * (size_t)BH * N * P);
    l.off_fsr2 = take(sizeof(float) * (size_t)BH * N * P);
    s.total = off;
    l.total = off;
    return l;
}

// Sum of the angles of every (b, g, chunk) and pair k, in float64.  Block =
// (b, g, chunk); threads = (token lane, pair).
__global__ void __launch_bounds__(1024)
m3_angle_sums_kernel(const float* __restrict__ theta, double* __restrict__ csum, int64_t L, int G, int K, int Q,
                     int nchunks) {
    __shared__ double part[1024];
    const int c = (int)(blockIdx.x % (unsigned)nchunks);
    const int64_t bg = blockIdx.x / (unsigned)nchunks;
    const int g = (int)(bg % G);
    const int64_t b = bg / G;
    const int lanes = 1024 / K;                 // K = N/2 <= 128, so at least 8
    const int tid = threadIdx.x;
    double s = 0.0;
    if (tid < lanes * K) {
        const int k = tid % K, lane = tid / K;
        for (int l = lane; l < Q; l += lanes) {
            const int64_t t = (int64_t)c * Q + l;
            if (t < L) s += (double)theta[((b * L + t) * G + g) * K + k];
        }
    }
    part[tid] = s;
    __syncthreads();
    if (tid < K) {
        double v = 0.0;
        for (int j = 0; j < lanes; ++j) v += part[j * K + tid];
        csum[(bg * nchunks + c) * K + tid] = v;
    }
}

// The same sums with dstate a multiple of 8: block = (b, g, chunk, 4 pairs),
// thread = token (one 16-byte load of its 4 angles), a block reduction.
__global__ void __launch_bounds__(256)
m3_angle_sums4_kernel(const float* __restrict__ theta, double* __restrict__ csum, int64_t L, int G, int K, int Q,
                      int nchunks, int KG) {
    __shared__ double wsum[8][4];
    const int kg = (int)(blockIdx.x % (unsigned)KG);
    const int64_t rest = blockIdx.x / (unsigned)KG;
    const int c = (int)(rest % nchunks);
    const int64_t bg = rest / nchunks;
    const int g = (int)(bg % G);
    const int64_t b = bg / G;
    const int l = threadIdx.x, lane = l & 31, warp = l >> 5;
    const int64_t t = (int64_t)c * Q + l;
    double v[4] = {0.0, 0.0, 0.0, 0.0};
    if (l < Q && t < L) {
        const float4 a = *reinterpret_cast<const float4*>(theta + ((b * L + t) * G + g) * K + 4 * kg);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
        for (int o = 16; o > 0; o >>= 1) v[q] += __shfl_xor_sync(0xffffffffu, v[q], o);
    if (lane == 0)
#pragma unroll
        for (int q = 0; q < 4; ++q) wsum[warp][q] = v[q];
    __syncthreads();
    if (l < 4) {
        double tot = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += wsum[w][l];
        csum[(bg * nchunks + c) * K + 4 * kg + l] = tot;
    }
}

// 8 consecutive operand values (16-byte aligned) to fp32 and back
__device__ __forceinline__ void ld8(const bf16* p, float* o) { Vec16<bf16>::load(p, o); }
__device__ __forceinline__ void ld8(const float* p, float* o) {
    Vec16<float>::load(p, o);
    Vec16<float>::load(p + 4, o + 4);
}
__device__ __forceinline__ void st8(bf16* p, const float* v) { Vec16<bf16>::store(p, v); }
__device__ __forceinline__ void st8(float* p, const float* v) {
    Vec16<float>::store(p, v);
    Vec16<float>::store(p + 4, v + 4);
}

// ~B = R(-Theta_t) B, ~C = R(-Theta_t) C.  Block = (b, g, chunk, 4 pairs),
// thread = token: the cumulative angle is the previous chunks' sums (warp 0,
// lanes over chunks) plus a block scan over the chunk's tokens, in float64.
// The last token's angle is kept for rotating the final state back.
template <typename IoT>
__global__ void __launch_bounds__(256)
m3_rotate_kernel(const IoT* __restrict__ B, const IoT* __restrict__ C, const float* __restrict__ theta,
                 const double* __restrict__ csum, IoT* __restrict__ Bt, IoT* __restrict__ Ct, IoT* __restrict__ Btl,
                 IoT* __restrict__ Ctl, float2* __restrict__ rotL, int64_t L, int G, int N, int Q, int nchunks,
                 int KG, int ostride) {
    __shared__ double wtot[8][4];
    __shared__ double carry[4];
    const int kg = (int)(blockIdx.x % (unsigned)KG);
    const int64_t rest = blockIdx.x / (unsigned)KG;
    const int c = (int)(rest % nchunks);
    const int64_t bg = rest / nchunks;
    const int g = (int)(bg % G);
    const int64_t b = bg / G;
    const int K = N / 2, k0 = kg * 4;
    const int l = threadIdx.x, lane = l & 31, warp = l >> 5;
    const int64_t t = (int64_t)c * Q + l;
    const bool live = l < Q && t < L;
    if (warp == 0) {
        double cv[4] = {0.0, 0.0, 0.0, 0.0};
        for (int cc = lane; cc < c; cc += 32)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (k0 + q < K) cv[q] += csum[(bg * nchunks + cc) * K + k0 + q];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            for (int o = 16; o > 0; o >>= 1) cv[q] += __shfl_xor_sync(0xffffffffu, cv[q], o);
        if (lane == 0)
#pragma unroll
            for (int q = 0; q < 4; ++q) carry[q] = cv[q];
    }
    const bool vec = (N & 7) == 0;            // 4 whole pairs: 16-byte loads and stores
    double v[4] = {0.0, 0.0, 0.0, 0.0};
    if (vec && live) {
        const float4 a = *reinterpret_cast<const float4*>(theta + ((b * L + t) * G + g) * K + k0);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else if (!vec) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            v[q] = (live && k0 + q < K) ? (double)theta[((b * L + t) * G + g) * K + k0 + q] : 0.0;
    }
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double u = __shfl_up_sync(0xffffffffu, v[q], o);
            if (lane >= o) v[q] += u;
        }
    }
    if (lane == 31)
#pragma unroll
        for (int q = 0; q < 4; ++q) wtot[warp][q] = v[q];
    __syncthreads();
    for (int w = 0; w < warp; ++w)
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] += wtot[w][q];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] += carry[q];
    if (!live) return;
    const int64_t row = ((b * L + t) * G + g) * N;
    const int64_t orow = ((b * L + t) * G + g) * ostride;     // N, or 2N with hi and lo interleaved
    if (vec) {
        const int n0 = 2 * k0;
        float bv[8], cv[8], r[2][8];
        ld8(B + row + n0, bv);
        ld8(C + row + n0, cv);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            double sd, cd;
            sincos(v[q], &sd, &cd);
            const float cs = (float)cd, sn = (float)sd;
            r[0][2 * q] = cs * bv[2 * q] + sn * bv[2 * q + 1];
            r[0][2 * q + 1] = cs * bv[2 * q + 1] - sn * bv[2 * q];
            r[1][2 * q] = cs * cv[2 * q] + sn * cv[2 * q + 1];
            r[1][2 * q + 1] = cs * cv[2 * q + 1] - sn * cv[2 * q];
            if (t == L - 1) rotL[bg * K + k0 + q] = make_float2(cs, sn);
        }
        st8(Bt + orow + n0, r[0]);
        st8(Ct + orow + n0, r[1]);
        if (Btl) {
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int e = 0; e < 8; ++e) r[i][e] -= to_f32(from_f32<IoT>(r[i][e]));
            st8(Btl + orow + n0, r[0]);
            st8(Ctl + orow + n0, r[1]);
        }
        return;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if (k0 + q >= K) break;
        const int n0 = 2 * (k0 + q);
        double sd, cd;
        sincos(v[q], &sd, &cd);
        const float cs = (float)cd, sn = (float)sd;
        const float b0 = to_f32(B[row + n0]), b1 = to_f32(B[row + n0 + 1]);
        const float c0 = to_f32(C[row + n0]), c1 = to_f32(C[row + n0 + 1]);
        // R(-Theta): (u, w) -> (cos u + sin w, -sin u + cos w); stored as hi (+ lo for bf16)
        const float r[4] = {cs * b0 + sn * b1, cs * b1 - sn * b0, cs * c0 + sn * c1, cs * c1 - sn * c0};
        IoT* dst[4] = {Bt + orow + n0, Bt + orow + n0 + 1, Ct + orow + n0, Ct + orow + n0 + 1};
        IoT* dlo[4] = {Btl + orow + n0, Btl + orow + n0 + 1, Ctl + orow + n0, Ctl + orow + n0 + 1};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const IoT hi = from_f32<IoT>(r[i]);
            *dst[i] = hi;
            if (Btl) *dlo[i] = from_f32<IoT>(r[i] - to_f32(hi));
        }
        if (t == L - 1) rotL[bg * K + k0 + q] = make_float2(cs, sn);
    }
}

// Scan weights w, chunk-local decay cumsum and the diagonal correction's
// coefficient c, as the forward's decay kernel lays them out ([b*H][Lpad]);
// also clears the scan's hand-off flags.  Block = (b, chunk, 8 heads), thread =
// token.  With diag_w (the fused form) the third output is instead the weight of
// a token's own term, lam_t dt_t = w_t - c_t.
constexpr int M3_HG = 8;

template <typename IoT>
__global__ void __launch_bounds__(256)
m3_decay_kernel(const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias, const float* __restrict__ A,
                const float* __restrict__ lam, float* __restrict__ w_out, float* __restrict__ acs_out,
                float* __restrict__ corr_out, int* __restrict__ flags, int64_t L, int64_t Lpad, int H, int Q,
                int nflags, int nchunks, int hgroups, int diag_w) {
    __shared__ float warp_tot[8][M3_HG];
    const int hg = (int)(blockIdx.x % (unsigned)hgroups);
    const int c = (int)((blockIdx.x / (unsigned)hgroups) % (unsigned)nchunks);
    const int64_t b = blockIdx.x / ((unsigned)hgroups * (unsigned)nchunks);
    const int h0 = hg * M3_HG;
    const int l = threadIdx.x, lane = l & 31, warp = l >> 5;
    const int64_t t = (int64_t)c * Q + l;
    const bool live = l < Q && t < L, next = l < Q && t + 1 < L;
    float v[M3_HG], w[M3_HG], cr[M3_HG];
    // dt and lam of this token for the block's heads (16-byte loads when the 8 heads
    // are whole and aligned), then those of the next token from the next thread;
    // the last thread of a warp or of the chunk reads the next token itself
    auto load8 = [&](int64_t tt, float (&dtv)[M3_HG], float (&lmv)[M3_HG]) {
        const bool whole = (H & 7) == 0;
        if (whole) {
            float raw[M3_HG];
            if (sizeof(IoT) == 2) {
                Vec16<bf16>::load(reinterpret_cast<const bf16*>(dt_raw) + (b * L + tt) * H + h0, raw);
            } else {
                Vec16<float>::load(reinterpret_cast<const float*>(dt_raw) + (b * L + tt) * H + h0, raw);
                Vec16<float>::load(reinterpret_cast<const float*>(dt_raw) + (b * L + tt) * H + h0 + 4, raw + 4);
            }
            if (lam) {
                Vec16<float>::load(lam + (b * L + tt) * H + h0, lmv);
                Vec16<float>::load(lam + (b * L + tt) * H + h0 + 4, lmv + 4);
            }
#pragma unroll
            for (int k = 0; k < M3_HG; ++k) {
                dtv[k] = softplus_f32(raw[k] + (dt_bias ? dt_bias[h0 + k] : 0.f));
                if (!lam) lmv[k] = 1.f;
            }
        } else {
#pragma unroll
            for (int k = 0; k < M3_HG; ++k) {
                const int h = h0 + k;
                dtv[k] = 0.f;
                lmv[k] = 1.f;
                if (h < H) {
                    dtv[k] = softplus_f32(to_f32(dt_raw[(b * L + tt) * H + h]) + (dt_bias ? dt_bias[h] : 0.f));
                    if (lam) lmv[k] = lam[(b * L + tt) * H + h];
                }
            }
        }
    };
    float dt[M3_HG], lm[M3_HG], dtn[M3_HG], lmn[M3_HG];
#pragma unroll
    for (int k = 0; k < M3_HG; ++k) { dt[k] = 0.f; lm[k] = 1.f; dtn[k] = 0.f; lmn[k] = 1.f; }
    if (live) load8(t, dt, lm);
    const bool edge = lane == 31 || l == Q - 1;
#pragma unroll
    for (int k = 0; k < M3_HG; ++k) {
        dtn[k] = __shfl_down_sync(0xffffffffu, dt[k], 1);
        lmn[k] = __shfl_down_sync(0xffffffffu, lm[k], 1);
    }
    if (edge) {
#pragma unroll
        for (int k = 0; k < M3_HG; ++k) { dtn[k] = 0.f; lmn[k] = 1.f; }
        if (next) load8(t + 1, dtn, lmn);
    }
#pragma unroll
    for (int k = 0; k < M3_HG; ++k) {
        const int h = h0 + k;
        if (h >= H) { dt[k] = 0.f; dtn[k] = 0.f; lm[k] = 1.f; lmn[k] = 1.f; }
        if (!lam) { lm[k] = 1.f; lmn[k] = 1.f; }
        cr[k] = (1.f - lmn[k]) * dtn[k];      // 0 without lam, at the last token and past it
        w[k] = lm[k] * dt[k] + cr[k];
        v[k] = h < H ? dt[k] * A[h] : 0.f;
        if (diag_w) cr[k] = lm[k] * dt[k];
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int k = 0; k < M3_HG; ++k) {
            const float u = __shfl_up_sync(0xffffffffu, v[k], o);
            if (lane >= o) v[k] += u;
        }
    }
    if (lane == 31)
#pragma unroll
        for (int k = 0; k < M3_HG; ++k) warp_tot[warp][k] = v[k];
    __syncthreads();
    for (int ww = 0; ww < warp; ++ww)
#pragma unroll
        for (int k = 0; k < M3_HG; ++k) v[k] += warp_tot[ww][k];
    if (l < Q) {
#pragma unroll
        for (int k = 0; k < M3_HG; ++k) {
            if (h0 + k >= H) break;
            const int64_t o = (b * H + h0 + k) * Lpad + t;
            w_out[o] = w[k];
            acs_out[o] = v[k];
            corr_out[o] = cr[k];
        }
    }
    const int per = (int)((nflags + gridDim.x - 1) / gridDim.x);
    const int f0 = (int)blockIdx.x * per;
    for (int i = f0 + l; i < nflags && i < f0 + per; i += blockDim.x) flags[i] = 0;
}

// y_t = sum of the scans' outputs - c_t (C_t . B_t) x_t (corr NULL: no
// correction; y2, y3 NULL: one scan); one block per token row.  C_t . B_t is
// formed once per group (a warp per group, into shared memory), then the row's
// H * P outputs go 4 at a time (16-byte loads of y1, y2, y3), every thread of
// the block on consecutive vectors.  y1 and y may be the same fp32 array
// (corrected in place: each vector is read before it is written, by one thread).
template <typename IoT, typename YT>
__global__ void __launch_bounds__(256)
m3_combine_kernel(const float* y1, const float* __restrict__ y2, const float* __restrict__ y3,
                  const IoT* __restrict__ x, const IoT* __restrict__ B, const IoT* __restrict__ C,
                  const float* __restrict__ corr, YT* y, int64_t batch, int64_t L, int64_t Lpad, int H, int P, int N,
                  int G) {
    __shared__ float s_cb[256];                // C_t . B_t per group (G <= 256; else formed per vector)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int hpg = H / G;
    const int vpr = H * P / 4;                 // 4-vectors of a token row (P is a multiple of 8)
    for (int64_t r = blockIdx.x; r < batch * L; r += gridDim.x) {
        const int64_t b = r / L, t = r - b * L;
        const bool sh = corr && G <= 256;
        if (sh) {
            for (int g = warp; g < G; g += nwarps) {
                const int64_t grow = (r * G + g) * N;
                float cb = 0.f;
                for (int n = lane; n < N; n += 32) cb += to_f32(C[grow + n]) * to_f32(B[grow + n]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) cb += __shfl_xor_sync(0xffffffffu, cb, o);
                if (lane == 0) s_cb[g] = cb;
            }
            __syncthreads();
        }
        const int64_t row = r * H * P;
        for (int i = threadIdx.x; i < vpr; i += blockDim.x) {
            const int h = (4 * i) / P;
            float4 v = reinterpret_cast<const float4*>(y1 + row)[i];
            if (y2) {
                const float4 v2 = reinterpret_cast<const float4*>(y2 + row)[i];
                const float4 v3 = reinterpret_cast<const float4*>(y3 + row)[i];
                v.x += v2.x + v3.x; v.y += v2.y + v3.y; v.z += v2.z + v3.z; v.w += v2.w + v3.w;
            }
            float f = 0.f;
            if (corr) {
                float cb;
                if (sh) {
                    cb = s_cb[h / hpg];
                } else {                       // more groups than the table holds: per vector
                    const int64_t grow = (r * G + h / hpg) * N;
                    cb = 0.f;
                    for (int n = 0; n < N; ++n) cb += to_f32(C[grow + n]) * to_f32(B[grow + n]);
                }
                f = corr[(b * H + h) * Lpad + t] * cb;
            }
            float xv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) xv[e] = to_f32(x[row + 4 * i + e]);
            YT* o = y + row + 4 * i;
            o[0] = from_f32<YT>(v.x - f * xv[0]);
            o[1] = from_f32<YT>(v.y - f * xv[1]);
            o[2] = from_f32<YT>(v.z - f * xv[2]);
            o[3] = from_f32<YT>(v.w - f * xv[3]);
        }
        if (sh) __syncthreads();               // s_cb is rewritten for the next row
    }
}

// h_{L-1} = R(Theta_{L-1}) ~S_{L-1}: rows (2k, 2k+1) of every head of group g;
// ~S_{L-1} = src (+ src2, the B_lo scan's final state, when split).  Block =
// (b, h); rotL holds cos, sin of the last token's angle per (b, g, pair).
template <typename SrcT, typename StateT>
__global__ void __launch_bounds__(256)
m3_unrotate_state_kernel(const SrcT* __restrict__ src, const float* __restrict__ src2,
                         const float2* __restrict__ rotL, StateT* __restrict__ dst, int H, int P, int N, int G) {
    const int K = N / 2, hpg = H / G;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int64_t b = bh / H;
    const float2* rr = rotL + (b * G + h / hpg) * K;
    for (int i = threadIdx.x; i < K * P; i += blockDim.x) {
        const int k = i / P, p = i - k * P;
        const float2 cs = rr[k];
        const int64_t o0 = (bh * N + 2 * k) * P + p, o1 = o0 + P;
        float u = to_f32(src[o0]), v = to_f32(src[o1]);
        if (src2) {
            u += src2[o0];
            v += src2[o1];
        }
        dst[o0] = from_f32<StateT>(cs.x * u - cs.y * v);
        dst[o1] = from_f32<StateT>(cs.y * u + cs.x * v);
    }
}

static unsigned m3_grid(int64_t work, int64_t per_block) {
    const int64_t g = (work + per_block - 1) / per_block;
    return (unsigned)(g < 1 ? 1 : (g > 148 * 16 ? 148 * 16 : g));
}

__global__ void m3_clear_flags_kernel(int* __restrict__ flags, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) flags[i] = 0;
}

template <typename IoT>
static cudaError_t mamba3_t(const Mamba3Args& a, cudaStream_t s) {
    const Mamba3Layout& l = a.lay;
    char* ws = a.ws;
    const int H = (int)a.H, P = (int)a.P, N = (int)a.N, G = (int)a.G, Q = (int)a.Q;
    const int nchunks = (int)l.scan.nchunks, K = N / 2;
    const int nflags = (int)(a.batch * a.H + 64);
    const bool split = a.theta != nullptr && a.io_bf16;       // hi/lo operands, three scans
    cudaError_t e;
    IoT* Bt = (IoT*)(ws + l.off_Bt);
    IoT* Ct = (IoT*)(ws + l.off_Ct);
    // the fused form (one head-pair scan of the turned hi/lo operands): hi and lo
    // interleaved per group, [b][L][G][2][N]
    const bool fused = split && l.fused;
    IoT* Btl = split ? (fused ? Bt + N : (IoT*)(ws + l.off_Btl)) : nullptr;
    IoT* Ctl = split ? (fused ? Ct + N : (IoT*)(ws + l.off_Ctl)) : nullptr;
    float2* rotL = (float2*)(ws + l.off_rotL);
    if (a.theta) {
        const int KG = (K + 3) / 4;
        if ((N & 7) == 0)
            m3_angle_sums4_kernel<<<(unsigned)(a.batch * G * nchunks * KG), (unsigned)(Q < 32 ? 32 : Q), 0, s>>>(
                a.theta, (double*)(ws + l.off_csum), a.L, G, K, Q, nchunks, KG);
        else
            m3_angle_sums_kernel<<<(unsigned)(a.batch * G * nchunks), 1024, 0, s>>>(
                a.theta, (double*)(ws + l.off_csum), a.L, G, K, Q, nchunks);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        m3_rotate_kernel<IoT><<<(unsigned)(a.batch * G * nchunks * KG), (unsigned)(Q < 32 ? 32 : Q), 0, s>>>(
            (const IoT*)a.B, (const IoT*)a.C, a.theta, (const double*)(ws + l.off_csum), Bt, Ct, Btl, Ctl, rotL, a.L,
            G, N, Q, nchunks, KG, fused ? 2 * N : N);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const int hgroups = (H + M3_HG - 1) / M3_HG;
        m3_decay_kernel<IoT><<<(unsigned)(a.batch * nchunks * hgroups), (unsigned)(Q < 32 ? 32 : Q), 0, s>>>(
            (const IoT*)a.dt_raw, a.dt_bias, a.A, a.lam, (float*)(ws + l.scan.off_dt), (float*)(ws + l.scan.off_acs),
            (float*)(ws + l.off_corr), (int*)(ws + l.scan.off_flags), a.L, l.scan.Lpad, H, Q, nflags, nchunks,
            hgroups, fused ? 1 : 0);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (fused) {
        // one scan: the head-pair kernel's Mamba-3 form writes y (with D and the
        // trapezoid's own-token weights lam dt) and the final state, turned back
        // from fp32 as it is stored; the initial state enters the turned frame
        // unchanged (no angle before the first token)
        PrefillArgs p{};
        p.batch = a.batch; p.L = a.L; p.H = a.H; p.P = a.P; p.N = a.N; p.G = a.G; p.Q = a.Q;
        p.io_bf16 = true; p.y_bf16 = a.y_bf16; p.state_bf16 = a.state_bf16;
        p.x = a.x; p.dt_raw = a.dt_raw; p.dt_bias = a.dt_bias; p.A = a.A;
        p.B = Bt; p.C = Ct; p.D = a.D;
        p.init_state = a.init_state; p.y = a.y; p.final_state = a.final_state;
        p.ws = ws; p.lay = l.scan; p.pad_left = nullptr; p.dev_err = a.dev_err; p.drop_publish = 0;
        return launch_prefill_pair_mamba3(p, a.lam ? (const float*)(ws + l.off_corr) : nullptr, rotL, a.state_bf16,
                                          s);
    }
    // the scans: with lam or the split the outputs are combined (and corrected)
    // afterwards from fp32; with theta the final state is rotated back afterwards
    const bool combine = a.lam != nullptr || split;
    const bool unrotate = a.theta != nullptr && a.final_state != nullptr;
    const bool in_place = combine && !split && !a.y_bf16;     // one fp32 scan output, corrected in place
    float* y32[3] = {(float*)(ws + l.off_y32[0]), (float*)(ws + l.off_y32[1]), (float*)(ws + l.off_y32[2])};
    if (in_place) y32[0] = (float*)a.y;
    auto scan = [&](const void* Bs, const void* Cs, const float* D, const void* init, void* y, bool y_bf16,
                    void* fin, bool state_bf16, bool clear) -> cudaError_t {
        if (clear) {
            m3_clear_flags_kernel<<<m3_grid(nflags, 256), 256, 0, s>>>((int*)(ws + l.scan.off_flags), nflags);
            cudaError_t ce = cudaGetLastError();
            if (ce != cudaSuccess) return ce;
        }
        PrefillArgs p{};
        p.batch = a.batch; p.L = a.L; p.H = a.H; p.P = a.P; p.N = a.N; p.G = a.G; p.Q = a.Q;
        p.io_bf16 = a.io_bf16; p.y_bf16 = y_bf16; p.state_bf16 = state_bf16;
        p.x = a.x; p.dt_raw = a.dt_raw; p.dt_bias = a.dt_bias; p.A = a.A;
        p.B = Bs; p.C = Cs; p.D = D;
        p.init_state = init; p.y = y; p.final_state = fin;
        p.ws = ws; p.lay = l.scan; p.pad_left = nullptr; p.dev_err = a.dev_err; p.drop_publish = 0;
        return a.tc ? launch_prefill_tc(p, s) : launch_prefill_simt(p, s);
    };
    const void* B1 = a.theta ? (const void*)Bt : a.B;
    const void* C1 = a.theta ? (const void*)Ct : a.C;
    // scan 1 (hi, hi): D, the initial state, the final state in the state dtype
    e = scan(B1, C1, a.D, a.init_state, combine ? (void*)y32[0] : a.y, combine ? false : a.y_bf16,
             unrotate ? (void*)(ws + l.off_fsr) : a.final_state, a.state_bf16, false);
    if (e != cudaSuccess) return e;
    if (split) {
        // scan 2 (lo, hi): no initial state, its final state in fp32; scan 3 (hi, lo): the initial state read by C_lo
        e = scan(Btl, Ct, nullptr, nullptr, y32[1], false, unrotate ? (void*)(ws + l.off_fsr2) : nullptr, false, true);
        if (e != cudaSuccess) return e;
        e = scan(Bt, Ctl, nullptr, a.init_state, y32[2], false, nullptr, a.state_bf16, true);
        if (e != cudaSuccess) return e;
    }
    if (combine) {
        const unsigned grid = m3_grid(a.batch * a.L, 1);
        const float* y2 = split ? y32[1] : nullptr;
        const float* y3 = split ? y32[2] : nullptr;
        const float* corr = a.lam ? (const float*)(ws + l.off_corr) : nullptr;
        if (a.y_bf16)
            m3_combine_kernel<IoT, bf16><<<grid, 256, 0, s>>>(y32[0], y2, y3, (const IoT*)a.x, (const IoT*)a.B,
                                                             (const IoT*)a.C, corr, (bf16*)a.y, a.batch, a.L,
                                                             l.scan.Lpad, H, P, N, G);
        else
            m3_combine_kernel<IoT, float><<<grid, 256, 0, s>>>(y32[0], y2, y3, (const IoT*)a.x, (const IoT*)a.B,
                                                              (const IoT*)a.C, corr, (float*)a.y, a.batch, a.L,
                                                              l.scan.Lpad, H, P, N, G);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (unrotate) {
        const unsigned grid = (unsigned)(a.batch * H);
        const float* src2 = split ? (const float*)(ws + l.off_fsr2) : nullptr;
        if (a.state_bf16)
            m3_unrotate_state_kernel<bf16, bf16><<<grid, 256, 0, s>>>((const bf16*)(ws + l.off_fsr), src2, rotL,
                                                                     (bf16*)a.final_state, H, P, N, G);
        else
            m3_unrotate_state_kernel<float, float><<<grid, 256, 0, s>>>((const float*)(ws + l.off_fsr), src2, rotL,
                                                                      (float*)a.final_state, H, P, N, G);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_mamba3(const Mamba3Args& a, cudaStream_t s) {
    return a.io_bf16 ? mamba3_t<bf16>(a, s) : mamba3_t<float>(a, s);
}

int mamba3_launches(bool tc, bool io_bf16, bool has_lam, bool has_theta, bool has_final, bool fused) {
    const int scan = tc ? 1 : 3;
    const bool split = has_theta && io_bf16;
    // the fused form: angle sums, rotation, weights, the head-pair scan (which turns the final state back)
    if (split && fused) return 4;
    return (has_theta ? 2 : 0) + 1 + scan + (split ? 2 * (1 + scan) : 0) + ((has_lam || split) ? 1 : 0) +
           ((has_theta && has_final) ? 1 : 0);
}

}  // namespace ssd
