// Backward pass of the chunked prefill scan in block form (CUDA cores).
//
// The pages only say that end-to-end training also needs the backward pass
// ("Mamba-3 : SSM optimise inference", opening paragraph); what it computes
// follows from the forward recurrence h_t = exp(a_t) h_{t-1} + dt_t B_t x_t^T,
// a_t = dt_t A, y_t = C_t^T h_t + D x_t, for the loss
// sum_t <dy_t, y_t> + <dfinal, h_{L-1}>.
//
// The sequence is cut into blocks of qb tokens.  Two sequential passes give,
// per block j of every (b, h), the state entering it (h0_j) and the adjoint of
// the state at its end that comes from later blocks (Ge_j; dfinal for the last
// block); the second pass ends with d init_state.  Every gradient is then a
// function of one block's tokens, h0_j and Ge_j.  Inside a block, with r the
// block-local cumulative log-decay (r_t = sum of a over the block up to t),
// L[l][s] = exp(r_l - r_s) [s <= l], S[l][s] = C_l . B_s, w_s = exp(r_last - r_s):
//
//   dS[l][s] = L[l][s] dt_s (dy_l . x_s)
//   dxu_s    = sum_l S[l][s] L[l][s] dy_l + w_s (B_s^T Ge)          (= B_s^T G_s)
//   dx_s     = dt_s dxu_s + D dy_s
//   dB_s    += sum_l dS[l][s] C_l + dt_s w_s Ge x_s                 (summed over the group's heads)
//   dC_l    += sum_s dS[l][s] B_s + exp(r_l) h0 dy_l
//   d a_t    = <G_t, exp(a_t) h_{t-1}>
//            = sum_{l>=t, s<t} S[l][s] dS[l][s] + sum_{l>=t} exp(r_l) dy_l.(C_l^T h0)
//              + sum_{s<t} dt_s w_s x_s.(B_s^T Ge) + exp(r_last) <Ge, h0>
//   d dt_t   = x_t . dxu_t + A d a_t;  d dt_raw_t = d dt_t sigmoid(dt_raw_t + dt_bias)
//   dA = sum dt_t d a_t;  d dt_bias = sum d dt_raw;  dD = sum x_t . dy_t
//
// d a_t is formed inside its block from terms that do not cancel across the
// sequence, so its rounding error does not grow with the sequence length.  The
// first sum of d a_t runs over the rectangle l >= t > s; with the strict column
// and row sums c_k = sum_{l>k} S dS [l][k] and q_k = sum_{s<k} S dS [k][s] it is
// sum_{k<t} (c_k - q_k), a prefix over at most qb tokens.
#include "../../include/ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

namespace blk {

constexpr int THREADS = 256;
constexpr int EPT = 4;                   // state elements per thread in the state passes

// per-token scalars of the block kernel, fp32 unless noted
struct TokArrays {
    float *dt, *w, *er, *dk, *u, *v, *xdxu, *xdy;
};

}  // namespace blk

// The two sequential passes.  grid.x = (b*H) * 2: even blocks run forward in
// time (h0_j, the state entering block j), odd blocks backward (Ge_j, the
// adjoint of the state at the end of block j from later blocks, then
// d init_state); grid.y tiles the N*P state elements, EPT per thread.
template <typename IoT, typename StateT>
__global__ void __launch_bounds__(blk::THREADS)
bwd_blk_states_kernel(const IoT* __restrict__ x, const IoT* __restrict__ dy, const IoT* __restrict__ B,
                      const IoT* __restrict__ C, const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias,
                      const float* __restrict__ A, const StateT* __restrict__ init, const StateT* __restrict__ dfin,
                      float* __restrict__ h0, float* __restrict__ ge, StateT* __restrict__ dinit, int64_t L,
                      int H, int P, int N, int G, int qb, int64_t nb) {
    const int64_t bh = blockIdx.x >> 1;
    const bool rev = blockIdx.x & 1;
    const int h = (int)(bh % H);
    const int64_t b = bh / H;
    const int g = h / (H / G);
    const int64_t NP = (int64_t)N * P;
    const float Ah = A[h], bias = dt_bias ? dt_bias[h] : 0.f;
    int64_t e[blk::EPT];
    int nn[blk::EPT], pp[blk::EPT];
    float s[blk::EPT];
#pragma unroll
    for (int k = 0; k < blk::EPT; ++k) {
        e[k] = (int64_t)blockIdx.y * blk::THREADS * blk::EPT + k * blk::THREADS + threadIdx.x;
        const bool ok = e[k] < NP;
        nn[k] = ok ? (int)(e[k] / P) : 0;
        pp[k] = ok ? (int)(e[k] % P) : 0;
        const StateT* src = rev ? dfin : init;
        s[k] = (ok && src) ? to_f32(src[bh * NP + e[k]]) : 0.f;
    }
    const IoT* vin = rev ? dy : x;            // the P-side operand
    const IoT* nin = rev ? C : B;             // the N-side operand
    float* out = rev ? ge : h0;
    for (int64_t i = 0; i < L; ++i) {
        const int64_t t = rev ? L - 1 - i : i;
        const int64_t row = b * L + t;
        const float dt = softplus_f32(to_f32(dt_raw[row * H + h]) + bias);
        const float decay = expf(dt * Ah);
        const bool store = rev ? (t % qb == qb - 1 || t == L - 1) : (t % qb == 0);
        const IoT* vr = vin + (row * H + h) * P;
        const IoT* nr = nin + (row * G + g) * N;
#pragma unroll
        for (int k = 0; k < blk::EPT; ++k) {
            if (e[k] >= NP) continue;
            if (store) out[(bh * nb + t / qb) * NP + e[k]] = s[k];
            const float prod = to_f32(nr[nn[k]]) * to_f32(vr[pp[k]]);
            s[k] = rev ? decay * (s[k] + prod) : fmaf(decay, s[k], dt * prod);
        }
    }
    if (rev && dinit) {
#pragma unroll
        for (int k = 0; k < blk::EPT; ++k)
            if (e[k] < NP) dinit[bh * NP + e[k]] = from_f32<StateT>(s[k]);
    }
}

// One block per (b, group, block j): the group's heads one after another, dB
// and dC summed over them in shared memory (fixed order: bitwise
// deterministic).  Dynamic shared memory, floats: B, C, dB, dC [qb][N]; x, dy,
// t1, t2 [qb][P]; S, M, dS [qb][qb]; 8 per-token arrays [qb]; then the
// block-local cumulative log-decay as doubles [qb] and a reduction scratch.
template <typename IoT, typename GT>
__global__ void __launch_bounds__(blk::THREADS)
bwd_blk_kernel(const IoT* __restrict__ x, const IoT* __restrict__ dy, const IoT* __restrict__ B,
               const IoT* __restrict__ C, const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias,
               const float* __restrict__ A, const float* __restrict__ Dv, const float* __restrict__ h0,
               const float* __restrict__ ge, GT* __restrict__ dx, GT* __restrict__ ddt_raw, GT* __restrict__ dB,
               GT* __restrict__ dC, float* __restrict__ part, int64_t L, int H, int P, int N, int G, int qb,
               int64_t nb) {
    extern __shared__ __align__(16) float sm[];
    const int tid = threadIdx.x;
    const int64_t j = blockIdx.x % nb;
    const int64_t bg = blockIdx.x / nb;
    const int g = (int)(bg % G);
    const int64_t b = bg / G;
    const int hpg = H / G;
    const int64_t t0 = j * qb;
    const int n = (int)(L - t0 < qb ? L - t0 : qb);
    const int64_t NP = (int64_t)N * P;

    float* Bs = sm;
    float* Cs = Bs + qb * N;
    float* dBa = Cs + qb * N;
    float* dCa = dBa + qb * N;
    float* Xs = dCa + qb * N;
    float* Ys = Xs + qb * P;
    float* T1 = Ys + qb * P;                  // B Ge
    float* T2 = T1 + qb * P;                  // C h0, then dxu
    float* S = T2 + qb * P;
    float* Mf = S + qb * qb;                  // S L (no dt)
    float* dS = Mf + qb * qb;
    blk::TokArrays ta;
    ta.dt = dS + qb * qb;
    ta.w = ta.dt + qb;
    ta.er = ta.w + qb;
    ta.dk = ta.er + qb;
    ta.u = ta.dk + qb;
    ta.v = ta.u + qb;
    ta.xdxu = ta.v + qb;
    ta.xdy = ta.xdxu + qb;
    double* rr = reinterpret_cast<double*>(ta.xdy + qb + (qb & 1));
    float* red = reinterpret_cast<float*>(rr + qb);          // THREADS floats

    // B, C of the block; dB, dC accumulators; S = C B^T (lower triangle)
    for (int i = tid; i < qb * N; i += blk::THREADS) {
        const int l = i / N, k = i % N;
        const bool ok = l < n;
        Bs[i] = ok ? to_f32(B[((b * L + t0 + l) * G + g) * N + k]) : 0.f;
        Cs[i] = ok ? to_f32(C[((b * L + t0 + l) * G + g) * N + k]) : 0.f;
        dBa[i] = 0.f;
        dCa[i] = 0.f;
    }
    __syncthreads();
    for (int i = tid; i < qb * qb; i += blk::THREADS) {
        const int l = i / qb, s = i % qb;
        float acc = 0.f;
        if (s <= l && l < n)
            for (int k = 0; k < N; ++k) acc = fmaf(Cs[l * N + k], Bs[s * N + k], acc);
        S[i] = acc;
    }

    for (int q = 0; q < hpg; ++q) {
        const int h = g * hpg + q;
        const int64_t bh = b * H + h;
        const float Ah = A[h], bias = dt_bias ? dt_bias[h] : 0.f, dsk = Dv ? Dv[h] : 0.f;
        const float* h0j = h0 + (bh * nb + j) * NP;
        const float* gej = ge + (bh * nb + j) * NP;
        __syncthreads();                      // the previous head is done with every array
        for (int i = tid; i < qb * P; i += blk::THREADS) {
            const int l = i / P, p = i % P;
            const bool ok = l < n;
            Xs[i] = ok ? to_f32(x[((b * L + t0 + l) * H + h) * P + p]) : 0.f;
            Ys[i] = ok ? to_f32(dy[((b * L + t0 + l) * H + h) * P + p]) : 0.f;
        }
        if (tid < 32) {
            // dt and the block-local cumulative log-decay (double), one warp, qb <= 32
            const int t = tid;
            float dt = 0.f;
            if (t < n) dt = softplus_f32(to_f32(dt_raw[(b * L + t0 + t) * H + h]) + bias);
            double v = t < n ? (double)(dt * Ah) : 0.0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double w = __shfl_up_sync(0xffffffffu, v, o);
                if (t >= o) v += w;
            }
            const double rlast = __shfl_sync(0xffffffffu, v, n - 1);
            if (t < qb) {
                rr[t] = v;
                ta.dt[t] = dt;
                ta.w[t] = t < n ? expf((float)(rlast - v)) : 0.f;
                ta.er[t] = t < n ? expf((float)v) : 0.f;
            }
        }
        __syncthreads();
        // M = S L and dS = L dt_s (dy_l . x_s) on the lower triangle
        for (int i = tid; i < qb * qb; i += blk::THREADS) {
            const int l = i / qb, s = i % qb;
            float m = 0.f, d = 0.f;
            if (s <= l && l < n) {
                const float f = expf((float)(rr[l] - rr[s]));
                float dyx = 0.f;
                for (int p = 0; p < P; ++p) dyx = fmaf(Ys[l * P + p], Xs[s * P + p], dyx);
                m = S[i] * f;
                d = f * ta.dt[s] * dyx;
            }
            Mf[i] = m;
            dS[i] = d;
        }
        // T1 = B Ge, T2 = C h0 (rows of the block)
        for (int i = tid; i < qb * P; i += blk::THREADS) {
            const int l = i / P, p = i % P;
            float a1 = 0.f, a2 = 0.f;
            if (l < n)
                for (int k = 0; k < N; ++k) {
                    a1 = fmaf(Bs[l * N + k], gej[(int64_t)k * P + p], a1);
                    a2 = fmaf(Cs[l * N + k], h0j[(int64_t)k * P + p], a2);
                }
            T1[i] = a1;
            T2[i] = a2;
        }
        // exp(r_last) <Ge, h0>
        float kp = 0.f;
        for (int64_t i = tid; i < NP; i += blk::THREADS) kp = fmaf(gej[i], h0j[i], kp);
        red[tid] = kp;
        __syncthreads();
        if (tid < qb) {
            // c_k - q_k (strict column and row sums of S dS), u, v, x . dy
            const int k = tid;
            float c = 0.f, r = 0.f, u = 0.f, v = 0.f, xdy = 0.f;
            if (k < n) {
                for (int l = k + 1; l < n; ++l) c = fmaf(S[l * qb + k], dS[l * qb + k], c);
                for (int s = 0; s < k; ++s) r = fmaf(S[k * qb + s], dS[k * qb + s], r);
                for (int p = 0; p < P; ++p) {
                    u = fmaf(Ys[k * P + p], T2[k * P + p], u);
                    v = fmaf(Xs[k * P + p], T1[k * P + p], v);
                    xdy = fmaf(Xs[k * P + p], Ys[k * P + p], xdy);
                }
            }
            ta.dk[k] = c - r;
            ta.u[k] = ta.er[k] * u;
            ta.v[k] = ta.dt[k] * ta.w[k] * v;
            ta.xdy[k] = xdy;
        }
        if (tid == blk::THREADS - 1) {
            float s = 0.f;
            for (int i = 0; i < blk::THREADS; ++i) s += red[i];
            red[0] = s;                       // read after the next barrier only
        }
        __syncthreads();
        const float K = ta.er[n - 1] * red[0];
        // dxu = M^T dy + w (B Ge) into T2; dx
        for (int i = tid; i < qb * P; i += blk::THREADS) {
            const int s = i / P, p = i % P;
            float acc = 0.f;
            if (s < n) {
                for (int l = s; l < n; ++l) acc = fmaf(Mf[l * qb + s], Ys[l * P + p], acc);
                acc = fmaf(ta.w[s], T1[i], acc);
                dx[((b * L + t0 + s) * H + h) * P + p] = from_f32<GT>(fmaf(ta.dt[s], acc, dsk * Ys[i]));
            }
            T2[i] = acc;
        }
        // dB += dS^T C + dt w (x Ge^T);  dC += dS B + exp(r) (dy h0^T)
        for (int i = tid; i < qb * N; i += blk::THREADS) {
            const int s = i / N, k = i % N;
            if (s >= n) continue;
            float ab = 0.f, ac = 0.f, xg = 0.f, yh = 0.f;
            for (int l = s; l < n; ++l) ab = fmaf(dS[l * qb + s], Cs[l * N + k], ab);
            for (int t = 0; t <= s; ++t) ac = fmaf(dS[s * qb + t], Bs[t * N + k], ac);
            for (int p = 0; p < P; ++p) {
                xg = fmaf(Xs[s * P + p], gej[(int64_t)k * P + p], xg);
                yh = fmaf(Ys[s * P + p], h0j[(int64_t)k * P + p], yh);
            }
            dBa[i] += fmaf(ta.dt[s] * ta.w[s], xg, ab);
            dCa[i] += fmaf(ta.er[s], yh, ac);
        }
        __syncthreads();
        if (tid < qb) {
            const int t = tid;
            float xdxu = 0.f;
            for (int p = 0; p < P; ++p) xdxu = fmaf(Xs[t * P + p], T2[t * P + p], xdxu);
            ta.xdxu[t] = xdxu;
        }
        __syncthreads();
        if (tid < 32) {
            // d a_t, d dt_raw, and this block's shares of dA, d dt_bias, dD
            const int t = tid;
            float da = 0.f, sa = 0.f, sb = 0.f, sd = 0.f;
            if (t < n) {
                float R = 0.f, U = 0.f, V = 0.f;
                for (int k = 0; k < t; ++k) {
                    R += ta.dk[k];
                    V += ta.v[k];
                }
                for (int l = t; l < n; ++l) U += ta.u[l];
                da = R + U + V + K;
                const float z = to_f32(dt_raw[(b * L + t0 + t) * H + h]) + bias;
                const float dz = (ta.xdxu[t] + Ah * da) / (1.f + expf(-z));
                ddt_raw[(b * L + t0 + t) * H + h] = from_f32<GT>(dz);
                sa = ta.dt[t] * da;
                sb = dz;
                sd = ta.xdy[t];
            }
            // fixed-order sums over the block's tokens
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sa += __shfl_down_sync(0xffffffffu, sa, o);
                sb += __shfl_down_sync(0xffffffffu, sb, o);
                sd += __shfl_down_sync(0xffffffffu, sd, o);
            }
            if (t == 0) {
                float* pp = part + ((b * nb + j) * H + h) * 3;
                pp[0] = sa;
                pp[1] = sb;
                pp[2] = sd;
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < n * N; i += blk::THREADS) {
        const int l = i / N, k = i % N;
        dB[((b * L + t0 + l) * G + g) * N + k] = from_f32<GT>(dBa[i]);
        dC[((b * L + t0 + l) * G + g) * N + k] = from_f32<GT>(dCa[i]);
    }
}

size_t blk_smem_bytes(int qb, int P, int N) {
    return sizeof(float) * ((size_t)4 * qb * N + (size_t)4 * qb * P + (size_t)3 * qb * qb + 8 * qb + 1) +
           sizeof(double) * (qb + 1) + sizeof(float) * blk::THREADS;
}

int blk_block_size(int P, int N) {
    return blk_smem_bytes(32, P, N) <= 200 * 1024 ? 32 : 16;
}

cudaError_t launch_backward_blocks_cc(const BackwardArgs& a, cudaStream_t s);

template <typename IoT, typename GT, typename StateT>
static cudaError_t blocks_cc_t(const BackwardArgs& a, cudaStream_t s) {
    const BackwardLayout& l = a.lay;
    const int qb = (int)l.qb;
    const int64_t nb = l.nb;
    const int H = (int)a.H, P = (int)a.P, N = (int)a.N, G = (int)a.G;
    float* h0 = (float*)(a.ws + l.off_h0);
    float* ge = (float*)(a.ws + l.off_ge);
    float* part = (float*)(a.ws + l.off_part);
    const int64_t NP = a.N * a.P;
    const dim3 sgrid((unsigned)(a.batch * a.H * 2), (unsigned)((NP + blk::THREADS * blk::EPT - 1) / (blk::THREADS * blk::EPT)));
    bwd_blk_states_kernel<IoT, StateT><<<sgrid, blk::THREADS, 0, s>>>(
        (const IoT*)a.x, (const IoT*)a.dy, (const IoT*)a.B, (const IoT*)a.C, (const IoT*)a.dt_raw, a.dt_bias, a.A,
        (const StateT*)a.init_state, (const StateT*)a.dfinal, h0, ge, (StateT*)a.dinit, a.L, H, P, N, G, qb, nb);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = blk_smem_bytes(qb, P, N);
    auto k = bwd_blk_kernel<IoT, GT>;
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k<<<(unsigned)(a.batch * a.G * nb), blk::THREADS, smem, s>>>(
        (const IoT*)a.x, (const IoT*)a.dy, (const IoT*)a.B, (const IoT*)a.C, (const IoT*)a.dt_raw, a.dt_bias, a.A,
        a.D, h0, ge, (GT*)a.dx, (GT*)a.ddt_raw, (GT*)a.dB, (GT*)a.dC, part, a.L, H, P, N, G, qb, nb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_backward_params(part, a.dA, a.ddt_bias, a.dD, a.batch * nb, H, s);
}

template <typename IoT, typename GT>
static cudaError_t blocks_cc_s(const BackwardArgs& a, cudaStream_t s) {
    return a.state_bf16 ? blocks_cc_t<IoT, GT, bf16>(a, s) : blocks_cc_t<IoT, GT, float>(a, s);
}

template <typename IoT>
static cudaError_t blocks_cc_g(const BackwardArgs& a, cudaStream_t s) {
    return a.grad_bf16 ? blocks_cc_s<IoT, bf16>(a, s) : blocks_cc_s<IoT, float>(a, s);
}

cudaError_t launch_backward_blocks_cc(const BackwardArgs& a, cudaStream_t s) {
    return a.io_bf16 ? blocks_cc_g<bf16>(a, s) : blocks_cc_g<float>(a, s);
}

}  // namespace ssd
