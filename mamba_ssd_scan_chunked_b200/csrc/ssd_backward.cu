// Backward pass of the chunked prefill scan.
//
// The pages only say that end-to-end training also needs the backward pass
// ("Mamba-3 : SSM optimise inference", opening paragraph); what it computes
// follows from the forward recurrence h_t = exp(dt_t A) h_{t-1} + dt_t B_t x_t^T,
// y_t = C_t^T h_t + D x_t, for the loss sum_t <dy_t, y_t> + <dfinal, h_{L-1}>.
//
// Every gradient is again a scan of the same shape, so the forward's chunked
// kernels (tensor-core or CUDA-core path) compute them on rearranged operands.
// With S_t = exp(alpha_t) S_{t-1} + w_t Bs_t xs_t^T and out_t = Cs_t^T S_t the
// forward scan's contract (weights w and log-decays alpha are written straight
// into the scan's workspace):
//
//  R1  the state adjoint G_t = C_t dy_t^T + exp(a_{t+1}) G_{t+1} (N x P),
//      a_t = dt_t A, is that scan run backwards in time: tau = L-1-t, w = 1,
//      alpha_tau = a_{L-tau} (alpha_0 = 0), xs = dy, Bs = C, Cs = B, initial
//      state dfinal.  out = B_t^T G_t ("dxu"); final state = G_0.
//  R2  the same recurrence transposed (G^T, P x N): xs = C (per head),
//      Bs = dy, Cs = x, initial state dfinal^T.  out = G_t x_t.
//  F   the forward state transposed (h^T, P x N): xs = B (per head), Bs = x,
//      Cs = dy, the forward's own dt and decays, initial state init^T.
//      out = h_t dy_t; final state = h_{L-1}^T.
//  R2 and F have headdim N and dstate P; on the tensor-core path N is split in
//  64-column slices (columns of a state are independent), one scan per slice.
//
// Then per token (b, t, h):
//   dx_t    = dt_t dxu_t + D dy_t
//   dB_t    = sum over the group's heads of dt_t G_t x_t;  dC_t = sum of h_t dy_t
//   the log-decay gradient uses the identity (differentiate y and the final
//   state in the cumulative log-decay Lam_u = sum_{r<=u} a_r, with Lam_u and
//   every other Lam independent):
//     d loss / d Lam_u = dy_u.(y_u - D x_u) - dt_u x_u.dxu_u + [u = L-1] <dfinal, h_{L-1}>
//   with dy_u.(y_u - D x_u) = C_u . (h_u dy_u); then d loss / d a_t is its suffix
//   sum over u >= t, and
//   d dt_t  = x_t.dxu_t + A d a_t;   d dt_raw_t = d dt_t sigmoid(dt_raw_t + dt_bias)
//   dA = sum dt_t d a_t;  d dt_bias = sum d dt_raw;  dD = sum <dy_t, x_t>;
//   d init_state = exp(a_0) G_0.
#include "../../include/ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

static inline size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

BackwardLayout backward_layout(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, int64_t Q,
                               bool io_bf16) {
    BackwardLayout l{};
    const int64_t BH = batch * H;
    const int64_t nb128 = (L + 127) / 128;
    if (bwd_tc_supports(H, P, N, G, io_bf16) && batch * (nb128 > 0 ? nb128 : 1) * G <= 65535 &&
        BH * nb128 < ((int64_t)1 << 31)) {
        // bf16 inputs, dstate 128, headdim 64, head pairs: the block form on tensor cores
        l.mode = 2;
        l.qb = 128;
        l.nb = nb128;
        size_t off = 0;
        auto take = [&](size_t bytes) { const size_t o = off; off = al256(off + bytes); return o; };
        const int64_t nbk = l.nb > 0 ? l.nb : 1;
        const size_t st = (size_t)2 * 2 * BH * nbk * N * P;        // bf16 hi and lo
        l.off_h0 = take(st);
        l.off_ge = take(st);
        l.off_part = take(sizeof(float) * 3 * (size_t)batch * nbk * H);
        int64_t grid = 0, smax = 0;
        bwd_tc_grid(batch, L, H, G, &grid, &smax);
        l.off_dbc = take(sizeof(float) * (size_t)grid * smax * 2 * 128 * 128);
        l.total = off;
        return l;
    }
    if (!io_bf16) {
        // fp32 inputs: the block form on CUDA cores
        l.mode = 1;
        l.qb = blk_block_size((int)P, (int)N);
        l.nb = (L + l.qb - 1) / l.qb;
        size_t off = 0;
        auto take = [&](size_t bytes) { const size_t o = off; off = al256(off + bytes); return o; };
        const size_t st = sizeof(float) * (size_t)BH * (l.nb > 0 ? l.nb : 1) * N * P;
        l.off_h0 = take(st);
        l.off_ge = take(st);
        l.off_part = take(sizeof(float) * 3 * (size_t)batch * (l.nb > 0 ? l.nb : 1) * H);
        l.total = off;
        return l;
    }
    l.nchunks = (L + Q - 1) / Q;
    l.Lpad = l.nchunks * Q;
    l.tc_main = tc_path_supports(P, N, Q, io_bf16);
    l.pw = (N % 64 == 0 && tc_path_supports(64, P, Q, io_bf16)) ? 64 : N;
    l.nblk = N / l.pw;
    l.tc_t = tc_path_supports(l.pw, P, Q, io_bf16);
    const size_t e = io_bf16 ? 2 : 4, f = 4;
    const size_t tok = (size_t)batch * L;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t o = off; off = al256(off + bytes); return o; };
    l.off_dtf = take(f * BH * l.Lpad);
    l.off_acsf = take(f * BH * l.Lpad);
    l.off_dtr = take(f * BH * l.Lpad);
    l.off_acsr = take(f * BH * l.Lpad);
    // run-entry states (tensor-core path) or chunk states (CUDA-core path) of
    // whichever scan needs most; the scans run one after another
    auto states = [&](bool tc, int64_t n, int64_t p) {
        const int64_t k = tc ? tc_runs(BH, l.nchunks, n) - 1 : l.nchunks;
        return f * (size_t)n * p * BH * k;
    };
    const size_t s1 = states(l.tc_main, N, P), s2 = states(l.tc_t, P, l.pw);
    l.off_states = take(s1 > s2 ? s1 : s2);
    l.off_flags = take(sizeof(int) * ((size_t)BH + 64));
    l.off_dyr = take(e * tok * H * P);
    l.off_xr = take(e * tok * H * P);
    l.off_Cr = take(e * tok * G * N);
    l.off_Br = take(e * tok * G * N);
    l.slice_io = al256(e * tok * H * l.pw);
    l.off_Cer = take(l.slice_io * l.nblk);
    l.off_Be = take(l.slice_io * l.nblk);
    const size_t st = f * (size_t)BH * N * P;
    l.slice_st = al256(f * (size_t)BH * P * l.pw);
    l.off_dfin = take(st);
    l.off_G0 = take(st);
    l.off_dfinT = take(l.slice_st * l.nblk);
    l.off_h0T = take(l.slice_st * l.nblk);
    l.off_hfT = take(l.slice_st * l.nblk);
    l.off_y1 = take(f * tok * H * P);
    l.slice_y = al256(f * tok * H * l.pw);
    l.off_y2 = take(l.slice_y * l.nblk);
    l.off_y3 = take(l.slice_y * l.nblk);
    l.off_tok = take(f * 3 * (size_t)BH * L);
    l.off_part = take(f * 3 * (size_t)BH);
    l.total = off;
    return l;
}

// ---------------------------------------------------------------- kernels

// Time-reversed and per-head copies of the token operands, one (b, t) row per
// block iteration, in 16-byte vectors (every row segment copied is a multiple
// of 16 bytes and starts on a 16-byte boundary: H*P, G*N, N and pw are
// multiples of 8 elements): dy, x, C, B reversed; C reversed and B forward,
// expanded to every head and cut into column slices of width pw.
template <typename IoT>
__global__ void __launch_bounds__(256)
bwd_prep_tokens_kernel(const IoT* __restrict__ x, const IoT* __restrict__ dy, const IoT* __restrict__ B,
                       const IoT* __restrict__ C, IoT* __restrict__ dyr, IoT* __restrict__ xr,
                       IoT* __restrict__ Cr, IoT* __restrict__ Br, IoT* __restrict__ Cer, IoT* __restrict__ Be,
                       int64_t batch, int64_t L, int H, int P, int N, int G, int pw, int nblk,
                       int64_t slice_elems) {
    constexpr int V = 16 / sizeof(IoT);            // elements per vector
    const int64_t rows = batch * L;
    const int hpv = H * P / V, gnv = G * N / V, pwv = pw / V, hpg = H / G;
    const int segs = nblk * H * pwv;               // vectors of the expanded rows
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t b = r / L, t = r % L;
        const int64_t rr = b * L + (L - 1 - t);
        const uint4* xs = reinterpret_cast<const uint4*>(x + r * H * P);
        const uint4* dys = reinterpret_cast<const uint4*>(dy + r * H * P);
        uint4* xd = reinterpret_cast<uint4*>(xr + rr * H * P);
        uint4* dyd = reinterpret_cast<uint4*>(dyr + rr * H * P);
        for (int i = threadIdx.x; i < hpv; i += blockDim.x) {
            dyd[i] = __ldcs(dys + i);
            xd[i] = __ldcs(xs + i);
        }
        const uint4* Cs = reinterpret_cast<const uint4*>(C + r * G * N);
        const uint4* Bs = reinterpret_cast<const uint4*>(B + r * G * N);
        uint4* Cd = reinterpret_cast<uint4*>(Cr + rr * G * N);
        uint4* Bd = reinterpret_cast<uint4*>(Br + rr * G * N);
        for (int i = threadIdx.x; i < gnv; i += blockDim.x) {
            Cd[i] = Cs[i];
            Bd[i] = Bs[i];
        }
        for (int i = threadIdx.x; i < segs; i += blockDim.x) {
            const int j = i / (H * pwv), rem = i % (H * pwv), h = rem / pwv, k = rem % pwv;
            const int64_t src = (int64_t)(h / hpg) * N + j * pw;          // element offset in the (b, t) row
            const uint4 cv = reinterpret_cast<const uint4*>(C + r * G * N + src)[k];
            const uint4 bv = reinterpret_cast<const uint4*>(B + r * G * N + src)[k];
            reinterpret_cast<uint4*>(Cer + j * slice_elems + (rr * H + h) * pw)[k] = cv;
            reinterpret_cast<uint4*>(Be + j * slice_elems + (r * H + h) * pw)[k] = bv;
        }
    }
}

// fp32 copies of dfinal ([N][P] and, per column slice, transposed [P][pw]) and
// of init_state transposed.  Either source may be NULL (then not written).
template <typename StateT>
__global__ void __launch_bounds__(256)
bwd_prep_states_kernel(const StateT* __restrict__ dfinal, const StateT* __restrict__ init,
                       float* __restrict__ dfin, float* __restrict__ dfinT, float* __restrict__ h0T,
                       int64_t BH, int P, int N, int pw, int64_t slice_elems) {
    const int64_t n_all = BH * N * P;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_all; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bh = i / ((int64_t)N * P);
        const int n = (int)((i / P) % N), p = (int)(i % P);
        const int j = n / pw, k = n % pw;
        const int64_t tr = j * slice_elems + (bh * P + p) * pw + k;
        if (dfinal) {
            const float v = to_f32(dfinal[i]);
            dfin[i] = v;
            dfinT[tr] = v;
        }
        if (init) h0T[tr] = to_f32(init[i]);
    }
}

// Weights and chunk-local log-decay cumsum of the time-reversed scans (R1, R2):
// reversed token tau < L has weight 1 and log-decay a_{L-tau} (0 at tau = 0);
// padding tokens tau >= L have both 0.  One block per (b, h, chunk), thread =
// token; also clears the scan's hand-off flags (a slice per block).
template <typename IoT>
__global__ void __launch_bounds__(256)
bwd_rev_decay_kernel(const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias, const float* __restrict__ A,
                     float* __restrict__ w_out, float* __restrict__ acs_out, int* __restrict__ flags, int64_t L,
                     int64_t Lpad, int H, int Q, int nchunks, int nflags) {
    __shared__ float warp_tot[8];
    const int c = (int)(blockIdx.x % (unsigned)nchunks);
    const int64_t bh = blockIdx.x / (unsigned)nchunks;
    const int h = (int)(bh % H);
    const int64_t b = bh / H;
    const int l = threadIdx.x, lane = l & 31, warp = l >> 5;
    const int64_t tau = (int64_t)c * Q + l;
    float v = 0.f;
    if (l < Q && tau >= 1 && tau < L) {
        const int64_t s = L - tau;
        const float dt = softplus_f32(to_f32(dt_raw[(b * L + s) * H + h]) + (dt_bias ? dt_bias[h] : 0.f));
        v = dt * A[h];
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    for (int w = 0; w < warp; ++w) v += warp_tot[w];
    if (l < Q) {
        w_out[bh * Lpad + tau] = tau < L ? 1.f : 0.f;
        acs_out[bh * Lpad + tau] = v;
    }
    const int per = (int)((nflags + gridDim.x - 1) / gridDim.x);
    const int f0 = (int)blockIdx.x * per;
    for (int i = f0 + l; i < nflags && i < f0 + per; i += blockDim.x) flags[i] = 0;
}

__global__ void bwd_clear_flags_kernel(int* __restrict__ flags, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) flags[i] = 0;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Everything local to one token row (b, t), one block per row: per head (a
// warp each) dx and the scalars x.dxu, C.(h dy) and x.dy; per (group, n) dB and
// dC summed over the group's heads.  The row's scan outputs (y1, y2, y3) are
// read once from HBM (y3 twice, the second time from L1/L2).  The scalars go
// out as tok[3][b*L][H].
template <typename IoT, typename GT>
__global__ void __launch_bounds__(256)
bwd_row_kernel(const IoT* __restrict__ x, const IoT* __restrict__ dy, const IoT* __restrict__ C,
               const float* __restrict__ D, const float* __restrict__ dtf, const float* __restrict__ y1,
               const float* __restrict__ y2, const float* __restrict__ y3, GT* __restrict__ dx, GT* __restrict__ dB,
               GT* __restrict__ dC, float* __restrict__ tok, int64_t batch, int64_t L, int64_t Lpad, int H, int P,
               int N, int G, int pw, int64_t slice_y) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int hpg = H / G;
    const int64_t rows = batch * L;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t b = r / L, t = r - b * L;
        const int64_t rr = b * L + (L - 1 - t);              // the row's index in reversed time
        for (int h = warp; h < H; h += nwarps) {
            const float dt = dtf[(b * H + h) * Lpad + t];
            const float dsk = D ? D[h] : 0.f;
            const int64_t row = r * H + h, rrow = rr * H + h;
            float xdxu = 0.f, xdy = 0.f, ydy = 0.f;
            for (int p = lane; p < P; p += 32) {
                const float xv = to_f32(x[row * P + p]), dyv = to_f32(dy[row * P + p]);
                const float dxu = y1[rrow * P + p];
                dx[row * P + p] = from_f32<GT>(dt * dxu + dsk * dyv);
                xdxu += xv * dxu;
                xdy += xv * dyv;
            }
            const IoT* Cg = C + (r * G + h / hpg) * N;
            for (int n = lane; n < N; n += 32) {
                const int j = n / pw;
                ydy += to_f32(Cg[n]) * y3[j * slice_y + row * pw + (n - j * pw)];
            }
            xdxu = warp_sum(xdxu);
            xdy = warp_sum(xdy);
            ydy = warp_sum(ydy);
            if (lane == 0) {
                tok[row] = xdxu;
                tok[rows * H + row] = ydy;
                tok[2 * rows * H + row] = xdy;
            }
        }
        for (int i = threadIdx.x; i < G * N; i += blockDim.x) {
            const int g = i / N, n = i - g * N, j = n / pw, k = n - j * pw;
            const float* y2r = y2 + j * slice_y + (rr * H + g * hpg) * pw + k;
            const float* y3r = y3 + j * slice_y + (r * H + g * hpg) * pw + k;
            const float* dtr = dtf + (b * H + g * hpg) * Lpad + t;
            float sb = 0.f, sc = 0.f;
#pragma unroll 8
            for (int q = 0; q < hpg; ++q) {
                sb += dtr[q * Lpad] * y2r[q * pw];
                sc += y3r[q * pw];
            }
            dB[r * G * N + i] = from_f32<GT>(sb);
            dC[r * G * N + i] = from_f32<GT>(sc);
        }
    }
}

// The same per-row work in 16-byte vectors for power-of-two headdim and dstate
// (P/4 and N/4 powers of two, P <= 128): all threads of the block load a whole
// row at once instead of a warp walking its heads one by one.  Per-head sums
// are shuffle reductions over segments of P/4 (or min(32, N/4)) lanes; dB and
// dC are summed over RSPLIT ranges of the group's heads, the partial sums
// meeting in shared memory in a fixed order (bitwise deterministic).
constexpr int ROW_THREADS = 256;

template <typename T> struct Io4;
template <> struct Io4<float> {
    __device__ __forceinline__ static void load(const float* p, float v[4]) {
        const float4 a = *reinterpret_cast<const float4*>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
    __device__ __forceinline__ static void store(float* p, const float v[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Io4<bf16> {
    __device__ __forceinline__ static void load(const bf16* p, float v[4]) {
        const uint2 a = *reinterpret_cast<const uint2*>(p);
        v[0] = __uint_as_float(a.x << 16); v[1] = __uint_as_float(a.x & 0xffff0000u);
        v[2] = __uint_as_float(a.y << 16); v[3] = __uint_as_float(a.y & 0xffff0000u);
    }
    __device__ __forceinline__ static void store(bf16* p, const float v[4]) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
        *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
};

__device__ __forceinline__ float seg_sum(float v, int width) {
    for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename IoT, typename GT>
__global__ void __launch_bounds__(ROW_THREADS)
bwd_row_vec_kernel(const IoT* __restrict__ x, const IoT* __restrict__ dy, const IoT* __restrict__ C,
                   const float* __restrict__ D, const float* __restrict__ dtf, const float* __restrict__ y1,
                   const float* __restrict__ y2, const float* __restrict__ y3, GT* __restrict__ dx,
                   GT* __restrict__ dB, GT* __restrict__ dC, float* __restrict__ tok, int64_t batch, int64_t L,
                   int64_t Lpad, int H, int P, int N, int G, int pw, int64_t slice_y) {
    __shared__ __align__(16) float part[2][ROW_THREADS * 4];   // dB, dC partial sums [split][column]
    const int tid = threadIdx.x;
    const int hpg = H / G;
    const int64_t rows = batch * L;
    const int SP = P >> 2;                                   // lanes per head, dx phase
    const int SN = (N >> 2) < 32 ? (N >> 2) : 32;            // lanes per head, C.(h dy) phase
    const int VN = (N >> 2) / SN;                            // 4-vectors per lane there
    const int ncol4 = (G * N) >> 2;                          // 4-vectors of a dB / dC row
    int rsplit = ROW_THREADS / ncol4;                        // head ranges summed apart
    if (rsplit < 1) rsplit = 1;
    if (rsplit > hpg) rsplit = hpg;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t b = r / L, t = r - b * L;
        const int64_t rr = b * L + (L - 1 - t);
        // dx, x.dxu, x.dy
        for (int h0 = 0; h0 < H; h0 += ROW_THREADS / SP) {
            const int h = h0 + tid / SP, p4 = tid % SP;
            float xdxu = 0.f, xdy = 0.f;
            if (h < H) {
                const int64_t row = r * H + h;
                const float dt = dtf[(b * H + h) * Lpad + t];
                const float dsk = D ? D[h] : 0.f;
                float xv[4], dyv[4], u[4], o[4];
                Io4<IoT>::load(x + row * P + 4 * p4, xv);
                Io4<IoT>::load(dy + row * P + 4 * p4, dyv);
                Io4<float>::load(y1 + (rr * H + h) * P + 4 * p4, u);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    o[e] = dt * u[e] + dsk * dyv[e];
                    xdxu += xv[e] * u[e];
                    xdy += xv[e] * dyv[e];
                }
                Io4<GT>::store(dx + row * P + 4 * p4, o);
            }
            xdxu = seg_sum(xdxu, SP);
            xdy = seg_sum(xdy, SP);
            if (h < H && p4 == 0) {
                tok[r * H + h] = xdxu;
                tok[2 * rows * H + r * H + h] = xdy;
            }
        }
        // C . (h dy)
        for (int h0 = 0; h0 < H; h0 += ROW_THREADS / SN) {
            const int h = h0 + tid / SN, l4 = tid % SN;
            float ydy = 0.f;
            if (h < H) {
                const IoT* Cg = C + (r * G + h / hpg) * N;
                for (int i = 0; i < VN; ++i) {
                    const int n = 4 * (l4 + SN * i), j = n / pw;
                    float cv[4], yv[4];
                    Io4<IoT>::load(Cg + n, cv);
                    Io4<float>::load(y3 + j * slice_y + (r * H + h) * pw + (n - j * pw), yv);
                    ydy += cv[0] * yv[0] + cv[1] * yv[1] + cv[2] * yv[2] + cv[3] * yv[3];
                }
            }
            ydy = seg_sum(ydy, SN);
            if (h < H && l4 == 0) tok[rows * H + r * H + h] = ydy;
        }
        // dB, dC: column vector c4 of the (g, n) row, head range sp
        for (int i = tid; i < ncol4 * rsplit; i += ROW_THREADS) {
            const int c4 = i % ncol4, sp = i / ncol4;
            const int g = (4 * c4) / N, n = 4 * c4 - g * N, j = n / pw, k = n - j * pw;
            const int q0 = (sp * hpg) / rsplit, q1 = ((sp + 1) * hpg) / rsplit;
            float sb[4] = {0.f, 0.f, 0.f, 0.f}, sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int q = q0; q < q1; ++q) {
                const int h = g * hpg + q;
                const float dt = dtf[(b * H + h) * Lpad + t];
                float v2[4], v3[4];
                Io4<float>::load(y2 + j * slice_y + (rr * H + h) * pw + k, v2);
                Io4<float>::load(y3 + j * slice_y + (r * H + h) * pw + k, v3);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sb[e] += dt * v2[e];
                    sc[e] += v3[e];
                }
            }
            if (rsplit == 1) {
                Io4<GT>::store(dB + r * G * N + 4 * c4, sb);
                Io4<GT>::store(dC + r * G * N + 4 * c4, sc);
            } else {
                Io4<float>::store(&part[0][4 * i], sb);
                Io4<float>::store(&part[1][4 * i], sc);
            }
        }
        if (rsplit > 1) {
            __syncthreads();
            for (int c = tid; c < 4 * ncol4; c += ROW_THREADS) {
                float vb = 0.f, vc = 0.f;
                for (int sp = 0; sp < rsplit; ++sp) {
                    vb += part[0][sp * 4 * ncol4 + c];
                    vc += part[1][sp * 4 * ncol4 + c];
                }
                dB[r * G * N + c] = from_f32<GT>(vb);
                dC[r * G * N + c] = from_f32<GT>(vc);
            }
            __syncthreads();
        }
    }
}

static bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// One block per (b, h): <dfinal, h_final>, d init_state, then the suffix sum
// of the log-decay gradient over the sequence (tiles of 256 tokens from the
// end), d dt_raw, and this sequence's shares of dA, d dt_bias and dD.
constexpr int DTB = 256;

template <typename IoT, typename GT, typename StateT>
__global__ void __launch_bounds__(DTB)
bwd_decay_kernel(const IoT* __restrict__ dt_raw, const float* __restrict__ dt_bias, const float* __restrict__ A,
                 const float* __restrict__ dtf, const float* __restrict__ tok, const float* __restrict__ dfin,
                 const float* __restrict__ hfT, const float* __restrict__ G0, GT* __restrict__ ddt_raw,
                 StateT* __restrict__ dinit, float* __restrict__ part, int64_t batch, int64_t L, int64_t Lpad,
                 int H, int P, int N, int pw, int64_t slice_st) {
    __shared__ float red[DTB / 32][3];
    __shared__ float s_hf;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int64_t b = bh / H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t BHL = batch * H * L;
    const float Ah = A[h];
    // <dfinal, h_final> (h_final^T arrives in column slices [P][pw]) and dinit
    const int64_t NP = (int64_t)N * P;
    float hf = 0.f;
    const float e0 = expf(dtf[bh * Lpad] * Ah);
    for (int64_t i = tid; i < NP; i += DTB) {
        const int n = (int)(i / P), p = (int)(i % P);
        if (dfin) hf += dfin[bh * NP + i] * hfT[(n / pw) * slice_st + (bh * P + p) * pw + n % pw];
        if (dinit) dinit[bh * NP + i] = from_f32<StateT>(e0 * G0[bh * NP + i]);
    }
    hf = warp_sum(hf);
    if (lane == 0) red[warp][0] = hf;
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < DTB / 32; ++w) s += red[w][0];
        s_hf = s;
    }
    __syncthreads();
    const float hfdot = s_hf;
    const float bias = dt_bias ? dt_bias[h] : 0.f;
    float carry = 0.f, sdA = 0.f, sdb = 0.f, sdD = 0.f;
    __shared__ float wtot[DTB / 32];
    for (int64_t end = L - 1; end >= 0; end -= DTB) {
        const int64_t t = end - tid;          // thread tid walks the tile backwards
        float dcum = 0.f, xdxu = 0.f, dt = 0.f, xdy = 0.f;
        if (t >= 0) {
            const int64_t row = (b * L + t) * H + h;
            xdxu = tok[row];
            xdy = tok[2 * BHL + row];
            dt = dtf[bh * Lpad + t];
            dcum = tok[BHL + row] - dt * xdxu + (t == L - 1 ? hfdot : 0.f);
        }
        // inclusive prefix over tid = suffix over t within the tile
        float v = dcum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += u;
        }
        if (lane == 31) wtot[warp] = v;
        __syncthreads();
        float before = 0.f, tile = 0.f;
        for (int w = 0; w < DTB / 32; ++w) {
            if (w < warp) before += wtot[w];
            tile += wtot[w];
        }
        __syncthreads();
        if (t >= 0) {
            const float da = carry + before + v;
            const float z = to_f32(dt_raw[(b * L + t) * H + h]) + bias;
            const float dz = (xdxu + Ah * da) / (1.f + expf(-z));
            ddt_raw[(b * L + t) * H + h] = from_f32<GT>(dz);
            sdA += dt * da;
            sdb += dz;
            sdD += xdy;
        }
        carry += tile;
    }
    sdA = warp_sum(sdA);
    sdb = warp_sum(sdb);
    sdD = warp_sum(sdD);
    if (lane == 0) { red[warp][0] = sdA; red[warp][1] = sdb; red[warp][2] = sdD; }
    __syncthreads();
    if (tid < 3) {
        float s = 0.f;
        for (int w = 0; w < DTB / 32; ++w) s += red[w][tid];
        part[bh * 3 + tid] = s;
    }
}

// dA, d dt_bias, dD: per head, the sequences' shares summed in batch order.
__global__ void bwd_params_kernel(const float* __restrict__ part, float* __restrict__ dA, float* __restrict__ ddt_bias,
                                  float* __restrict__ dD, int64_t batch, int H) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    float sa = 0.f, sb = 0.f, sd = 0.f;
    for (int64_t b = 0; b < batch; ++b) {
        sa += part[(b * H + h) * 3 + 0];
        sb += part[(b * H + h) * 3 + 1];
        sd += part[(b * H + h) * 3 + 2];
    }
    dA[h] = sa;
    if (ddt_bias) ddt_bias[h] = sb;
    if (dD) dD[h] = sd;
}

// ---------------------------------------------------------------- host side

cudaError_t launch_backward_params(const float* part, float* dA, float* ddt_bias, float* dD, int64_t nseg, int H,
                                   cudaStream_t s) {
    bwd_params_kernel<<<(unsigned)((H + 127) / 128), 128, 0, s>>>(part, dA, ddt_bias, dD, nseg, H);
    return cudaGetLastError();
}

static unsigned grid_for(int64_t work, int64_t per_block) {
    const int64_t g = (work + per_block - 1) / per_block;
    return (unsigned)(g < 1 ? 1 : (g > 148 * 16 ? 148 * 16 : g));
}

// What runs before a scan: the forward's dt / decay kernel (which also clears
// the hand-off flags), nothing (the reversed-decay kernel just did both), or
// only the flag clear (the weights and decays are already in the workspace).
enum ScanPrologue { kForwardDecay, kNone, kClearFlags };

// one scan with the forward's contract, run on the backward's workspace
static cudaError_t run_scan(const BackwardArgs& a, const BackwardLayout& l, bool transposed, bool reversed,
                            ScanPrologue pro, const void* xs, const void* Bs, const void* Cs, const void* init,
                            void* out, void* fin, cudaStream_t s) {
    PrefillArgs p{};
    p.batch = a.batch; p.L = a.L; p.H = a.H; p.Q = a.Q;
    p.P = transposed ? l.pw : a.P;
    p.N = transposed ? a.P : a.N;
    p.G = transposed ? a.H : a.G;
    p.io_bf16 = a.io_bf16; p.y_bf16 = false; p.state_bf16 = false;
    p.x = xs; p.B = Bs; p.C = Cs; p.D = nullptr;
    p.dt_raw = a.dt_raw; p.dt_bias = a.dt_bias; p.A = a.A;
    p.init_state = init; p.y = out; p.final_state = fin;
    p.ws = a.ws;
    p.lay.nchunks = l.nchunks;
    p.lay.Lpad = l.Lpad;
    p.lay.off_dt = reversed ? l.off_dtr : l.off_dtf;
    p.lay.off_acs = reversed ? l.off_acsr : l.off_acsf;
    p.lay.off_states = l.off_states;
    p.lay.off_flags = l.off_flags;
    p.lay.total = l.total;
    p.pad_left = nullptr;
    p.dev_err = a.dev_err;
    p.drop_publish = 0;
    cudaError_t e = cudaSuccess;
    if (pro == kForwardDecay) {
        e = launch_dt_cumsum(p, s);
    } else if (pro == kClearFlags) {
        const int nflags = (int)(a.batch * a.H + 64);
        bwd_clear_flags_kernel<<<grid_for(nflags, 256), 256, 0, s>>>((int*)(a.ws + l.off_flags), nflags);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    const bool tc = transposed ? l.tc_t : l.tc_main;
    return tc ? launch_prefill_tc(p, s) : launch_prefill_simt(p, s);
}

template <typename IoT, typename GT, typename StateT>
static cudaError_t backward_t(const BackwardArgs& a, cudaStream_t s) {
    const BackwardLayout& l = a.lay;
    char* ws = a.ws;
    const int64_t BH = a.batch * a.H;
    const int H = (int)a.H, P = (int)a.P, N = (int)a.N, G = (int)a.G, Q = (int)a.Q, pw = (int)l.pw;
    const int nblk = (int)l.nblk;
    const int64_t slice_io = (int64_t)(l.slice_io / sizeof(IoT));
    const int64_t slice_st = (int64_t)(l.slice_st / sizeof(float));
    const int64_t slice_y = (int64_t)(l.slice_y / sizeof(float));
    IoT* dyr = (IoT*)(ws + l.off_dyr);
    IoT* xr = (IoT*)(ws + l.off_xr);
    IoT* Cr = (IoT*)(ws + l.off_Cr);
    IoT* Br = (IoT*)(ws + l.off_Br);
    IoT* Cer = (IoT*)(ws + l.off_Cer);
    IoT* Be = (IoT*)(ws + l.off_Be);
    float* dfin = (float*)(ws + l.off_dfin);
    float* G0 = (float*)(ws + l.off_G0);
    float* dfinT = (float*)(ws + l.off_dfinT);
    float* h0T = (float*)(ws + l.off_h0T);
    float* hfT = (float*)(ws + l.off_hfT);
    float* y1 = (float*)(ws + l.off_y1);
    float* y2 = (float*)(ws + l.off_y2);
    float* y3 = (float*)(ws + l.off_y3);
    float* tok = (float*)(ws + l.off_tok);
    float* part = (float*)(ws + l.off_part);
    const bool has_dfin = a.dfinal != nullptr, has_init = a.init_state != nullptr;
    cudaError_t e;

    bwd_prep_tokens_kernel<IoT><<<grid_for(a.batch * a.L, 1), 256, 0, s>>>(
        (const IoT*)a.x, (const IoT*)a.dy, (const IoT*)a.B, (const IoT*)a.C, dyr, xr, Cr, Br, Cer, Be, a.batch, a.L,
        H, P, N, G, pw, nblk, slice_io);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (has_dfin || has_init) {
        bwd_prep_states_kernel<StateT><<<grid_for(BH * N * P, 256), 256, 0, s>>>(
            (const StateT*)a.dfinal, (const StateT*)a.init_state, dfin, dfinT, h0T, BH, P, N, pw, slice_st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // F: h^T scans (forward time), per column slice
    for (int j = 0; j < nblk; ++j) {
        e = run_scan(a, l, true, false, j == 0 ? kForwardDecay : kClearFlags, Be + j * slice_io, a.x, a.dy,
                     has_init ? h0T + j * slice_st : nullptr, y3 + j * slice_y,
                     has_dfin ? hfT + j * slice_st : nullptr, s);
        if (e != cudaSuccess) return e;
    }
    // R1: the state adjoint, reversed time
    {
        const int nflags = (int)(BH + 64);
        const unsigned threads = (unsigned)(Q < 32 ? 32 : Q);
        bwd_rev_decay_kernel<IoT><<<(unsigned)(BH * l.nchunks), threads, 0, s>>>(
            (const IoT*)a.dt_raw, a.dt_bias, a.A, (float*)(ws + l.off_dtr), (float*)(ws + l.off_acsr),
            (int*)(ws + l.off_flags), a.L, l.Lpad, H, Q, (int)l.nchunks, nflags);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        e = run_scan(a, l, false, true, kNone, dyr, Cr, Br, has_dfin ? dfin : nullptr, y1, a.dinit ? G0 : nullptr,
                     s);
        if (e != cudaSuccess) return e;
    }
    // R2: the transposed adjoint, reversed time, per column slice
    for (int j = 0; j < nblk; ++j) {
        e = run_scan(a, l, true, true, kClearFlags, Cer + j * slice_io, dyr, xr,
                     has_dfin ? dfinT + j * slice_st : nullptr, y2 + j * slice_y, nullptr, s);
        if (e != cudaSuccess) return e;
    }
    const float* dtf = (const float*)(ws + l.off_dtf);
    if (pow2(P / 4) && P <= 128 && pow2(N / 4))
        bwd_row_vec_kernel<IoT, GT><<<grid_for(a.batch * a.L, 1), ROW_THREADS, 0, s>>>(
            (const IoT*)a.x, (const IoT*)a.dy, (const IoT*)a.C, a.D, dtf, y1, y2, y3, (GT*)a.dx, (GT*)a.dB,
            (GT*)a.dC, tok, a.batch, a.L, l.Lpad, H, P, N, G, pw, slice_y);
    else
        bwd_row_kernel<IoT, GT><<<grid_for(a.batch * a.L, 1), 256, 0, s>>>(
            (const IoT*)a.x, (const IoT*)a.dy, (const IoT*)a.C, a.D, dtf, y1, y2, y3, (GT*)a.dx, (GT*)a.dB,
            (GT*)a.dC, tok, a.batch, a.L, l.Lpad, H, P, N, G, pw, slice_y);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_decay_kernel<IoT, GT, StateT><<<(unsigned)BH, DTB, 0, s>>>(
        (const IoT*)a.dt_raw, a.dt_bias, a.A, dtf, tok, has_dfin ? dfin : nullptr, hfT, G0, (GT*)a.ddt_raw,
        (StateT*)a.dinit, part, a.batch, a.L, l.Lpad, H, P, N, pw, slice_st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_params_kernel<<<(unsigned)((H + 127) / 128), 128, 0, s>>>(part, a.dA, a.ddt_bias, a.dD, a.batch, H);
    return cudaGetLastError();
}

template <typename IoT, typename GT>
static cudaError_t backward_s(const BackwardArgs& a, cudaStream_t s) {
    return a.state_bf16 ? backward_t<IoT, GT, bf16>(a, s) : backward_t<IoT, GT, float>(a, s);
}

template <typename IoT>
static cudaError_t backward_g(const BackwardArgs& a, cudaStream_t s) {
    return a.grad_bf16 ? backward_s<IoT, bf16>(a, s) : backward_s<IoT, float>(a, s);
}

// Empty sequences (seqlen 0): the parameter gradients are zero and the final
// state is the initial one, so d init_state = dfinal.
template <typename StateT>
__global__ void bwd_empty_kernel(const StateT* __restrict__ dfinal, StateT* __restrict__ dinit, int64_t n_state,
                                 float* __restrict__ dA, float* __restrict__ ddt_bias, float* __restrict__ dD,
                                 int H) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_state || i < H;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (dinit && i < n_state) dinit[i] = dfinal ? dfinal[i] : from_f32<StateT>(0.f);
        if (i < H) {
            dA[i] = 0.f;
            if (ddt_bias) ddt_bias[i] = 0.f;
            if (dD) dD[i] = 0.f;
        }
    }
}

cudaError_t launch_backward_empty(const BackwardArgs& a, cudaStream_t s) {
    const int64_t n = a.batch * a.H * a.N * a.P;
    const unsigned grid = grid_for(n > a.H ? n : a.H, 256);
    if (a.state_bf16)
        bwd_empty_kernel<bf16><<<grid, 256, 0, s>>>((const bf16*)a.dfinal, (bf16*)a.dinit, n, a.dA, a.ddt_bias, a.dD,
                                                    (int)a.H);
    else
        bwd_empty_kernel<float><<<grid, 256, 0, s>>>((const float*)a.dfinal, (float*)a.dinit, n, a.dA, a.ddt_bias,
                                                     a.dD, (int)a.H);
    return cudaGetLastError();
}

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s) {
    if (a.lay.mode == 1) return launch_backward_blocks_cc(a, s);
    if (a.lay.mode == 2) return launch_backward_tc(a, s);
    return a.io_bf16 ? backward_g<bf16>(a, s) : backward_g<float>(a, s);
}

int backward_launches(const BackwardLayout& l, bool has_states) {
    if (l.mode == 1) return 3;                 // state passes, blocks, parameter sums
    if (l.mode == 2) return 4;                 // state passes, blocks, dB / dC partial sums, parameter sums
    // a scan is one launch on the tensor-core path, three on the CUDA-core one;
    // prep tokens (+ prep states); F: dt_cumsum, nblk scans, nblk - 1 flag
    // clears; R1: decay kernel and scan; R2: nblk clears and nblk scans; then
    // three finishing kernels (rows, decay gradient, parameters)
    const int st = l.tc_t ? 1 : 3, sm = l.tc_main ? 1 : 3;
    return 1 + (has_states ? 1 : 0) + (int)(l.nblk * (st + 1)) + 1 + sm + (int)(l.nblk * (st + 1)) + 3;
}

}  // namespace ssd
