// Backward pass of the chunked prefill scan in block form on tensor cores
// (sm_100a), dstate 128 and headdim 64, bf16 inputs.
//
// The same block form as the CUDA-core backward (its derivation is in
// ssd_backward_blocks.cu): every gradient of a block of 128 tokens is a
// function of the block's tokens, the state entering the block (h0_j) and the
// adjoint of the state at its end from later blocks (Ge_j).  Three kernels:
//
//   1. bwd_states_tc_kernel   two sequential passes over every (b, h), forward
//      for h0_j and backward for Ge_j (and d init_state), the state in TMEM,
//      one tcgen05 rank-128 update per block; h0_j and Ge_j leave as bf16
//      pairs hi + lo, in the tile layout of kernel 2's operands;
//   2. bwd_main_tc_kernel     the block gradients, one head-block after the
//      other in a contiguous range of (b, block, group, head) per CTA: dx and
//      the log-decay gradient per head, dB and dC summed over the range's heads
//      of one (b, block, group) in TMEM and written as one partial per range;
//   3. bwd_reduce_dbc_kernel  sums the partials of every (b, block, group) in
//      range order (bitwise deterministic) into dB and dC; the parameter
//      gradients come from the per-block shares as in the CUDA-core form.
//
// Precision as in the forward's tensor-core kernels: every operand computed in
// a kernel (the weighted x and dy, the decay-weighted score matrices, the
// states and adjoints) is contracted as a bf16 pair hi + lo against an exact
// bf16 input, with fp32 accumulation.
#include "ssd_internal.h"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace bwdtc {
using namespace ::ssd::tc;

constexpr int NS = 128;              // dstate
constexpr int PD = 64;               // headdim

// bounded wait that gives up at once when another wait of the CTA has given up
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort) {
    uint32_t spins = 0;
    unsigned long long deadline = 0;
    while (!mbar_try_sleep(bar, parity, 100000u)) {
        if ((++spins & 3u) == 0) {
            if (*abort) return false;
            const unsigned long long now = gtimer();
            if (deadline == 0) {
                deadline = now + WAIT_NS;
            } else if (now > deadline) {
                *abort = 1;
                return false;
            }
        }
    }
    return true;
}

// 4 consecutive 32-bit TMEM columns of this warp's 32 lanes
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]) : "memory");
}

// ============================================================ 1. state passes
//
// Item = (direction, b, pair of heads of one group).  Forward: h <- 2^(R_last) h
// + B^T (w o X), w_s = dt_s 2^(R_last - R_s); backward: G <- 2^(R_last) G +
// C^T (2^R o dY).  R = block-local cumsum of dt A times log2(e) (double).  The
// value before each block's update is written out (h0_j, Ge_j).
namespace st {
constexpr int NCW = 8;                            // compute warps: head k = w / 4, lane quarter w % 4
constexpr int NCT = NCW * 32;
constexpr int THREADS = NCT + 32;                 // + the TMA / MMA warp
constexpr uint32_t STAGE = 4 * TILE;              // N-side tiles (n 0-63, 64-127), P-side tile per head
constexpr uint32_t OFF_W = 2 * STAGE;             // per head: (w o X) hi, lo
constexpr uint32_t OFF_TOT = OFF_W + 4 * TILE;    // [2 heads][4 quarters] double: warp totals of the scan
constexpr uint32_t OFF_BAR = OFF_TOT + 2 * 4 * 8;
enum { B_FULL0, B_FULL1, B_WX, B_MMA, NBAR };
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr uint32_t SMEM = OFF_MISC + 16;
static_assert(SMEM <= 232448, "shared memory per CTA");

struct Params {
    const void* dt_raw;        // bf16 [b][L][H]
    const float* dt_bias;      // [H] or NULL
    const float* A;            // [H]
    const void* init_state;    // state dtype [b*H][N][P] or NULL
    const void* dfinal;        // state dtype [b*H][N][P] or NULL
    uint16_t* h0;              // bf16 [b*H][nblk][N][2][P]
    uint16_t* ge;              // bf16 [b*H][nblk][N][2][P]
    void* dinit;               // state dtype [b*H][N][P] or NULL
    unsigned* dev_err;
    long long L;
    int H, G, nblk, npairs, state_bf16;
};
}  // namespace st

__global__ void __launch_bounds__(st::THREADS, 1)
bwd_states_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmDY,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                     const st::Params p) {
    using namespace st;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t base = smem_u32(sm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
    auto bar = [&](int i) -> uint32_t { return base + OFF_BAR + 8u * (uint32_t)i; };
    if (base & 1023u) {
        if (threadIdx.x == 0) atomicOr(p.dev_err, kErrAsyncTimeout);
        return;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;"
                     ::"r"(base + OFF_MISC) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (threadIdx.x == NCT) {
        const uint32_t cnt[NBAR] = {1, 1, NCT, 1};
        for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), cnt[i]);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_MISC);

    const int item = (int)blockIdx.x;
    const bool rev = item >= p.npairs;
    const int pr = rev ? item - p.npairs : item;
    const int hpg = p.H / p.G;
    const int bg = pr / (hpg >> 1);
    const int g = bg % p.G, b = bg / p.G;
    const int h0 = g * hpg + 2 * (pr % (hpg >> 1));
    const int nblk = p.nblk;
    auto blk_of = [&](int i) { return rev ? nblk - 1 - i : i; };
    unsigned err = 0;
    auto wait = [&](int i, uint32_t ph) {
        if (!wait_or_abort(bar(i), ph, s_abort)) err |= kErrAsyncTimeout;
    };

    if (warp == NCW) {
        // ======================================================== TMA and MMA
        const uint32_t lead = elect_one();
        const CUtensorMap* tmN = rev ? &tmC : &tmB;
        const CUtensorMap* tmP = rev ? &tmDY : &tmX;
        auto load = [&](int i) {
            const int t0 = blk_of(i) * SUB;
            const uint32_t stg = base + (uint32_t)(i & 1) * STAGE, bb = bar(B_FULL0 + (i & 1));
            mbar_expect_tx(bb, 4 * TILE);
            tma_load_4d(stg, tmN, 0, g, t0, b, bb);
            tma_load_4d(stg + TILE, tmN, 64, g, t0, b, bb);
            tma_load_4d(stg + 2 * TILE, tmP, 0, h0, t0, b, bb);
            tma_load_4d(stg + 3 * TILE, tmP, 0, h0 + 1, t0, b, bb);
        };
        if (lead) {
            load(0);
            if (nblk > 1) load(1);
        }
        __syncwarp();
        constexpr uint32_t ID = idesc_bf16(128, PD, true, true);   // N-side^T (MN-major) x w o P-side (MN-major)
        constexpr uint32_t KSTEP_MN = 2048 >> 4;
        for (int i = 0; i < nblk; ++i) {
            const uint32_t stg = base + (uint32_t)(i & 1) * STAGE;
            wait(B_WX, i & 1);               // states scaled, w o X written (implies the tiles landed)
            tc_fence_after();
            const uint64_t dN = sdesc(stg, TILE, 1024);
            const bool go = lead && !*s_abort;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint64_t dWh = sdesc(base + OFF_W + 2 * k * TILE, TILE, 1024);
                const uint64_t dWl = sdesc(base + OFF_W + (2 * k + 1) * TILE, TILE, 1024);
#pragma unroll
                for (int kk = 0; kk < SUB / 16; ++kk) {
                    if (go) mma_ss<ID, 1>(tmem + 64 * k, dN + kk * KSTEP_MN, dWh + kk * KSTEP_MN);
                    if (go) mma_ss<ID, 1>(tmem + 64 * k, dN + kk * KSTEP_MN, dWl + kk * KSTEP_MN);
                }
            }
            if (go) mma_commit(bar(B_MMA));
            __syncwarp();
            wait(B_MMA, i & 1);              // the stage and the w o X tiles are free again
            if (lead && i + 2 < nblk && !*s_abort) load(i + 2);
            __syncwarp();
        }
    } else {
        // ======================================================== compute warps
        const int k = warp >> 2, q = warp & 3;
        const int row = 32 * q + lane;               // state row n, and token s of the block
        const uint32_t lo16 = (uint32_t)(32 * q) << 16;
        const int h = h0 + k;
        const long long bh = (long long)b * p.H + h;
        const float Ah = p.A[h], bias = p.dt_bias ? p.dt_bias[h] : 0.f;
        double* s_tot = reinterpret_cast<double*>(sm + OFF_TOT);
        const uint16_t* dtr = reinterpret_cast<const uint16_t*>(p.dt_raw);
        // the starting value of the pass: init_state (forward) or dfinal (backward), else 0
        {
            const void* src = rev ? p.dfinal : p.init_state;
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float f = 0.f;
                    if (src) {
                        const long long o = (bh * NS + row) * PD + 32 * c + e;
                        f = p.state_bf16 ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(src)[o] << 16)
                                         : reinterpret_cast<const float*>(src)[o];
                    }
                    v[e] = __float_as_uint(f);
                }
                tmem_st32(tmem + lo16 + 64 * k + 32 * c, v);
            }
            tmem_wait_st();
        }
        uint16_t* out = rev ? p.ge : p.h0;
        for (int i = 0; i < nblk; ++i) {
            const int j = blk_of(i);
            const long long t = (long long)j * SUB + row;
            // dt and the block-local cumsum of dt A log2(e) (double), token s = row
            float dt = 0.f;
            if (t < p.L) dt = softplus_f32(__uint_as_float((uint32_t)dtr[(b * p.L + t) * p.H + h] << 16) + bias);
            double v = (double)(dt * Ah) * (double)LOG2E;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double w = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += w;
            }
            if (lane == 31) s_tot[k * 4 + q] = v;
            asm volatile("bar.sync %0, %1;" ::"r"(1 + k), "r"(128) : "memory");
            double off = 0.0, tot = 0.0;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const double tw = s_tot[k * 4 + w];
                if (w < q) off += tw;
                tot += tw;
            }
            asm volatile("bar.sync %0, %1;" ::"r"(1 + k), "r"(128) : "memory");   // totals read before reuse
            const double R = v + off;
            const float wgt = rev ? ex2((float)R) : dt * ex2((float)(tot - R));
            const float scale = ex2((float)tot);
            // the previous block's update is complete: write the value out, scale it
            if (i > 0) wait(B_MMA, (i - 1) & 1);
            tc_fence_after();
            {
                uint16_t* o = out + ((bh * nblk + j) * NS + row) * (2 * PD);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t sv[32];
                    tmem_ld32(tmem + lo16 + 64 * k + 32 * c, sv);
                    tmem_wait_ld();
                    uint32_t hw[16], lw[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float a = __uint_as_float(sv[2 * e]), bb = __uint_as_float(sv[2 * e + 1]);
                        hw[e] = pack_bf16(a, bb);
                        lw[e] = pack_bf16(a - bf16_lo(hw[e]), bb - bf16_hi(hw[e]));
                        sv[2 * e] = __float_as_uint(a * scale);
                        sv[2 * e + 1] = __float_as_uint(bb * scale);
                    }
                    uint4* oh = reinterpret_cast<uint4*>(o + 32 * c);
                    uint4* ol = reinterpret_cast<uint4*>(o + PD + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        oh[e] = make_uint4(hw[4 * e], hw[4 * e + 1], hw[4 * e + 2], hw[4 * e + 3]);
                        ol[e] = make_uint4(lw[4 * e], lw[4 * e + 1], lw[4 * e + 2], lw[4 * e + 3]);
                    }
                    tmem_st32(tmem + lo16 + 64 * k + 32 * c, sv);
                }
                tmem_wait_st();
            }
            // w o (x or dy) of token `row`, as hi and lo tiles (MN-major B operand)
            wait(B_FULL0 + (i & 1), (i >> 1) & 1);
            {
                const uint8_t* src = sm + (i & 1) * STAGE + (2 + k) * TILE;
                uint8_t* dh = sm + OFF_W + 2 * k * TILE;
                uint8_t* dl = dh + TILE;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t so = swz(row, c);
                    const uint4 raw = *reinterpret_cast<const uint4*>(src + so);
                    const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a = bf16_lo(wv[e]) * wgt, bb = bf16_hi(wv[e]) * wgt;
                        hw[e] = pack_bf16(a, bb);
                        lw[e] = pack_bf16(a - bf16_lo(hw[e]), bb - bf16_hi(hw[e]));
                    }
                    *reinterpret_cast<uint4*>(dh + so) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4*>(dl + so) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(bar(B_WX));
        }
        // the value after the whole sequence: d init_state (backward pass)
        wait(B_MMA, (nblk - 1) & 1);
        tc_fence_after();
        if (rev && p.dinit) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t sv[32];
                tmem_ld32(tmem + lo16 + 64 * k + 32 * c, sv);
                tmem_wait_ld();
                const long long o = (bh * NS + row) * PD + 32 * c;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float f = __uint_as_float(sv[e]);
                    if (p.state_bf16) reinterpret_cast<bf16*>(p.dinit)[o + e] = __float2bfloat16_rn(f);
                    else reinterpret_cast<float*>(p.dinit)[o + e] = f;
                }
            }
        }
    }
    if (err) atomicOr(p.dev_err, err);
    tc_fence_before();
    __syncthreads();
    if (*s_abort) {
        // a wait gave up: let copies and MMAs still in flight land before TMEM is freed
        const unsigned long long t0 = gtimer();
        while (gtimer() - t0 < 1000000ull) {
        }
    }
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem) : "memory");
}


// ============================================================ 2. block gradients
//
// Unit u = ((b * nblk + j) * G + g) * hpg + q: head g*hpg + q of block j of
// batch element b.  CTA c takes units [c U / grid, (c + 1) U / grid); a run of
// its units with the same (b, j, g) is a segment, whose dB and dC accumulate in
// TMEM over the segment's heads and leave as one partial.  Per unit (rows s or
// l are the block's tokens, 128 TMEM lanes):
//
//   M1  S^T = B C^T                           -> TMEM S
//   M2  X dY^T                                -> TMEM X
//   C1  (w o X), (2^R o dY) as hi/lo tiles; x.dy; <Ge, h0> shares
//   M3  dB += (w o X) Ge^T, dC += (2^R o dY) h0^T     (hi.hi + hi.lo + lo.hi)
//   C2  transform: Mt = S^T e (in TMEM S as bf16 hi|lo), dS^T = dt_s e X dY^T
//       (hi/lo tiles), e = 2^(R_l - R_s) [l >= s]; column and row sums of S dS
//   M4  B Ge -> TMEM X[0:64], C h0 -> TMEM X[64:128]
//   M5  dB += dS^T C, dC += dS B
//   C3  u_l = 2^(R_l) dy_l . (C h0)_l, v_s = w_s x_s . (B Ge)_s
//   M6  Mt dY -> TMEM X[64:128]
//   C4  dxu = Mt dY + 2^(R_last - R_s) B Ge; dx; x . dxu; then d a, d dt_raw and
//       the unit's shares of dA, d dt_bias, dD
//   end of segment: TMEM dB, dC -> partial slot
namespace mn {
constexpr int NCW = 16;
constexpr int NCT = NCW * 32;
constexpr int WARP_MMA = NCW, WARP_TMA = NCW + 1;
constexpr int THREADS = NCT + 64;
constexpr uint32_t COL_S = 0, COL_X = 128, COL_DB = 256, COL_DC = 384;
constexpr uint32_t OFF_B = 0;                    // B tiles: n 0-63, n 64-127 (rows = tokens)
constexpr uint32_t OFF_C = 2 * TILE;             // C tiles
constexpr uint32_t OFF_X = 4 * TILE;             // x tile (rows = tokens, 64 p)
constexpr uint32_t OFF_DY = 5 * TILE;            // dy tile
constexpr uint32_t OFF_H0 = 6 * TILE;            // h0 hi, lo (rows = n, 64 p)
constexpr uint32_t OFF_GE = 8 * TILE;            // Ge hi, lo
constexpr uint32_t OFF_WD = 10 * TILE;           // (w o X) hi, lo, (2^R o dY) hi, lo; later dS^T
                                                 // hi (l 0-63, 64-127), lo (l 0-63, 64-127); then scratch
constexpr uint32_t OFF_RT = 14 * TILE;           // float2 [128]: R (hi, lo) of the block's tokens
constexpr uint32_t OFF_TOT = OFF_RT + 128 * 8;   // double [4]: scan totals of the lane quarters
constexpr uint32_t OFF_BAR = OFF_TOT + 4 * 8;
enum { F_BC, F_X, F_DY, F_HG, M_SX, C_WE, M_WE, C_T, M_BC, C_U, M_DX, C_E, C_FL, NBAR };
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr uint32_t SMEM = OFF_MISC + 16;
static_assert(SMEM <= 232448, "shared memory per CTA");
// scratch in the OFF_WD region once dS^T is consumed: floats
constexpr int SC_C = 0, SC_R = 512, SC_U = 1024, SC_V = 1536, SC_XDY = 2048, SC_XDXU = 2560, SC_K = 3072;

struct Params {
    const void* x;             // bf16 [b][L][H][P]
    const void* dy;            // bf16 [b][L][H][P]
    const void* dt_raw;        // bf16 [b][L][H]
    const float* dt_bias;      // [H] or NULL
    const float* A;            // [H]
    const float* D;            // [H] or NULL
    void* dx;                  // grad dtype [b][L][H][P]
    void* ddt_raw;             // grad dtype [b][L][H]
    float* part;               // [b * nblk][H][3]
    float* dbc;                // [grid * smax][2][128][128] partial dB, dC
    unsigned* dev_err;
    long long L, U;
    int H, G, nblk, smax, grad_bf16;
};
}  // namespace mn

__global__ void __launch_bounds__(mn::THREADS, 1)
bwd_main_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmDY,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmH0, const __grid_constant__ CUtensorMap tmGE,
                   const mn::Params p) {
    using namespace mn;
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t base = smem_u32(sm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
    auto bar = [&](int i) -> uint32_t { return base + OFF_BAR + 8u * (uint32_t)i; };
    if (base & 1023u) {
        if (threadIdx.x == 0) atomicOr(p.dev_err, kErrAsyncTimeout);
        return;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;"
                     ::"r"(base + OFF_MISC) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (threadIdx.x == NCT) {
        //                          BC X  DY HG SX WE   MWE T    MBC U    MDX E    FL
        const uint32_t cnt[NBAR] = {1, 1, 1, 1, 1, NCT, 1, NCT, 1, NCT, 1, NCT, NCT};
        for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), cnt[i]);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_MISC);

    const int hpg = p.H / p.G;
    const long long u0 = (long long)blockIdx.x * p.U / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * p.U / gridDim.x;
    const int nu = (int)(u1 - u0);
    struct Unit { int b, j, g, h; long long seg; bool first, last; };
    auto unit = [&](int i) -> Unit {
        const long long u = u0 + i;
        Unit d;
        d.seg = u / hpg;
        d.h = (int)(d.seg % p.G) * hpg + (int)(u % hpg);
        d.g = (int)(d.seg % p.G);
        d.j = (int)((d.seg / p.G) % p.nblk);
        d.b = (int)(d.seg / p.G / p.nblk);
        d.first = i == 0 || u % hpg == 0;
        d.last = i == nu - 1 || (u + 1) % hpg == 0;
        return d;
    };
    const long long seg0 = u0 / hpg;
    unsigned err = 0;
    auto wait = [&](int i, uint32_t ph) {
        if (!wait_or_abort(bar(i), ph, s_abort)) err |= kErrAsyncTimeout;
    };

    if (warp == WARP_TMA) {
        // ======================================================== TMA producer
        const uint32_t lead = elect_one();
        int nseg = 0;
        for (int i = 0; i < nu; ++i) {
            const Unit d = unit(i);
            const int t0 = d.j * SUB;
            const long long un = ((long long)d.b * p.H + d.h) * p.nblk + d.j;   // state unit (b, h, j)
            if (d.first) {
                if (i > 0) wait(M_DX, (i - 1) & 1);     // the previous segment's last dS MMAs are done
                if (lead && !*s_abort) {
                    mbar_expect_tx(bar(F_BC), 4 * TILE);
                    tma_load_4d(base + OFF_B, &tmB, 0, d.g, t0, d.b, bar(F_BC));
                    tma_load_4d(base + OFF_B + TILE, &tmB, 64, d.g, t0, d.b, bar(F_BC));
                    tma_load_4d(base + OFF_C, &tmC, 0, d.g, t0, d.b, bar(F_BC));
                    tma_load_4d(base + OFF_C + TILE, &tmC, 64, d.g, t0, d.b, bar(F_BC));
                }
                ++nseg;
            }
            // x: read by M2 and C1 of the previous unit
            if (i > 0) { wait(M_SX, (i - 1) & 1); wait(C_WE, (i - 1) & 1); }
            if (lead && !*s_abort) {
                mbar_expect_tx(bar(F_X), TILE);
                tma_load_4d(base + OFF_X, &tmX, 0, d.h, t0, d.b, bar(F_X));
            }
            // h0, Ge: read by M3, M4 (and C1) of the previous unit
            if (i > 0) wait(M_BC, (i - 1) & 1);
            if (lead && !*s_abort) {
                mbar_expect_tx(bar(F_HG), 4 * TILE);
                tma_load_4d(base + OFF_H0, &tmH0, 0, 0, 0, (int)un, bar(F_HG));
                tma_load_4d(base + OFF_H0 + TILE, &tmH0, 0, 1, 0, (int)un, bar(F_HG));
                tma_load_4d(base + OFF_GE, &tmGE, 0, 0, 0, (int)un, bar(F_HG));
                tma_load_4d(base + OFF_GE + TILE, &tmGE, 0, 1, 0, (int)un, bar(F_HG));
            }
            // dy: read by M2, C1, C3 and M6 of the previous unit
            if (i > 0) { wait(M_DX, (i - 1) & 1); wait(C_U, (i - 1) & 1); }
            if (lead && !*s_abort) {
                mbar_expect_tx(bar(F_DY), TILE);
                tma_load_4d(base + OFF_DY, &tmDY, 0, d.h, t0, d.b, bar(F_DY));
            }
            __syncwarp();
        }
        (void)nseg;
    } else if (warp == WARP_MMA) {
        // ======================================================== MMA issue
        const uint32_t lead0 = elect_one();
        constexpr uint32_t ID_SS = idesc_bf16(128, 128, false, false);     // K-major x K-major, N = 128
        constexpr uint32_t ID_XD = idesc_bf16(128, 128, false, false);     // X (K-major) x dY^T (K-major)
        constexpr uint32_t ID_KN = idesc_bf16(128, 128, false, false);     // (w o X) x Ge^T: both K-major over p
        constexpr uint32_t ID_P64 = idesc_bf16(128, PD, false, true);      // K-major x MN-major, N = 64
        constexpr uint32_t ID_DB = idesc_bf16(128, 128, false, true);      // dS^T (K-major) x C (MN-major)
        constexpr uint32_t ID_DC = idesc_bf16(128, 128, true, true);       // dS (MN-major) x B (MN-major)
        constexpr uint32_t ID_MT = idesc_bf16(128, PD, false, true);       // Mt (TMEM) x dY (MN-major)
        constexpr uint32_t KSTEP_K = 2, KBLOCK_K = TILE >> 4, KSTEP_MN = 2048 >> 4;
        int nseg = 0;
        for (int i = 0; i < nu; ++i) {
            const Unit d = unit(i);
            const uint32_t ph = i & 1;
            const uint32_t lead = lead0 && !*s_abort;
            if (d.first) {
                wait(F_BC, nseg & 1);
                ++nseg;
            }
            wait(F_X, ph);
            wait(F_DY, ph);
            if (i > 0) { wait(M_DX, ph ^ 1u); wait(C_E, ph ^ 1u); }   // TMEM S and X free
            tc_fence_after();
            __syncwarp();
            // M1: S^T = B C^T (K = n, 8 steps); M2: X dY^T (K = p, 4 steps)
            {
                const uint64_t dB = sdesc(base + OFF_B, 16, 1024), dC = sdesc(base + OFF_C, 16, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                    if (k == 0) { if (lead) mma_ss<ID_SS, 0>(tmem + COL_S, dB + o, dC + o);
                    } else if (lead) mma_ss<ID_SS, 1>(tmem + COL_S, dB + o, dC + o);
                }
                const uint64_t dX = sdesc(base + OFF_X, 16, 1024), dY = sdesc(base + OFF_DY, 16, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t o = (uint32_t)k * KSTEP_K;
                    if (k == 0) { if (lead) mma_ss<ID_XD, 0>(tmem + COL_X, dX + o, dY + o);
                    } else if (lead) mma_ss<ID_XD, 1>(tmem + COL_X, dX + o, dY + o);
                }
                if (lead) mma_commit(bar(M_SX));
            }
            // M3: dB += (w o X) Ge^T, dC += (2^R o dY) h0^T (K = p, 4 steps; hi.hi, hi.lo, lo.hi)
            wait(C_WE, ph);
            wait(F_HG, ph);
            if (d.first && nseg > 1) wait(C_FL, (nseg - 2) & 1);     // the previous partial is out
            tc_fence_after();
            __syncwarp();
            {
                const uint64_t wh = sdesc(base + OFF_WD, 16, 1024), wl = sdesc(base + OFF_WD + TILE, 16, 1024);
                const uint64_t eh = sdesc(base + OFF_WD + 2 * TILE, 16, 1024);
                const uint64_t el = sdesc(base + OFF_WD + 3 * TILE, 16, 1024);
                const uint64_t gh = sdesc(base + OFF_GE, 16, 1024), gl = sdesc(base + OFF_GE + TILE, 16, 1024);
                const uint64_t hh = sdesc(base + OFF_H0, 16, 1024), hl = sdesc(base + OFF_H0 + TILE, 16, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t o = (uint32_t)k * KSTEP_K;
                    if (k == 0 && d.first) {
                        if (lead) mma_ss<ID_KN, 0>(tmem + COL_DB, wh + o, gh + o);
                        if (lead) mma_ss<ID_KN, 0>(tmem + COL_DC, eh + o, hh + o);
                    } else {
                        if (lead) mma_ss<ID_KN, 1>(tmem + COL_DB, wh + o, gh + o);
                        if (lead) mma_ss<ID_KN, 1>(tmem + COL_DC, eh + o, hh + o);
                    }
                    if (lead) mma_ss<ID_KN, 1>(tmem + COL_DB, wh + o, gl + o);
                    if (lead) mma_ss<ID_KN, 1>(tmem + COL_DB, wl + o, gh + o);
                    if (lead) mma_ss<ID_KN, 1>(tmem + COL_DC, eh + o, hl + o);
                    if (lead) mma_ss<ID_KN, 1>(tmem + COL_DC, el + o, hh + o);
                }
                if (lead) mma_commit(bar(M_WE));
            }
            // M4: B Ge -> X[0:64], C h0 -> X[64:128] (K = n, 8 steps; Ge, h0 MN-major, hi + lo)
            wait(C_T, ph);
            tc_fence_after();
            __syncwarp();
            {
                const uint64_t dB = sdesc(base + OFF_B, 16, 1024), dC = sdesc(base + OFF_C, 16, 1024);
                const uint64_t gh = sdesc(base + OFF_GE, TILE, 1024), gl = sdesc(base + OFF_GE + TILE, TILE, 1024);
                const uint64_t hh = sdesc(base + OFF_H0, TILE, 1024), hl = sdesc(base + OFF_H0 + TILE, TILE, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                    if (k == 0) {
                        if (lead) mma_ss<ID_P64, 0>(tmem + COL_X, dB + o, gh);
                        if (lead) mma_ss<ID_P64, 0>(tmem + COL_X + 64, dC + o, hh);
                    } else {
                        if (lead) mma_ss<ID_P64, 1>(tmem + COL_X, dB + o, gh + k * KSTEP_MN);
                        if (lead) mma_ss<ID_P64, 1>(tmem + COL_X + 64, dC + o, hh + k * KSTEP_MN);
                    }
                    if (lead) mma_ss<ID_P64, 1>(tmem + COL_X, dB + o, gl + k * KSTEP_MN);
                    if (lead) mma_ss<ID_P64, 1>(tmem + COL_X + 64, dC + o, hl + k * KSTEP_MN);
                }
                if (lead) mma_commit(bar(M_BC));
            }
            // M5: dB += dS^T C (K = l), dC += dS B (K = s); dS^T hi/lo tiles in OFF_WD
            {
                const uint64_t dCm = sdesc(base + OFF_C, TILE, 1024), dBm = sdesc(base + OFF_B, TILE, 1024);
#pragma unroll
                for (int hl = 0; hl < 2; ++hl) {
                    const uint32_t ds = base + OFF_WD + 2 * hl * TILE;
                    const uint64_t aK = sdesc(ds, 16, 1024);       // dS^T as K-major A (rows s, K = l)
                    const uint64_t aM = sdesc(ds, TILE, 1024);     // dS as MN-major A (M = l, K = s rows)
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                        if (lead) mma_ss<ID_DB, 1>(tmem + COL_DB, aK + o, dCm + k * KSTEP_MN);
                        if (lead) mma_ss<ID_DC, 1>(tmem + COL_DC, aM + k * KSTEP_MN, dBm + k * KSTEP_MN);
                    }
                }
            }
            // M6: Mt dY -> X[64:128] (A = Mt hi|lo from TMEM S, K = l)
            wait(C_U, ph);
            tc_fence_after();
            __syncwarp();
            {
                const uint64_t dYm = sdesc(base + OFF_DY, TILE, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (k == 0) { if (lead) mma_ts<ID_MT, 0>(tmem + COL_X + 64, tmem + COL_S, dYm);
                    } else if (lead) mma_ts<ID_MT, 1>(tmem + COL_X + 64, tmem + COL_S + 16 * k, dYm + k * KSTEP_MN);
                    if (lead) mma_ts<ID_MT, 1>(tmem + COL_X + 64, tmem + COL_S + 16 * k + 8, dYm + k * KSTEP_MN);
                }
                if (lead) mma_commit(bar(M_DX));
            }
            __syncwarp();
        }
    } else {
        // ======================================================== compute warps
        const int q = warp & 3, c = warp >> 2;          // lane quarter, column quarter
        const int row = 32 * q + lane;                  // token s (or l) of the block, TMEM lane
        const uint32_t lo16 = (uint32_t)(32 * q) << 16;
        float2* s_rt = reinterpret_cast<float2*>(sm + OFF_RT);
        double* s_tot = reinterpret_cast<double*>(sm + OFF_TOT);
        float* scr = reinterpret_cast<float*>(sm + OFF_WD);
        const uint16_t* dtr = reinterpret_cast<const uint16_t*>(p.dt_raw);
        const uint16_t* xg = reinterpret_cast<const uint16_t*>(p.x);
        const uint16_t* dyg = reinterpret_cast<const uint16_t*>(p.dy);
        auto csync = [&]() { asm volatile("bar.sync 1, %0;" ::"r"(NCT) : "memory"); };
        int nseg = 0;
        float dtr_next = 0.f;
        auto fetch_dtr = [&](int i) -> float {
            const Unit d = unit(i);
            const long long t = (long long)d.j * SUB + row;
            return t < p.L ? __uint_as_float((uint32_t)dtr[((long long)d.b * p.L + t) * p.H + d.h] << 16) : 0.f;
        };
        if (nu > 0) dtr_next = fetch_dtr(0);
        for (int i = 0; i < nu; ++i) {
            const Unit d = unit(i);
            const uint32_t ph = i & 1;
            if (d.first) ++nseg;
            const long long t = (long long)d.j * SUB + row;
            const bool valid = t < p.L;
            const float Ah = p.A[d.h], bias = p.dt_bias ? p.dt_bias[d.h] : 0.f;
            const float z = dtr_next + bias;
            const float dt = valid ? softplus_f32(z) : 0.f;
            if (i + 1 < nu) dtr_next = fetch_dtr(i + 1);
            // ---- P1: block-local cumsum R of dt A log2(e) (double), per token
            double v = (double)(dt * Ah) * (double)LOG2E;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double w = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += w;
            }
            if (c == 0 && lane == 31) s_tot[q] = v;
            csync();
            double off = 0.0, tot = 0.0;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const double tw = s_tot[w];
                if (w < q) off += tw;
                tot += tw;
            }
            const double R = v + off;
            const float Rhi = (float)R, Rlo = (float)(R - (double)Rhi);
            const float wt = ex2((float)(tot - R));        // 2^(R_last - R_s)
            const float er = ex2(Rhi + Rlo);               // 2^(R_s)
            const float wv = dt * wt;                      // w_s
            if (c == 0) s_rt[row] = make_float2(Rhi, Rlo);
            // ---- C1: (w o X), (2^R o dY) hi/lo; x . dy; <Ge, h0>
            wait(F_X, ph);
            wait(F_DY, ph);
            if (i > 0) wait(M_DX, ph ^ 1u);                 // the previous dS^T (and scratch) are consumed
            csync();                                        // ... and every thread is past its scratch reads
            float xdy = 0.f;
            {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int ch = 2 * c + cc;              // 16-byte chunk of the 128-byte row
                    const uint32_t so = swz(row, ch);
                    const uint4 xr = *reinterpret_cast<const uint4*>(sm + OFF_X + so);
                    const uint4 yr = *reinterpret_cast<const uint4*>(sm + OFF_DY + so);
                    const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w}, yw[4] = {yr.x, yr.y, yr.z, yr.w};
                    uint32_t ah[4], al[4], bh[4], bl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = bf16_lo(xw[e]), x1 = bf16_hi(xw[e]);
                        const float y0 = bf16_lo(yw[e]), y1 = bf16_hi(yw[e]);
                        xdy = fmaf(x0, y0, fmaf(x1, y1, xdy));
                        const float a0 = wv * x0, a1 = wv * x1, b0 = er * y0, b1 = er * y1;
                        ah[e] = pack_bf16(a0, a1);
                        al[e] = pack_bf16(a0 - bf16_lo(ah[e]), a1 - bf16_hi(ah[e]));
                        bh[e] = pack_bf16(b0, b1);
                        bl[e] = pack_bf16(b0 - bf16_lo(bh[e]), b1 - bf16_hi(bh[e]));
                    }
                    *reinterpret_cast<uint4*>(sm + OFF_WD + so) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + TILE + so) = make_uint4(al[0], al[1], al[2], al[3]);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + 2 * TILE + so) = make_uint4(bh[0], bh[1], bh[2], bh[3]);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + 3 * TILE + so) = make_uint4(bl[0], bl[1], bl[2], bl[3]);
                }
            }
            wait(F_HG, ph);
            float kp = 0.f;                                  // share of <Ge, h0>: row n = row, 16 columns
            {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t so = swz(row, 2 * c + cc);
                    const uint4 gh = *reinterpret_cast<const uint4*>(sm + OFF_GE + so);
                    const uint4 gl = *reinterpret_cast<const uint4*>(sm + OFF_GE + TILE + so);
                    const uint4 hh = *reinterpret_cast<const uint4*>(sm + OFF_H0 + so);
                    const uint4 hl = *reinterpret_cast<const uint4*>(sm + OFF_H0 + TILE + so);
                    const uint32_t a[4] = {gh.x, gh.y, gh.z, gh.w}, a2[4] = {gl.x, gl.y, gl.z, gl.w};
                    const uint32_t b[4] = {hh.x, hh.y, hh.z, hh.w}, b2[4] = {hl.x, hl.y, hl.z, hl.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        kp = fmaf(bf16_lo(a[e]) + bf16_lo(a2[e]), bf16_lo(b[e]) + bf16_lo(b2[e]), kp);
                        kp = fmaf(bf16_hi(a[e]) + bf16_hi(a2[e]), bf16_hi(b[e]) + bf16_hi(b2[e]), kp);
                    }
                }
            }
            fence_proxy_async();
            mbar_arrive(bar(C_WE));
            // ---- C2: the transform of the tile (rows 32q.., columns 32c..)
            wait(M_SX, ph);
            wait(M_WE, ph);                                  // the WE tiles are consumed: dS^T may go there
            tc_fence_after();
            csync();                                         // the R table is complete
            float csum = 0.f, rsum[2] = {0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                // one 16-column K step: columns lc .. lc + 15
                const int lc = 32 * c + 16 * ks;
                uint32_t sv[16], xv[16];
                if (c >= q) {
                    tmem_ld16(tmem + lo16 + COL_S + lc, sv);
                    tmem_ld16(tmem + lo16 + COL_X + lc, xv);
                    tmem_wait_ld();
                }
                float wcol[16];
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    uint32_t mh[4], ml[4], dh[4], dl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float m2[2], g2[2];
#pragma unroll
                        for (int z2 = 0; z2 < 2; ++z2) {
                            const int kc = 8 * h8 + 2 * e + z2;      // column within the K step
                            const int l = lc + kc;
                            float m = 0.f, gd = 0.f, wcl = 0.f;
                            if (c >= q && l >= row) {
                                const float2 rl = s_rt[l];
                                const float f = ex2((rl.x - Rhi) + (rl.y - Rlo));
                                const float sval = __uint_as_float(sv[kc]);
                                m = sval * f;
                                gd = dt * f * __uint_as_float(xv[kc]);
                                if (l > row) {
                                    wcl = sval * gd;
                                    csum += wcl;
                                }
                            }
                            m2[z2] = m;
                            g2[z2] = gd;
                            wcol[kc] = wcl;
                        }
                        mh[e] = pack_bf16(m2[0], m2[1]);
                        ml[e] = pack_bf16(m2[0] - bf16_lo(mh[e]), m2[1] - bf16_hi(mh[e]));
                        dh[e] = pack_bf16(g2[0], g2[1]);
                        dl[e] = pack_bf16(g2[0] - bf16_lo(dh[e]), g2[1] - bf16_hi(dh[e]));
                    }
                    // Mt as the TMEM A operand: per K step 8 words hi, then 8 words lo
                    tmem_st4(tmem + lo16 + COL_S + lc + 4 * h8, mh);
                    tmem_st4(tmem + lo16 + COL_S + lc + 8 + 4 * h8, ml);
                    // dS^T hi / lo: K block lc / 64, 16-byte chunk (lc % 64) / 8 + h8
                    const uint32_t so = (uint32_t)(lc >> 6) * TILE + swz(row, ((lc & 63) >> 3) + h8);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + so) = make_uint4(dh[0], dh[1], dh[2], dh[3]);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + 2 * TILE + so) = make_uint4(dl[0], dl[1], dl[2], dl[3]);
                }
                // row sums over this warp's 32 rows of the 16 columns: lanes i and i + 16
                // end with column lc + (i & 15)
#pragma unroll
                for (int e = 0; e < 16; ++e) wcol[e] += __shfl_xor_sync(0xffffffffu, wcol[e], 16);
#pragma unroll
                for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
                    for (int e = 0; e < w; ++e) {
                        const bool up = (lane & w) != 0;
                        const float send = up ? wcol[e] : wcol[e + w];
                        const float keep = up ? wcol[e + w] : wcol[e];
                        wcol[e] = keep + __shfl_xor_sync(0xffffffffu, send, w);
                    }
                }
                rsum[ks] = wcol[0];
            }
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(bar(C_T));
            // ---- C3: u, v from TMEM X (B Ge | C h0), columns 16c..
            wait(M_BC, ph);
            tc_fence_after();
            float u = 0.f, vv = 0.f;
            uint32_t xpk[8];                                 // x of this row, columns 16c.., bf16 pairs
            {
                uint32_t bg[16], ch[16];
                tmem_ld16(tmem + lo16 + COL_X + 16 * c, bg);
                tmem_ld16(tmem + lo16 + COL_X + 64 + 16 * c, ch);
                const long long gofs = (((long long)d.b * p.L + (valid ? t : 0)) * p.H + d.h) * PD + 16 * c;
                const uint4 x0 = valid ? *reinterpret_cast<const uint4*>(xg + gofs) : make_uint4(0, 0, 0, 0);
                const uint4 x1 = valid ? *reinterpret_cast<const uint4*>(xg + gofs + 8) : make_uint4(0, 0, 0, 0);
                xpk[0] = x0.x; xpk[1] = x0.y; xpk[2] = x0.z; xpk[3] = x0.w;
                xpk[4] = x1.x; xpk[5] = x1.y; xpk[6] = x1.z; xpk[7] = x1.w;
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint4 yr = *reinterpret_cast<const uint4*>(sm + OFF_DY + swz(row, 2 * c + cc));
                    const uint32_t yw[4] = {yr.x, yr.y, yr.z, yr.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int k = 8 * cc + 2 * e;
                        u = fmaf(bf16_lo(yw[e]), __uint_as_float(ch[k]), fmaf(bf16_hi(yw[e]), __uint_as_float(ch[k + 1]), u));
                        vv = fmaf(bf16_lo(xpk[4 * cc + e]), __uint_as_float(bg[k]),
                                  fmaf(bf16_hi(xpk[4 * cc + e]), __uint_as_float(bg[k + 1]), vv));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bar(C_U));
            // ---- C4: dxu, dx, x . dxu
            wait(M_DX, ph);
            tc_fence_after();
            float xdxu = 0.f;
            {
                uint32_t bg[16], mt[16];
                tmem_ld16(tmem + lo16 + COL_X + 16 * c, bg);
                tmem_ld16(tmem + lo16 + COL_X + 64 + 16 * c, mt);
                const long long gofs = (((long long)d.b * p.L + (valid ? t : 0)) * p.H + d.h) * PD + 16 * c;
                uint4 y0 = make_uint4(0, 0, 0, 0), y1 = y0;
                if (valid) {
                    y0 = *reinterpret_cast<const uint4*>(dyg + gofs);
                    y1 = *reinterpret_cast<const uint4*>(dyg + gofs + 8);
                }
                const uint32_t yw[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
                tmem_wait_ld();
                const float dsk = p.D ? p.D[d.h] : 0.f;
                float o[16];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float du0 = fmaf(wt, __uint_as_float(bg[2 * e]), __uint_as_float(mt[2 * e]));
                    const float du1 = fmaf(wt, __uint_as_float(bg[2 * e + 1]), __uint_as_float(mt[2 * e + 1]));
                    xdxu = fmaf(bf16_lo(xpk[e]), du0, fmaf(bf16_hi(xpk[e]), du1, xdxu));
                    o[2 * e] = fmaf(dt, du0, dsk * bf16_lo(yw[e]));
                    o[2 * e + 1] = fmaf(dt, du1, dsk * bf16_hi(yw[e]));
                }
                if (valid) {
                    if (p.grad_bf16) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[e] = pack_bf16(o[2 * e], o[2 * e + 1]);
                        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.dx) + gofs);
                        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.dx) + gofs);
#pragma unroll
                        for (int e = 0; e < 4; ++e) dst[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                    }
                }
            }
            // ---- end of a segment: dB, dC partials (columns 32c..) -> slot
            if (d.last) {
                const long long slot = (long long)blockIdx.x * p.smax + (d.seg - seg0);
                float* dst = p.dbc + slot * 2 * 128 * 128;
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lo16 + (m ? COL_DC : COL_DB) + 32 * c, r);
                    tmem_wait_ld();
                    float4* o4 = reinterpret_cast<float4*>(dst + ((long long)m * 128 + row) * 128 + 32 * c);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        o4[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                            __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
                }
                tc_fence_before();
                mbar_arrive(bar(C_FL));
            }
            tc_fence_before();
            mbar_arrive(bar(C_E));
            // ---- the unit's token scalars into the scratch (dS^T is consumed: M_DX)
            scr[SC_C + c * 128 + row] = csum;
            if (lane < 16) {
                scr[SC_R + q * 128 + 32 * c + lane] = rsum[0];
                scr[SC_R + q * 128 + 32 * c + 16 + lane] = rsum[1];
            }
            scr[SC_U + c * 128 + row] = u;
            scr[SC_V + c * 128 + row] = vv;
            scr[SC_XDY + c * 128 + row] = xdy;
            scr[SC_XDXU + c * 128 + row] = xdxu;
            scr[SC_K + c * 128 + row] = kp;
            csync();
            // ---- d a, d dt_raw and the unit's parameter shares: warps c == 0, token = row
            if (c == 0) {
                float ksum = 0.f;
                for (int e = lane; e < 512; e += 32) ksum += scr[SC_K + e];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ksum += __shfl_xor_sync(0xffffffffu, ksum, o);
                const float K = ex2((float)tot) * ksum;
                float dk = 0.f, uu = 0.f, vs = 0.f, xd = 0.f, xu = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    dk += scr[SC_C + w * 128 + row] - scr[SC_R + w * 128 + row];
                    uu += scr[SC_U + w * 128 + row];
                    vs += scr[SC_V + w * 128 + row];
                    xd += scr[SC_XDY + w * 128 + row];
                    xu += scr[SC_XDXU + w * 128 + row];
                }
                uu *= er;
                vs *= wv;
                // exclusive prefix of dk and vs, inclusive suffix of uu over the 128 tokens
                float pd = dk, pv = vs, su = uu;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float a = __shfl_up_sync(0xffffffffu, pd, o), b2 = __shfl_up_sync(0xffffffffu, pv, o);
                    const float cu = __shfl_down_sync(0xffffffffu, su, o);
                    if (lane >= o) { pd += a; pv += b2; }
                    if (lane + o < 32) su += cu;
                }
                float* wt3 = scr + SC_K;                     // reused: [4][3] warp totals
                asm volatile("bar.sync 2, 128;" ::: "memory");   // every K share is read
                if (lane == 31) { wt3[q * 3] = pd; wt3[q * 3 + 1] = pv; }
                if (lane == 0) wt3[q * 3 + 2] = su;
                asm volatile("bar.sync 2, 128;" ::: "memory");
                float od = 0.f, ov = 0.f, ou = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (w < q) { od += wt3[w * 3]; ov += wt3[w * 3 + 1]; }
                    if (w > q) ou += wt3[w * 3 + 2];
                }
                const float Rx = od + pd - dk, Vx = ov + pv - vs, Ux = ou + su;
                const float da = Rx + Ux + Vx + K;
                const float dz = valid ? (xu + Ah * da) / (1.f + __expf(-z)) : 0.f;
                if (valid) {
                    const long long o = ((long long)d.b * p.L + t) * p.H + d.h;
                    if (p.grad_bf16) reinterpret_cast<bf16*>(p.ddt_raw)[o] = __float2bfloat16_rn(dz);
                    else reinterpret_cast<float*>(p.ddt_raw)[o] = dz;
                }
                float sa = valid ? dt * da : 0.f, sb = dz, sd = valid ? xd : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    sa += __shfl_xor_sync(0xffffffffu, sa, o);
                    sb += __shfl_xor_sync(0xffffffffu, sb, o);
                    sd += __shfl_xor_sync(0xffffffffu, sd, o);
                }
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (lane == 0) { wt3[q * 3] = sa; wt3[q * 3 + 1] = sb; wt3[q * 3 + 2] = sd; }
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (q == 0 && lane < 3) {
                    const float tsum = wt3[lane] + wt3[3 + lane] + wt3[6 + lane] + wt3[9 + lane];
                    p.part[(((long long)d.b * p.nblk + d.j) * p.H + d.h) * 3 + lane] = tsum;
                }
            }
        }
    }
    if (err) atomicOr(p.dev_err, err);
    tc_fence_before();
    __syncthreads();
    if (*s_abort) {
        const unsigned long long t0 = gtimer();
        while (gtimer() - t0 < 1000000ull) {
        }
    }
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

// ============================================================ 3. dB, dC partials
//
// (b, j, g) = T covers units [T hpg, (T + 1) hpg); the CTAs whose ranges meet it
// wrote one partial each, in slot (c, T - first segment of c).  They are summed
// in CTA order.  One thread per 4 consecutive elements of a [128][128] matrix.
template <typename GT>
__global__ void __launch_bounds__(256)
bwd_reduce_dbc_kernel(const float* __restrict__ dbc, GT* __restrict__ dB, GT* __restrict__ dC, long long L,
                      long long U, int grid, int smax, int hpg, int G, int nblk) {
    const long long T = blockIdx.y;
    const int m = (int)(blockIdx.x >> 4);                  // 0: dB, 1: dC
    const int e4 = (int)((blockIdx.x & 15) * 256 + threadIdx.x);   // float4 index in [128][128]
    const int row = e4 >> 5, col = (e4 & 31) * 4;
    const int g = (int)(T % G), j = (int)((T / G) % nblk);
    const long long b = T / G / nblk;
    const long long t = (long long)j * 128 + row;
    if (t >= L) return;
    auto cta_of = [&](long long u) -> long long { return ((u + 1) * grid + U - 1) / U - 1; };
    const long long c0 = cta_of(T * hpg), c1 = cta_of(T * hpg + hpg - 1);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long c = c0; c <= c1; ++c) {
        const long long seg0 = (c * U / grid) / hpg;
        const long long slot = c * smax + (T - seg0);
        const float4 v = *reinterpret_cast<const float4*>(dbc + ((slot * 2 + m) * 128 + row) * 128 + col);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    GT* out = (m ? dC : dB) + ((b * L + t) * G + g) * 128 + col;
    out[0] = from_f32<GT>(acc.x);
    out[1] = from_f32<GT>(acc.y);
    out[2] = from_f32<GT>(acc.z);
    out[3] = from_f32<GT>(acc.w);
}

}  // namespace bwdtc

// ---------------------------------------------------------------- host side

bool bwd_tc_supports(int64_t H, int64_t P, int64_t N, int64_t G, bool io_bf16) {
    return io_bf16 && P == bwdtc::PD && N == bwdtc::NS && (H / G) % 2 == 0;
}

// CTAs of the block-gradient kernel and partial slots per CTA (fixed by the
// shape alone, so that the workspace and the summation order do not depend on
// the device)
void bwd_tc_grid(int64_t batch, int64_t L, int64_t H, int64_t G, int64_t* grid, int64_t* smax) {
    const int64_t nblk = (L + tc::SUB - 1) / tc::SUB, U = batch * nblk * H, hpg = H / G;
    const int64_t gr = U < 148 ? (U > 0 ? U : 1) : 148;
    int64_t sm = 1;
    for (int64_t c = 0; c < gr && U > 0; ++c) {
        const int64_t a = c * U / gr, e = (c + 1) * U / gr;
        if (e > a) {
            const int64_t n = (e - 1) / hpg - a / hpg + 1;
            if (n > sm) sm = n;
        }
    }
    *grid = gr;
    *smax = sm;
}

cudaError_t launch_backward_tc(const BackwardArgs& a, cudaStream_t s) {
    using namespace bwdtc;
    const BackwardLayout& l = a.lay;
    const int64_t BH = a.batch * a.H, nblk = l.nb;
    CUtensorMap mx, mdy, mb, mc, mh0, mge;
    if (!tc::make_map(&mx, a.x, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.batch) ||
        !tc::make_map(&mdy, a.dy, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.batch) ||
        !tc::make_map(&mb, a.B, (uint64_t)a.N, (uint64_t)a.G, (uint64_t)a.L, (uint64_t)a.batch) ||
        !tc::make_map(&mc, a.C, (uint64_t)a.N, (uint64_t)a.G, (uint64_t)a.L, (uint64_t)a.batch) ||
        !tc::make_map(&mh0, a.ws + l.off_h0, PD, 2, NS, (uint64_t)(BH * nblk)) ||
        !tc::make_map(&mge, a.ws + l.off_ge, PD, 2, NS, (uint64_t)(BH * nblk)))
        return cudaErrorInvalidValue;
    static std::mutex mu;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!attr_set[dev]) {
            e = cudaFuncSetAttribute(bwd_states_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)st::SMEM);
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(bwd_main_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mn::SMEM);
            if (e != cudaSuccess) return e;
            attr_set[dev] = true;
        }
    }
    // 1. state passes
    st::Params sp{};
    sp.dt_raw = a.dt_raw;
    sp.dt_bias = a.dt_bias;
    sp.A = a.A;
    sp.init_state = a.init_state;
    sp.dfinal = a.dfinal;
    sp.h0 = (uint16_t*)(a.ws + l.off_h0);
    sp.ge = (uint16_t*)(a.ws + l.off_ge);
    sp.dinit = a.dinit;
    sp.dev_err = a.dev_err;
    sp.L = a.L;
    sp.H = (int)a.H;
    sp.G = (int)a.G;
    sp.nblk = (int)nblk;
    sp.npairs = (int)(BH / 2);
    sp.state_bf16 = a.state_bf16;
    bwd_states_tc_kernel<<<(unsigned)(2 * sp.npairs), st::THREADS, st::SMEM, s>>>(mx, mdy, mb, mc, sp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 2. block gradients
    int64_t grid = 0, smax = 0;
    bwd_tc_grid(a.batch, a.L, a.H, a.G, &grid, &smax);
    mn::Params mp{};
    mp.x = a.x;
    mp.dy = a.dy;
    mp.dt_raw = a.dt_raw;
    mp.dt_bias = a.dt_bias;
    mp.A = a.A;
    mp.D = a.D;
    mp.dx = a.dx;
    mp.ddt_raw = a.ddt_raw;
    mp.part = (float*)(a.ws + l.off_part);
    mp.dbc = (float*)(a.ws + l.off_dbc);
    mp.dev_err = a.dev_err;
    mp.L = a.L;
    mp.U = a.batch * nblk * a.H;
    mp.H = (int)a.H;
    mp.G = (int)a.G;
    mp.nblk = (int)nblk;
    mp.smax = (int)smax;
    mp.grad_bf16 = a.grad_bf16;
    bwd_main_tc_kernel<<<(unsigned)grid, mn::THREADS, mn::SMEM, s>>>(mx, mdy, mb, mc, mh0, mge, mp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3. dB, dC
    const dim3 rgrid(32, (unsigned)(a.batch * nblk * a.G));
    if (a.grad_bf16)
        bwd_reduce_dbc_kernel<bf16><<<rgrid, 256, 0, s>>>(mp.dbc, (bf16*)a.dB, (bf16*)a.dC, a.L, mp.U, (int)grid,
                                                          (int)smax, (int)(a.H / a.G), (int)a.G, (int)nblk);
    else
        bwd_reduce_dbc_kernel<float><<<rgrid, 256, 0, s>>>(mp.dbc, (float*)a.dB, (float*)a.dC, a.L, mp.U, (int)grid,
                                                           (int)smax, (int)(a.H / a.G), (int)a.G, (int)nblk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_backward_params(mp.part, a.dA, a.ddt_bias, a.dD, a.batch * nblk, (int)a.H, s);
}

}  // namespace ssd
