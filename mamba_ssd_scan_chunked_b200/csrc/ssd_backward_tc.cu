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
constexpr uint32_t OFF_N = 0;                     // 2 stages: N-side tiles (n 0-63, 64-127)
constexpr uint32_t OFF_P = 4 * TILE;              // P-side tile per head (single buffer)
constexpr uint32_t OFF_W = 6 * TILE;              // 2 buffers x 2 heads: (w o P-side) hi, lo
constexpr uint32_t OFF_TOT = OFF_W + 8 * TILE;    // [2 heads][4 quarters] double: warp totals of the scan
constexpr uint32_t OFF_BAR = OFF_TOT + 2 * 4 * 8;
enum { B_FULLN0, B_FULLN1, B_FULLP, B_PFREE, B_WX, B_MMA, NBAR };
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr uint32_t SMEM = OFF_MISC + 16;
static_assert(SMEM <= 232448, "shared memory per CTA");

struct Params {
    const void* dt_raw;        // bf16 [b][L][H]
    const float* dt_bias;      // [H] or NULL
    const float* A;            // [H]
    const void* init_state;    // state dtype [b*H][N][P] or NULL
    const void* dfinal;        // state dtype [b*H][N][P] or NULL
    void* dinit;               // state dtype [b*H][N][P] or NULL
    unsigned* dev_err;
    long long L;
    int H, G, nblk, npairs, state_bf16;
};
}  // namespace st

// Per block i of the walk: the compute warps form w o (x or dy) of block i into
// W buffer i & 1 while the MMAs of block i - 1 still run, then wait for them,
// stage the state as hi/lo tiles in W buffer (i + 1) & 1 (which those MMAs have
// just finished reading), scale it by 2^(R_last) in TMEM, and one thread per
// head stores the two tiles with TMA; the MMAs of block i follow.  The P-side
// tile is reloaded as soon as w o P of block i is formed, the N-side tiles (B
// or C) two blocks ahead.
__global__ void __launch_bounds__(st::THREADS, 1)
bwd_states_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmDY,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmH0, const __grid_constant__ CUtensorMap tmGE,
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
        const uint32_t cnt[NBAR] = {1, 1, 1, NCT, NCT, 1};
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
        auto load_n = [&](int i) {
            const int t0 = blk_of(i) * SUB;
            const uint32_t stg = base + OFF_N + (uint32_t)(i & 1) * 2 * TILE, bb = bar(B_FULLN0 + (i & 1));
            mbar_expect_tx(bb, 2 * TILE);
            tma_load_4d(stg, tmN, 0, g, t0, b, bb);
            tma_load_4d(stg + TILE, tmN, 64, g, t0, b, bb);
        };
        auto load_p = [&](int i) {
            const int t0 = blk_of(i) * SUB;
            mbar_expect_tx(bar(B_FULLP), 2 * TILE);
            tma_load_4d(base + OFF_P, tmP, 0, h0, t0, b, bar(B_FULLP));
            tma_load_4d(base + OFF_P + TILE, tmP, 0, h0 + 1, t0, b, bar(B_FULLP));
        };
        if (lead) {
            load_n(0);
            if (nblk > 1) load_n(1);
            load_p(0);
        }
        __syncwarp();
        constexpr uint32_t ID = idesc_bf16(128, PD, true, true);   // N-side^T (MN-major) x w o P-side (MN-major)
        constexpr uint32_t KSTEP_MN = 2048 >> 4;
        for (int i = 0; i < nblk; ++i) {
            wait(B_PFREE, i & 1);            // w o P of block i is formed: the P tile is free
            if (lead && i + 1 < nblk && !*s_abort) load_p(i + 1);
            __syncwarp();
            wait(B_WX, i & 1);               // states written out and scaled
            tc_fence_after();
            const uint64_t dN = sdesc(base + OFF_N + (uint32_t)(i & 1) * 2 * TILE, TILE, 1024);
            const bool go = lead && !*s_abort;
            const uint32_t wb = base + OFF_W + (uint32_t)(i & 1) * 4 * TILE;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint64_t dWh = sdesc(wb + 2 * k * TILE, TILE, 1024);
                const uint64_t dWl = sdesc(wb + (2 * k + 1) * TILE, TILE, 1024);
#pragma unroll
                for (int kk = 0; kk < SUB / 16; ++kk) {
                    if (go) mma_ss<ID, 1>(tmem + 64 * k, dN + kk * KSTEP_MN, dWh + kk * KSTEP_MN);
                    if (go) mma_ss<ID, 1>(tmem + 64 * k, dN + kk * KSTEP_MN, dWl + kk * KSTEP_MN);
                }
            }
            if (go) mma_commit(bar(B_MMA));
            __syncwarp();
            wait(B_MMA, i & 1);              // the N stage is free again
            if (lead && i + 2 < nblk && !*s_abort) load_n(i + 2);
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
        auto fetch = [&](int i) -> uint16_t {
            const long long t = (long long)blk_of(i) * SUB + row;
            return t < p.L ? dtr[(b * p.L + t) * p.H + h] : (uint16_t)0;
        };
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
        const bool issuer = q == 0 && lane == 0;     // stores head k's tiles
        uint16_t dtr_next = fetch(0);
        for (int i = 0; i < nblk; ++i) {
            const int j = blk_of(i);
            const long long t = (long long)j * SUB + row;
            // dt and the block-local cumsum of dt A log2(e) (double), token s = row
            const float dt = t < p.L ? softplus_f32(__uint_as_float((uint32_t)dtr_next << 16) + bias) : 0.f;
            if (i + 1 < nblk) dtr_next = fetch(i + 1);
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
            // w o (x or dy) of token `row` into W buffer i & 1 (the MMAs of block i - 2,
            // which read it, completed before block i - 1's state was written out; the
            // TMA store of that state, staged there, has read it: waited by its issuer)
            wait(B_FULLN0 + (i & 1), (i >> 1) & 1);
            wait(B_FULLP, i & 1);
            if (issuer) bulk_wait_read0();
            asm volatile("bar.sync %0, %1;" ::"r"(1 + k), "r"(128) : "memory");
            {
                const uint8_t* src = sm + OFF_P + k * TILE;
                uint8_t* dh = sm + OFF_W + (i & 1) * 4 * TILE + 2 * k * TILE;
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
            mbar_arrive(bar(B_PFREE));
            // the previous block's update is complete: write the value out, scale it
            if (i > 0) wait(B_MMA, (i - 1) & 1);
            tc_fence_after();
            {
                uint8_t* sh = sm + OFF_W + ((i + 1) & 1) * 4 * TILE + 2 * k * TILE;   // staging: hi, lo tiles
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
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t so = swz(row, 4 * c + e);
                        *reinterpret_cast<uint4*>(sh + so) = make_uint4(hw[4 * e], hw[4 * e + 1], hw[4 * e + 2], hw[4 * e + 3]);
                        *reinterpret_cast<uint4*>(sh + TILE + so) = make_uint4(lw[4 * e], lw[4 * e + 1], lw[4 * e + 2], lw[4 * e + 3]);
                    }
                    tmem_st32(tmem + lo16 + 64 * k + 32 * c, sv);
                }
                tmem_wait_st();
                fence_proxy_async();
                asm volatile("bar.sync %0, %1;" ::"r"(1 + k), "r"(128) : "memory");
                if (issuer && !*s_abort) {
                    const int un = (int)(bh * nblk + j);
                    const uint32_t sa = base + OFF_W + (uint32_t)((i + 1) & 1) * 4 * TILE + 2 * k * TILE;
                    tma_store_4d(rev ? &tmGE : &tmH0, sa, 0, 0, 0, un);
                    tma_store_4d(rev ? &tmGE : &tmH0, sa + TILE, 0, 1, 0, un);
                    bulk_commit();
                }
            }
            tc_fence_before();
            mbar_arrive(bar(B_WX));
        }
        if (issuer) bulk_wait0();                   // the last tiles are written
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

}  // namespace bwdtc

namespace bwdtc {
// ============================================================ 2. block gradients
//
// Unit u = ((b * nblk + j) * G + g) * hpg + q: head g*hpg + q of block j of
// batch element b.  CTA c takes units [c U / grid, (c + 1) U / grid); a run of
// its units with the same (b, j, g) is a segment, whose dB and dC accumulate in
// TMEM over the segment's heads and leave as one partial.  Per unit (rows s or
// l are the block's tokens, 128 TMEM lanes), in issue order:
//
//   M1  S^T = B C^T                           -> TMEM S
//   M2  X dY^T                                -> TMEM X
//   C2  transform: Mt = S^T e (in TMEM S as bf16 hi|lo), dS^T = dt_s e X dY^T
//       (hi/lo tiles), e = 2^(R_l - R_s) [l >= s]; column and row sums of S dS
//   M4  B Ge -> TMEM X[0:64], C h0 -> TMEM X[64:128]
//   C3  u_l = 2^(R_l) dy_l . (C h0)_l, v_s = w_s x_s . (B Ge)_s
//   M6  Mt dY -> TMEM X[64:128]
//   C4  dxu = Mt dY + 2^(R_last - R_s) B Ge; dx; x . dxu; d a, d dt_raw and the
//       unit's shares of dA, d dt_bias, dD
//   M5  dB += dS^T C, dC += dS B
//   C1  (w o X), (2^R o dY) as hi/lo tiles over the consumed dS^T
//   M3  dB += (w o X) Ge^T, dC += (2^R o dY) h0^T     (hi.hi + hi.lo + lo.hi)
//   end of segment: TMEM dB, dC -> partial slot
// The chain that gives dx and d a (M1 .. C4) does not wait for the dB, dC MMAs
// (M5, M3), which run while the next unit's operands load.
namespace mn {
constexpr int NCW = 16;
constexpr int NCT = NCW * 32;
constexpr int WARP_MMA = NCW, WARP_TMA = NCW + 1;
constexpr int THREADS = NCT + 64;
constexpr uint32_t COL_S = 0, COL_X = 128, COL_DB = 256, COL_DC = 384;
constexpr uint32_t OFF_B = 0;                    // B tiles: n 0-63, n 64-127 (rows = tokens)
constexpr uint32_t OFF_C = 2 * TILE;             // C tiles
constexpr uint32_t OFF_X = 4 * TILE;             // x tile (rows = tokens, 64 p); later the unit's scratch
constexpr uint32_t OFF_DY = 5 * TILE;            // dy tile
constexpr uint32_t OFF_H0 = 6 * TILE;            // h0 hi, lo (rows = n, 64 p)
constexpr uint32_t OFF_GE = 8 * TILE;            // Ge hi, lo
constexpr uint32_t OFF_WD = 10 * TILE;           // dS^T hi (l 0-63, 64-127), lo (l 0-63, 64-127);
                                                 // later (w o X) hi, lo, (2^R o dY) hi, lo
constexpr uint32_t OFF_RT = 14 * TILE;           // float2 [128]: R (hi, lo) of the block's tokens
constexpr uint32_t OFF_TOT = OFF_RT + 128 * 8;   // double [4]: scan totals of the lane quarters
constexpr uint32_t OFF_BAR = OFF_TOT + 4 * 8;
enum { F_BC, F_X, F_DY, F_HG, M_SX, C_T, M_BC, C_U, M_DX, C_E, M_DS, C_WE, M_WE, C_FL, NBAR };
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr uint32_t SMEM = OFF_MISC + 16;
static_assert(SMEM <= 232448, "shared memory per CTA");
// scratch in the x tile (floats) once its values are in registers and M2 has run
constexpr int SC_C = 0, SC_R = 512, SC_U = 1024, SC_V = 1536, SC_XDY = 2048, SC_XDXU = 2560, SC_K = 3072;
constexpr int SC_END = 3584;
static_assert(SC_END * 4 <= (int)TILE, "scratch fits the x tile");

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
        //                          BC X  DY HG SX T    BC U    DX E    DS WE   MWE FL
        const uint32_t cnt[NBAR] = {1, 1, 1, 1, 1, NCT, 1, NCT, 1, NCT, 1, NCT, 1, NCT};
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
        d.g = (int)(d.seg % p.G);
        d.h = d.g * hpg + (int)(u % hpg);
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
            // x, dy: read by M2, M6 and into registers; the x tile was the previous unit's scratch
            if (i > 0) { wait(M_DX, (i - 1) & 1); wait(C_E, (i - 1) & 1); }
            if (lead && !*s_abort) {
                mbar_expect_tx(bar(F_X), TILE);
                tma_load_4d(base + OFF_X, &tmX, 0, d.h, t0, d.b, bar(F_X));
                mbar_expect_tx(bar(F_DY), TILE);
                tma_load_4d(base + OFF_DY, &tmDY, 0, d.h, t0, d.b, bar(F_DY));
                if (i + 1 < nu) {                    // the next unit's x, dy into L2
                    const Unit e = unit(i + 1);
                    tma_prefetch_4d(&tmX, 0, e.h, e.j * SUB, e.b);
                    tma_prefetch_4d(&tmDY, 0, e.h, e.j * SUB, e.b);
                }
            }
            // h0, Ge (and at a segment's start B, C): the previous unit's MMAs are all done
            if (i > 0) wait(M_WE, (i - 1) & 1);
            if (lead && !*s_abort) {
                if (d.first) {
                    mbar_expect_tx(bar(F_BC), 4 * TILE);
                    tma_load_4d(base + OFF_B, &tmB, 0, d.g, t0, d.b, bar(F_BC));
                    tma_load_4d(base + OFF_B + TILE, &tmB, 64, d.g, t0, d.b, bar(F_BC));
                    tma_load_4d(base + OFF_C, &tmC, 0, d.g, t0, d.b, bar(F_BC));
                    tma_load_4d(base + OFF_C + TILE, &tmC, 64, d.g, t0, d.b, bar(F_BC));
                }
                mbar_expect_tx(bar(F_HG), 4 * TILE);
                tma_load_4d(base + OFF_H0, &tmH0, 0, 0, 0, (int)un, bar(F_HG));
                tma_load_4d(base + OFF_H0 + TILE, &tmH0, 0, 1, 0, (int)un, bar(F_HG));
                tma_load_4d(base + OFF_GE, &tmGE, 0, 0, 0, (int)un, bar(F_HG));
                tma_load_4d(base + OFF_GE + TILE, &tmGE, 0, 1, 0, (int)un, bar(F_HG));
            }
            if (d.first) ++nseg;
            __syncwarp();
        }
        (void)nseg;
    } else if (warp == WARP_MMA) {
        // ======================================================== MMA issue
        const uint32_t lead0 = elect_one();
        constexpr uint32_t ID_KK = idesc_bf16(128, 128, false, false);     // K-major x K-major, N = 128
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
            if (i > 0) wait(C_E, ph ^ 1u);           // TMEM X read (and TMEM S: M6 completed before)
            tc_fence_after();
            __syncwarp();
            // M1: S^T = B C^T (K = n, 8 steps); M2: X dY^T (K = p, 4 steps)
            {
                const uint64_t dB = sdesc(base + OFF_B, 16, 1024), dC = sdesc(base + OFF_C, 16, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                    if (k == 0) { if (lead) mma_ss<ID_KK, 0>(tmem + COL_S, dB + o, dC + o);
                    } else if (lead) mma_ss<ID_KK, 1>(tmem + COL_S, dB + o, dC + o);
                }
                const uint64_t dX = sdesc(base + OFF_X, 16, 1024), dY = sdesc(base + OFF_DY, 16, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t o = (uint32_t)k * KSTEP_K;
                    if (k == 0) { if (lead) mma_ss<ID_KK, 0>(tmem + COL_X, dX + o, dY + o);
                    } else if (lead) mma_ss<ID_KK, 1>(tmem + COL_X, dX + o, dY + o);
                }
                if (lead) mma_commit(bar(M_SX));
            }
            // M4: B Ge -> X[0:64], C h0 -> X[64:128] (K = n, 8 steps; Ge, h0 MN-major, hi + lo)
            wait(C_T, ph);
            wait(F_HG, ph);
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
            // M5: dB += dS^T C (K = l), dC += dS B (K = s); the segment's first MMAs overwrite
            if (d.first && nseg > 1) wait(C_FL, (nseg - 2) & 1);     // the previous partial is out
            tc_fence_after();
            __syncwarp();
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
                        if (hl == 0 && k == 0 && d.first) {
                            if (lead) mma_ss<ID_DB, 0>(tmem + COL_DB, aK + o, dCm);
                            if (lead) mma_ss<ID_DC, 0>(tmem + COL_DC, aM, dBm);
                        } else {
                            if (lead) mma_ss<ID_DB, 1>(tmem + COL_DB, aK + o, dCm + k * KSTEP_MN);
                            if (lead) mma_ss<ID_DC, 1>(tmem + COL_DC, aM + k * KSTEP_MN, dBm + k * KSTEP_MN);
                        }
                    }
                }
                if (lead) mma_commit(bar(M_DS));
            }
            // M3: dB += (w o X) Ge^T, dC += (2^R o dY) h0^T (K = p, 4 steps; hi.hi, hi.lo, lo.hi)
            wait(C_WE, ph);
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
                    if (lead) mma_ss<ID_KK, 1>(tmem + COL_DB, wh + o, gh + o);
                    if (lead) mma_ss<ID_KK, 1>(tmem + COL_DC, eh + o, hh + o);
                    if (lead) mma_ss<ID_KK, 1>(tmem + COL_DB, wh + o, gl + o);
                    if (lead) mma_ss<ID_KK, 1>(tmem + COL_DB, wl + o, gh + o);
                    if (lead) mma_ss<ID_KK, 1>(tmem + COL_DC, eh + o, hl + o);
                    if (lead) mma_ss<ID_KK, 1>(tmem + COL_DC, el + o, hh + o);
                }
                if (lead) mma_commit(bar(M_WE));
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
        float* scr = reinterpret_cast<float*>(sm + OFF_X);
        const uint16_t* dtr = reinterpret_cast<const uint16_t*>(p.dt_raw);
        auto csync = [&]() { asm volatile("bar.sync 1, %0;" ::"r"(NCT) : "memory"); };
        // the unit after d: (b, j, g, head in group) stepped as a counter
        auto step = [&](Unit d) -> Unit {
            Unit e = d;
            int qh = d.h - d.g * hpg + 1;
            e.first = qh == hpg;
            if (qh == hpg) {
                qh = 0;
                ++e.seg;
                if (++e.g == p.G) {
                    e.g = 0;
                    if (++e.j == p.nblk) { e.j = 0; ++e.b; }
                }
            }
            e.h = e.g * hpg + qh;
            e.last = qh == hpg - 1;
            return e;
        };
        struct Pre { uint16_t dtr; float A, bias, D; };
        auto fetch = [&](const Unit& d) -> Pre {
            const long long t = (long long)d.j * SUB + row;
            Pre r;
            r.dtr = t < p.L ? dtr[((long long)d.b * p.L + t) * p.H + d.h] : (uint16_t)0;
            r.A = p.A[d.h];
            r.bias = p.dt_bias ? p.dt_bias[d.h] : 0.f;
            r.D = p.D ? p.D[d.h] : 0.f;
            return r;
        };
        Unit dn = unit(0);
        Pre pn = fetch(dn);
        for (int i = 0; i < nu; ++i) {
            Unit d = dn;
            d.last = d.last || i == nu - 1;
            d.first = d.first || i == 0;
            const Pre pc = pn;
            if (i + 1 < nu) {
                dn = step(d);
                pn = fetch(dn);
            }
            const uint32_t ph = i & 1;
            const long long t = (long long)d.j * SUB + row;
            const bool valid = t < p.L;
            const float Ah = pc.A, bias = pc.bias;
            const float z = __uint_as_float((uint32_t)pc.dtr << 16) + bias;
            const float dt = valid ? softplus_f32(z) : 0.f;
            // ---- P1: block-local cumsum R of dt A log2(e) (double), per token
            double v = (double)(dt * Ah) * (double)LOG2E;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double w = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += w;
            }
            if (c == 0 && lane == 31) s_tot[q] = v;
            csync();                                        // (also: every thread is past the previous unit)
            double off = 0.0, tot = 0.0;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const double tw = s_tot[w];
                if (w < q) off += tw;
                tot += tw;
            }
            const double R = v + off;
            const float Rhi = (float)R, Rlo = (float)(R - (double)Rhi);
            const float totf = (float)tot;
            const float wt = ex2((float)(tot - R));        // 2^(R_last - R_s)
            const float er = ex2(Rhi + Rlo);               // 2^(R_s)
            const float wv = dt * wt;                      // w_s
            if (c == 0) s_rt[row] = make_float2(Rhi, Rlo);
            // ---- x and dy of this row, columns 16c .. 16c + 15, into registers
            wait(F_X, ph);
            wait(F_DY, ph);
            uint32_t xr[8], yr[8];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const uint32_t so = swz(row, 2 * c + cc);
                const uint4 a4 = *reinterpret_cast<const uint4*>(sm + OFF_X + so);
                const uint4 b4 = *reinterpret_cast<const uint4*>(sm + OFF_DY + so);
                xr[4 * cc] = a4.x; xr[4 * cc + 1] = a4.y; xr[4 * cc + 2] = a4.z; xr[4 * cc + 3] = a4.w;
                yr[4 * cc] = b4.x; yr[4 * cc + 1] = b4.y; yr[4 * cc + 2] = b4.z; yr[4 * cc + 3] = b4.w;
            }
            float xdy = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) xdy = fmaf(bf16_lo(xr[e]), bf16_lo(yr[e]), fmaf(bf16_hi(xr[e]), bf16_hi(yr[e]), xdy));
            // ---- C2: the transform of the tile (rows 32q.., columns 32c..); dS^T goes over
            // the previous unit's (w o X), (2^R o dY) tiles
            wait(M_SX, ph);
            if (i > 0) wait(M_WE, ph ^ 1u);
            tc_fence_after();
            csync();                                         // the R table is complete, x is in registers
            float csum = 0.f, rsum[4] = {0.f, 0.f, 0.f, 0.f};
            float* tw = scr + warp * 256;                    // this warp's [32 rows][8] transpose buffer
            if (c < q) {
                // the tile lies wholly above the diagonal (l < s): zeros
                const uint32_t zz[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const int lc = 32 * c + 8 * ch, kb = lc & ~15, wo = (lc & 15) >> 1;
                    tmem_st4(tmem + lo16 + COL_S + kb + wo, zz);
                    tmem_st4(tmem + lo16 + COL_S + kb + 8 + wo, zz);
                    const uint32_t so = (uint32_t)(lc >> 6) * TILE + swz(row, (lc & 63) >> 3);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + so) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + 2 * TILE + so) = make_uint4(0, 0, 0, 0);
                }
            } else {
#pragma unroll
            for (int ks2 = 0; ks2 < 2; ++ks2) {
                // one 16-column K step: its S^T is read whole before Mt overwrites it in place
                const int kb = 32 * c + 16 * ks2;
                uint32_t sv[16];
                tmem_ld16(tmem + lo16 + COL_S + kb, sv);
                tmem_wait_ld();
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    // 8 columns lc .. lc + 7
                    const int ch = 2 * ks2 + h8, lc = kb + 8 * h8;
                    uint32_t xv[8];
                    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                                 : "=r"(xv[0]), "=r"(xv[1]), "=r"(xv[2]), "=r"(xv[3]), "=r"(xv[4]), "=r"(xv[5]),
                                   "=r"(xv[6]), "=r"(xv[7]) : "r"(tmem + lo16 + COL_X + lc));
                    tmem_wait_ld();
                    uint32_t mh[4], ml[4], dh[4], dl[4];
                    float wcol[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float m2[2], g2[2];
#pragma unroll
                        for (int z2 = 0; z2 < 2; ++z2) {
                            const int kc = 2 * e + z2;
                            const int l = lc + kc;
                            float m = 0.f, gd = 0.f, wcl = 0.f;
                            if (l >= row) {
                                const float2 rl = s_rt[l];
                                const float f = ex2((rl.x - Rhi) + (rl.y - Rlo));
                                const float sval = __uint_as_float(sv[8 * h8 + kc]);
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
                    // Mt as the TMEM A operand: per 16-column K step 8 words hi, then 8 words lo
                    tmem_st4(tmem + lo16 + COL_S + kb + 4 * h8, mh);
                    tmem_st4(tmem + lo16 + COL_S + kb + 8 + 4 * h8, ml);
                    // dS^T hi / lo: K block lc / 64, 16-byte chunk (lc % 64) / 8
                    const uint32_t so = (uint32_t)(lc >> 6) * TILE + swz(row, (lc & 63) >> 3);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + so) = make_uint4(dh[0], dh[1], dh[2], dh[3]);
                    *reinterpret_cast<uint4*>(sm + OFF_WD + 2 * TILE + so) = make_uint4(dl[0], dl[1], dl[2], dl[3]);
                    // column sums of the 8 columns over this warp's 32 rows, through the
                    // transpose buffer: lane i sums column i & 7 over rows 8 (i >> 3) ..
                    *reinterpret_cast<float4*>(tw + lane * 8) = make_float4(wcol[0], wcol[1], wcol[2], wcol[3]);
                    *reinterpret_cast<float4*>(tw + lane * 8 + 4) = make_float4(wcol[4], wcol[5], wcol[6], wcol[7]);
                    __syncwarp();
                    float cs = 0.f;
#pragma unroll
                    for (int r = 0; r < 8; ++r) cs += tw[(8 * (lane >> 3) + r) * 8 + (lane & 7)];
                    cs += __shfl_xor_sync(0xffffffffu, cs, 8);
                    cs += __shfl_xor_sync(0xffffffffu, cs, 16);
                    rsum[ch] = cs;                           // lanes i and i ^ 8, i ^ 16, i ^ 24: column lc + (i & 7)
                    __syncwarp();
                }
            }
            }
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(bar(C_T));
            // the row's shares into the scratch (the x tile: M2 has read it, x is in registers,
            // and every warp is done with its transform buffer)
            csync();
            scr[SC_C + c * 128 + row] = csum;
            if (lane < 8) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) scr[SC_R + q * 128 + 32 * c + 8 * ch + lane] = rsum[ch];
            }
            scr[SC_XDY + c * 128 + row] = xdy;
            // ---- <Ge, h0> share: row n = row, columns 16c..
            wait(F_HG, ph);
            float kp = 0.f;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const uint32_t so = swz(row, 2 * c + cc);
                const uint4 gh = *reinterpret_cast<const uint4*>(sm + OFF_GE + so);
                const uint4 gl = *reinterpret_cast<const uint4*>(sm + OFF_GE + TILE + so);
                const uint4 hh = *reinterpret_cast<const uint4*>(sm + OFF_H0 + so);
                const uint4 hl = *reinterpret_cast<const uint4*>(sm + OFF_H0 + TILE + so);
                const uint32_t a1[4] = {gh.x, gh.y, gh.z, gh.w}, a2[4] = {gl.x, gl.y, gl.z, gl.w};
                const uint32_t b1[4] = {hh.x, hh.y, hh.z, hh.w}, b2[4] = {hl.x, hl.y, hl.z, hl.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kp = fmaf(bf16_lo(a1[e]) + bf16_lo(a2[e]), bf16_lo(b1[e]) + bf16_lo(b2[e]), kp);
                    kp = fmaf(bf16_hi(a1[e]) + bf16_hi(a2[e]), bf16_hi(b1[e]) + bf16_hi(b2[e]), kp);
                }
            }
            scr[SC_K + c * 128 + row] = kp;
            // ---- C3: u, v from TMEM X (B Ge | C h0), columns 16c..
            wait(M_BC, ph);
            tc_fence_after();
            float u = 0.f, vv = 0.f;
            {
                uint32_t bg[16], chv[16];
                tmem_ld16(tmem + lo16 + COL_X + 16 * c, bg);
                tmem_ld16(tmem + lo16 + COL_X + 64 + 16 * c, chv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    u = fmaf(bf16_lo(yr[e]), __uint_as_float(chv[2 * e]), fmaf(bf16_hi(yr[e]), __uint_as_float(chv[2 * e + 1]), u));
                    vv = fmaf(bf16_lo(xr[e]), __uint_as_float(bg[2 * e]), fmaf(bf16_hi(xr[e]), __uint_as_float(bg[2 * e + 1]), vv));
                }
            }
            scr[SC_U + c * 128 + row] = u;
            scr[SC_V + c * 128 + row] = vv;
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
                tmem_wait_ld();
                const float dsk = pc.D;
                float o[16];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float du0 = fmaf(wt, __uint_as_float(bg[2 * e]), __uint_as_float(mt[2 * e]));
                    const float du1 = fmaf(wt, __uint_as_float(bg[2 * e + 1]), __uint_as_float(mt[2 * e + 1]));
                    xdxu = fmaf(bf16_lo(xr[e]), du0, fmaf(bf16_hi(xr[e]), du1, xdxu));
                    o[2 * e] = fmaf(dt, du0, dsk * bf16_lo(yr[e]));
                    o[2 * e + 1] = fmaf(dt, du1, dsk * bf16_hi(yr[e]));
                }
                if (valid) {
                    const long long gofs = (((long long)d.b * p.L + t) * p.H + d.h) * PD + 16 * c;
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
            scr[SC_XDXU + c * 128 + row] = xdxu;
            csync();
            // ---- d a, d dt_raw and the unit's parameter shares: warps c == 0, token = row
            if (c == 0) {
                float ksum = 0.f;
                for (int e = lane; e < 512; e += 32) ksum += scr[SC_K + e];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ksum += __shfl_xor_sync(0xffffffffu, ksum, o);
                const float K = ex2(totf) * ksum;
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
                float* wt3 = scr + SC_END;                   // [4][3] warp totals (after the scratch arrays)
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
                asm volatile("bar.sync 2, 128;" ::: "memory");   // every warp total is read
                if (lane == 0) { wt3[q * 3] = sa; wt3[q * 3 + 1] = sb; wt3[q * 3 + 2] = sd; }
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (q == 0 && lane < 3) {
                    const float tsum = wt3[lane] + wt3[3 + lane] + wt3[6 + lane] + wt3[9 + lane];
                    p.part[(((long long)d.b * p.nblk + d.j) * p.H + d.h) * 3 + lane] = tsum;
                }
            }
            csync();                                         // the scratch is consumed
            tc_fence_before();
            mbar_arrive(bar(C_E));                           // TMEM X and the x tile are free
            // ---- C1: (w o X), (2^R o dY) hi/lo over the consumed dS^T
            wait(M_DS, ph);
            {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t so = swz(row, 2 * c + cc);
                    uint32_t ah[4], al[4], bh[4], bl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t xw = xr[4 * cc + e], yw = yr[4 * cc + e];
                        const float a0 = wv * bf16_lo(xw), a1 = wv * bf16_hi(xw);
                        const float b0 = er * bf16_lo(yw), b1 = er * bf16_hi(yw);
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
            fence_proxy_async();
            mbar_arrive(bar(C_WE));
            // ---- end of a segment: dB, dC partials (columns 32c..) -> slot
            if (d.last) {
                wait(M_WE, ph);
                tc_fence_after();
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
    sp.dinit = a.dinit;
    sp.dev_err = a.dev_err;
    sp.L = a.L;
    sp.H = (int)a.H;
    sp.G = (int)a.G;
    sp.nblk = (int)nblk;
    sp.npairs = (int)(BH / 2);
    sp.state_bf16 = a.state_bf16;
    bwd_states_tc_kernel<<<(unsigned)(2 * sp.npairs), st::THREADS, st::SMEM, s>>>(mx, mdy, mb, mc, mh0, mge, sp);
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
