// Tensor-core prefill of the SSD layer core for sm_100a, two heads at a time.
//
// The chunked contraction of the semiseparable matrix ("Mamba-2 vs
// Transformers / SSD", section "Mamba-2 and the SSD paper: what changed in
// practice": chunks processed in parallel, per-chunk states recombined; table
// row "Blocked two-pass contraction").  Heads of one group share B and C, and
// so share S = C B^T.  A work item here is a pair of heads (h0, h0+1) of one
// group and one batch element, walked through its sequence in blocks of 128
// tokens with both states kept in TMEM.  Per block, with r = decay cumsum *
// log2(e) relative to the block start (per head):
//
//   S      = C B^T                         once for both heads (tcgen05, fp32 in TMEM)
//   M_k    = S o [s<=l] 2^(r_l - r_s) dt_s  per head k (CUDA cores, TMEM -> regs -> TMEM)
//   Yoff_k = C h_k                          (tcgen05; then scaled by 2^(r_l) in place)
//   h_k'   = 2^(r_last) h_k + B^T (w o X_k) (tcgen05 onto the scaled state in TMEM)
//   y_k    = Yoff_k + M_k X_k + D_k x       (tcgen05 onto Yoff, fp32 epilogue, TMA store)
//
// For a 16-token column group J lying wholly before the rows it meets, the
// decay factor is split as 2^(r_l - r_J) * [2^(r_J - r_s) dt_s] (r_J = r at the
// group's last token): one exponential per row and group, and one per token
// shared by every row.  Both factors are <= 1 when the log-decays never
// increase; a block where some head's cumsum does increase (A > 0 in some
// token) takes the per-element form everywhere.
//
// Precision as in the single-head kernel: every operand computed in-kernel (M,
// w o X, h) is contracted as a bf16 pair hi + lo against the exact bf16 input.
//
// Roles (one CTA per SM, persistent over its items c, c + grid, ...):
//   warps 0-15  compute: warp w works on TMEM lanes 32*(w%4).. (tile rows) and
//               the 16-column part w/4 of the state, Yoff, x, w o X and
//               output tiles (x is read from shared memory once, for w o X and D x)
//   warp 16     MMA issue (one elected lane, converged warp)
//   warp 17     TMA: operand loads (C, B double-buffered one block ahead), the
//               y stores, which it stages in the C/B buffers of the block just
//               finished
// The per-token decay terms are read by the compute warps themselves, one block
// ahead into registers, and turned into shared tables at the block's start.
// Every wait on an mbarrier is bounded (2 s); the first one that gives up sets
// the device error word and a CTA-wide abort word that ends every later wait
// at once, so the launch always finishes.  No inter-CTA waits exist.
//
// The Mamba-3 form (template flag M3) runs the whole Mamba-3 prefill in one
// scan.  Its B and C are the operands turned by the cumulative angle, which are
// no longer bf16 numbers; each comes as a bf16 pair hi + lo (groups 2g and
// 2g + 1 of the operand arrays), and every product with them is taken as
// hi x hi + hi x lo + lo x hi:
//   S      = C_hi B_hi^T + C_hi B_lo^T + C_lo B_hi^T
//   Yoff_k = C_hi h_hi + C_hi h_lo + C_lo h_hi
//   h_k'  += B_hi^T wX_hi + B_hi^T wX_lo + B_lo^T wX_hi
// (the lo x lo terms are about 2^-16 of the product and dropped).  The four
// operand tiles fill both C/B stages, so there is one stage: C of the next
// block is loaded once C h is done, B once the state MMAs are, and y goes
// from the registers straight to global memory instead of through a staging
// tile.  The trapezoid's weights w_s stand where dt_s stands in the forward;
// a token's own term takes lam_t dt_t instead (the diagonal of M, with the
// exact C_t . B_t of S's diagonal), and the final state is turned back by the
// last token's angle as it is written (rows 2k, 2k+1 are lanes of one warp).
#include "ssd_internal.h"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace pair {
using namespace ::ssd::tc;

constexpr int NS = 128;              // dstate of this kernel
constexpr int PD = 64;               // headdim of this kernel
constexpr int NCW = 16;              // compute warps
constexpr int NCT = NCW * 32;
constexpr int WARP_MMA = NCW, WARP_TMA = NCW + 1;
constexpr int THREADS = NCT + 64;

// TMEM columns (512 allocated)
constexpr uint32_t COL_R0 = 0;      // S (fp32), turned in place into M of head 0 (bf16 hi|lo per K step)
constexpr uint32_t COL_R1 = 128;    // M of head 1
constexpr uint32_t COL_Y = 256;     // + 64 k: C h_k scaled, then + M_k X_k (fp32)
constexpr uint32_t COL_ST = 384;    // + 64 k: state of head k (fp32, lane = state row)

// shared memory (tiles 1024-byte aligned, 128-byte swizzle)
constexpr uint32_t STAGE = 4 * TILE;             // C (K blocks 0, 1), B (K blocks 0, 1); later y staging
constexpr uint32_t OFF_X = 2 * STAGE;            // x of head 0, head 1
constexpr uint32_t OFF_W = OFF_X + 2 * TILE;     // per head: hi, lo of h (C h), then of w o X (state)
constexpr uint32_t TILES = OFF_W + 4 * TILE;
// per-token tables of the block (written by the compute warps; single buffer)
constexpr uint32_t OFF_V = TILES;                // [2][128] v_s = log2(dt_s) + r_J - r_s (J: end of s's 16-token group)
constexpr int NFAC = 96;                         // tokens whose group can lie before a row block
constexpr uint32_t OFF_FAC = OFF_V + 2 * SUB * 4;     // [2][96] 2^(v_s)
constexpr uint32_t OFF_GE = OFF_FAC + 2 * NFAC * 4;   // [2][8] float2: cumsum (hi, lo) at the group ends
constexpr uint32_t OFF_BAR = OFF_GE + 2 * 8 * 8;
enum { B_CB0, B_CB1, B_X, B_S, B_OFF, B_ST, B_Y0, B_Y, B_H, B_WX, B_M, B_EPI, B_STG0, B_STG1, NBAR };
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * NBAR;      // TMEM base, abort word
constexpr uint32_t SMEM = OFF_MISC + 16;
static_assert(TILES % 1024 == 0 && OFF_BAR % 8 == 0, "alignment");
static_assert(SMEM <= 232448, "shared memory per CTA");

struct Params {
    const float* dtw;          // [BH][Lpad] dt
    const float* acsw;         // [BH][Lpad] chunk-local inclusive cumsum of dt*A (hi part)
    const float* acslo;        // [BH][Lpad] its lo part, or NULL (= 0)
    const void* init_state;    // [BH][N][P] state dtype or NULL
    void* final_state;         // [BH][N][P] state dtype or NULL
    const float* D;            // [H] or NULL
    unsigned* dev_err;
    long long Lpad;
    int H, G, Q, nblk, npairs;
    int state_bf16, y_bf16;    // Mamba-3 form: state_bf16 bit 0 the final state's dtype, bit 1 the initial one's
    // the Mamba-3 form only (the struct stays within 128 bytes: a larger one costs
    // the kernel registers)
    const float* dgw;          // [BH][Lpad] weight of a token's own term (lam dt), or NULL (= the scan weight)
    const float2* rot;         // [b][G][NS/2] cos, sin of the last token's angle per pair
    void* y;                   // [b][L][H][PD] y dtype
    int L;
};
static_assert(sizeof(Params) <= 128, "kernel parameter struct");

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

// hi/lo bf16 pairs of 2 x 4 fp32 values (element 2e in the low half of word e)
__device__ __forceinline__ void split8(const float* v, uint32_t (&hw)[4], uint32_t (&lw)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        hw[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        lw[e] = pack_bf16(v[2 * e] - bf16_lo(hw[e]), v[2 * e + 1] - bf16_hi(hw[e]));
    }
}

// 18 warps, 5 of them on one SM sub-partition (16384 registers each): at most 96
// registers a thread, which the launch bounds give
template <bool M3>
__global__ void __launch_bounds__(THREADS, 1)
ssd_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY, const Params p) {
    extern __shared__ __align__(1024) uint8_t sm[];
    const uint32_t base = smem_u32(sm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
    auto bar = [&](int i) -> uint32_t { return base + OFF_BAR + 8u * (uint32_t)i; };

    // the 128-byte swizzle of TMA and of the MMA descriptors assumes 1024-byte aligned tiles
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
        //                          CB0 CB1 X  S  OFF ST Y0 Y  H    WX       M    EPI  STG0 STG1
        const uint32_t cnt[NBAR] = {1, 1, 1, 1, 1, 1, 1, 1, NCT, M3 ? NCT / 2 : NCT, NCT, NCT, NCT, NCT};
        for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), cnt[i]);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + OFF_MISC);

    // items of this CTA: blockIdx.x, + gridDim.x, ...; flat block counter jj over them
    const int nitems = p.npairs > (int)blockIdx.x ? (p.npairs - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = nitems * p.nblk;
    const int hpg = p.H / p.G;
    struct Item { int b, g, h0; };
    auto item_of = [&](int i) -> Item {
        const int it = (int)blockIdx.x + i * (int)gridDim.x;
        const int pr = it % (hpg >> 1), bg = it / (hpg >> 1);
        Item d;
        d.g = bg % p.G;
        d.b = bg / p.G;
        d.h0 = d.g * hpg + 2 * pr;
        return d;
    };
    unsigned err = 0;
    auto wait = [&](int i, uint32_t ph) {
        if (!wait_or_abort(bar(i), ph, s_abort)) err |= kErrAsyncTimeout;
    };

    if (warp == WARP_TMA && M3) {
        // ======================================================== TMA producer (Mamba-3 form)
        // one stage: C hi, C lo at tiles 0-3 (K blocks 0, 1 each), B hi, B lo at 4-7
        const uint32_t lead = elect_one();
        auto load_c = [&](int t) {           // C of block t (+ x and the turned B, C of block t + 1 into L2)
            const Item d = item_of(t / p.nblk);
            const int t0 = (t % p.nblk) * SUB;
            mbar_expect_tx(bar(B_CB0), 4 * TILE);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tma_load_4d(base + (uint32_t)i * TILE, &tmC, 64 * (i & 1), 2 * d.g + (i >> 1), t0, d.b, bar(B_CB0));
            if (t + 1 < total) {
                const Item dn = item_of((t + 1) / p.nblk);
                const int tn = ((t + 1) % p.nblk) * SUB;
                tma_prefetch_4d(&tmX, 0, dn.h0, tn, dn.b);
                tma_prefetch_4d(&tmX, 0, dn.h0 + 1, tn, dn.b);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    tma_prefetch_4d(&tmC, 64 * (i & 1), 2 * dn.g + (i >> 1), tn, dn.b);
                    tma_prefetch_4d(&tmB, 64 * (i & 1), 2 * dn.g + (i >> 1), tn, dn.b);
                }
            }
        };
        auto load_b = [&](int t) {
            const Item d = item_of(t / p.nblk);
            const int t0 = (t % p.nblk) * SUB;
            mbar_expect_tx(bar(B_CB1), 4 * TILE);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tma_load_4d(base + (uint32_t)(4 + i) * TILE, &tmB, 64 * (i & 1), 2 * d.g + (i >> 1), t0, d.b,
                            bar(B_CB1));
        };
        auto load_x = [&](int t) {
            const Item d = item_of(t / p.nblk);
            const int t0 = (t % p.nblk) * SUB;
            mbar_expect_tx(bar(B_X), 2 * TILE);
            tma_load_4d(base + OFF_X, &tmX, 0, d.h0, t0, d.b, bar(B_X));
            tma_load_4d(base + OFF_X + TILE, &tmX, 0, d.h0 + 1, t0, d.b, bar(B_X));
        };
        if (lead && total > 0) {
            load_c(0);
            load_b(0);
            load_x(0);
        }
        // C is free once C h is done (B_OFF), B once the state MMAs are (B_ST), x once Y is (B_Y)
        for (int jj = 0; jj + 1 < total; ++jj) {
            const uint32_t ph = jj & 1;
            wait(B_OFF, ph);
            if (lead && !*s_abort) load_c(jj + 1);
            wait(B_ST, ph);
            if (lead && !*s_abort) load_b(jj + 1);
            wait(B_Y, ph);
            if (lead && !*s_abort) load_x(jj + 1);
            __syncwarp();
        }
    } else if (warp == WARP_TMA) {
        // ======================================================== TMA producer
        const uint32_t lead = elect_one();
        auto load_cb = [&](int t) {          // C, B of block t into stage t & 1 (+ its x into L2)
            const Item d = item_of(t / p.nblk);
            const int t0 = (t % p.nblk) * SUB;
            const uint32_t st = base + (uint32_t)(t & 1) * STAGE, bb = bar(B_CB0 + (t & 1));
            mbar_expect_tx(bb, 4 * TILE);
            tma_load_4d(st, &tmC, 0, d.g, t0, d.b, bb);
            tma_load_4d(st + TILE, &tmC, 64, d.g, t0, d.b, bb);
            tma_load_4d(st + 2 * TILE, &tmB, 0, d.g, t0, d.b, bb);
            tma_load_4d(st + 3 * TILE, &tmB, 64, d.g, t0, d.b, bb);
            tma_prefetch_4d(&tmX, 0, d.h0, t0, d.b);
            tma_prefetch_4d(&tmX, 0, d.h0 + 1, t0, d.b);
        };
        auto load_x = [&](int t) {
            const Item d = item_of(t / p.nblk);
            const int t0 = (t % p.nblk) * SUB;
            mbar_expect_tx(bar(B_X), 2 * TILE);
            tma_load_4d(base + OFF_X, &tmX, 0, d.h0, t0, d.b, bar(B_X));
            tma_load_4d(base + OFF_X + TILE, &tmX, 0, d.h0 + 1, t0, d.b, bar(B_X));
        };
        if (lead && total > 0) {
            load_cb(0);
            if (total > 1) load_cb(1);
            load_x(0);
        }
        for (int jj = 0; jj < total; ++jj) {
            const uint32_t ph = jj & 1;
            wait(B_Y, ph);                   // the block's x is consumed
            if (lead && jj + 1 < total && !*s_abort) load_x(jj + 1);
            wait(B_STG0 + (jj & 1), (jj >> 1) & 1);   // y staged in the block's C/B stage
            if (lead && !*s_abort) {
                const Item d = item_of(jj / p.nblk);
                const int t0 = (jj % p.nblk) * SUB;
                const uint32_t st = base + (uint32_t)(jj & 1) * STAGE;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    tma_store_4d(&tmY, st + k * 2 * TILE, 0, d.h0 + k, t0, d.b);
                    if (!p.y_bf16) tma_store_4d(&tmY, st + k * 2 * TILE + TILE, 32, d.h0 + k, t0, d.b);
                }
                bulk_commit();
                bulk_wait_read0();           // the stage is free again
                if (jj + 2 < total) load_cb(jj + 2);
            }
            __syncwarp();
        }
        if (lead) bulk_wait0();
    } else if (warp == WARP_MMA) {
        // ======================================================== MMA issue
        const uint32_t lead = elect_one();
        constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);   // C (K-major) x B^T (K-major)
        constexpr uint32_t ID_Y = idesc_bf16(128, PD, false, true);     // M (TMEM) x X (MN-major)
        // both heads at once: N = 128 columns = [head 0 | head 1] of the W tiles,
        // whose 64-column halves lie 2 TILE apart (the leading byte offset)
        constexpr uint32_t ID_OFF = idesc_bf16(128, 2 * PD, false, true);   // C (K-major) x [h_0 | h_1] (MN-major)
        constexpr uint32_t ID_ST = idesc_bf16(128, 2 * PD, true, true);     // B^T (MN-major) x [wX_0 | wX_1]
        constexpr uint32_t KSTEP_K = 2, KBLOCK_K = TILE >> 4, KSTEP_MN = 2048 >> 4;
        const uint64_t dX0 = sdesc(base + OFF_X, TILE, 1024), dX1 = sdesc(base + OFF_X + TILE, TILE, 1024);
        const uint64_t dWhi = sdesc(base + OFF_W, 2 * TILE, 1024), dWlo = sdesc(base + OFF_W + TILE, 2 * TILE, 1024);
        const uint32_t lead0 = lead;
        for (int jj = 0; jj < total; ++jj) {
            const uint32_t ph = jj & 1;
            const uint32_t lead = lead0 && !*s_abort;     // once a wait gave up, issue nothing more
            // operand tiles: the stage of the block (C at tiles 0-1, B at 2-3); in
            // the Mamba-3 form the one stage, C hi / C lo / B hi / B lo at tiles 0 / 2 / 4 / 6
            const uint32_t st = M3 ? base : base + (uint32_t)(jj & 1) * STAGE;
            const uint32_t offB = M3 ? 4 * TILE : 2 * TILE;
            const uint64_t dC = sdesc(st, 16, 1024), dBk = sdesc(st + offB, 16, 1024);
            const uint64_t dBm = sdesc(st + offB, TILE, 1024);
            const uint64_t dCl = sdesc(st + 2 * TILE, 16, 1024), dBkl = sdesc(st + 6 * TILE, 16, 1024);
            const uint64_t dBml = sdesc(st + 6 * TILE, TILE, 1024);
            // ---- S = C B^T into R0 once the previous block's head-0 Y has read M_0 there
            if (M3) {
                wait(B_CB0, ph);
                wait(B_CB1, ph);
            } else {
                wait(B_CB0 + (jj & 1), (jj >> 1) & 1);
            }
            if (jj > 0) wait(B_Y0, ph ^ 1u);
            tc_fence_after();
            __syncwarp();
#pragma unroll
            for (int k = 0; k < NS / 16; ++k) {
                const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                if (k == 0) { if (lead) mma_ss<ID_S, 0>(tmem + COL_R0, dC + o, dBk + o);
                } else if (lead) mma_ss<ID_S, 1>(tmem + COL_R0, dC + o, dBk + o);
            }
            if (M3) {
#pragma unroll
                for (int k = 0; k < NS / 16; ++k) {
                    const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                    if (lead) mma_ss<ID_S, 1>(tmem + COL_R0, dC + o, dBkl + o);
                    if (lead) mma_ss<ID_S, 1>(tmem + COL_R0, dCl + o, dBk + o);
                }
            }
            if (lead) mma_commit(bar(B_S));
            // ---- Yoff_k = C h_k,hi + C h_k,lo (h written by the compute warps; the
            // previous epilogue has read the Y accumulators)
            wait(B_H, ph);
            if (jj > 0) wait(B_EPI, ph ^ 1u);
            tc_fence_after();
            __syncwarp();
#pragma unroll
            for (int k = 0; k < NS / 16; ++k) {
                const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                if (k == 0) { if (lead) mma_ss<ID_OFF, 0>(tmem + COL_Y, dC, dWhi);
                } else if (lead) mma_ss<ID_OFF, 1>(tmem + COL_Y, dC + o, dWhi + k * KSTEP_MN);
            }
#pragma unroll
            for (int k = 0; k < NS / 16; ++k) {
                const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                if (lead) mma_ss<ID_OFF, 1>(tmem + COL_Y, dC + o, dWlo + k * KSTEP_MN);
            }
            if (M3) {
#pragma unroll
                for (int k = 0; k < NS / 16; ++k) {
                    const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                    if (lead) mma_ss<ID_OFF, 1>(tmem + COL_Y, dCl + o, dWhi + k * KSTEP_MN);
                }
            }
            if (lead) mma_commit(bar(B_OFF));
            // ---- state_k += B^T (w o X_k)_hi + B^T (w o X_k)_lo, onto 2^(r_last) h_k
            wait(B_WX, ph);
            tc_fence_after();
            __syncwarp();
#pragma unroll
            for (int k = 0; k < SUB / 16; ++k)
                if (lead) mma_ss<ID_ST, 1>(tmem + COL_ST, dBm + k * KSTEP_MN, dWhi + k * KSTEP_MN);
#pragma unroll
            for (int k = 0; k < SUB / 16; ++k)
                if (lead) mma_ss<ID_ST, 1>(tmem + COL_ST, dBm + k * KSTEP_MN, dWlo + k * KSTEP_MN);
            if (M3) {
#pragma unroll
                for (int k = 0; k < SUB / 16; ++k)
                    if (lead) mma_ss<ID_ST, 1>(tmem + COL_ST, dBml + k * KSTEP_MN, dWhi + k * KSTEP_MN);
            }
            if (lead) mma_commit(bar(B_ST));
            // ---- Y_k += M_k,hi X_k + M_k,lo X_k onto the scaled Yoff (A from TMEM)
            wait(B_M, ph);
            tc_fence_after();
            __syncwarp();
#pragma unroll
            for (int k = 0; k < SUB / 16; ++k) {
                if (lead) mma_ts<ID_Y, 1>(tmem + COL_Y, tmem + COL_R0 + 16 * k, dX0 + k * KSTEP_MN);
                if (lead) mma_ts<ID_Y, 1>(tmem + COL_Y, tmem + COL_R0 + 16 * k + 8, dX0 + k * KSTEP_MN);
            }
            if (lead) mma_commit(bar(B_Y0));
#pragma unroll
            for (int k = 0; k < SUB / 16; ++k) {
                if (lead) mma_ts<ID_Y, 1>(tmem + COL_Y + 64, tmem + COL_R1 + 16 * k, dX1 + k * KSTEP_MN);
                if (lead) mma_ts<ID_Y, 1>(tmem + COL_Y + 64, tmem + COL_R1 + 16 * k + 8, dX1 + k * KSTEP_MN);
            }
            if (lead) mma_commit(bar(B_Y));
            __syncwarp();
        }
    } else {
        // ======================================================== compute warps
        const int q = warp & 3, kq = warp >> 2;       // lane quarter, 16-column part
        const int row = 32 * q + lane;                // TMEM lane = tile row
        const uint32_t lo16 = (uint32_t)(32 * q) << 16;
        const float NEG_INF = __int_as_float(0xff800000u);
        float* s_v = reinterpret_cast<float*>(sm + OFF_V);           // [2][128]
        float* s_fac = reinterpret_cast<float*>(sm + OFF_FAC);       // [2][96]
        float2* s_ge = reinterpret_cast<float2*>(sm + OFF_GE);       // [2][8]
        // the workspace's dt and cumsum come from the decay kernel this launch may overlap
        asm volatile("griddepcontrol.wait;" ::: "memory");

        // the cumsum of (bh, token t) as its (hi, lo) pair
        auto cum = [&](long long bh, long long t) -> float2 {
            const long long o = bh * p.Lpad + t;
            return make_float2(__ldcg(p.acsw + o), p.acslo ? __ldcg(p.acslo + o) : 0.f);
        };
        // log2 of exp(a - b) for two cumsum pairs: the hi difference is exact when it is
        // small next to the values, the only case where the factor is not negligible
        auto dl2 = [](float2 a, float2 b) -> float { return ((a.x - b.x) + (a.y - b.y)) * LOG2E; };

        // h entering a block, for both heads: the initial state (first block of an
        // item) or the state the previous block left in TMEM.  2^(r_last) h goes back
        // into the state accumulator; h is split hi -> W tile, lo -> W tile + TILE for C h.
        auto h_enter = [&](bool first, long long bh, const float (&rlast)[2]) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                uint32_t hv[16];
                if (!first) {
                    tmem_ld16(tmem + lo16 + COL_ST + 64 * k + 16 * kq, hv);
                    tmem_wait_ld();
                } else if (p.init_state) {
                    float f[16];
                    const long long o = ((bh + k) * NS + row) * PD + 16 * kq;
                    if (M3 ? (p.state_bf16 & 2) : p.state_bf16) {
                        Vec16<bf16>::load(reinterpret_cast<const bf16*>(p.init_state) + o, f);
                        Vec16<bf16>::load(reinterpret_cast<const bf16*>(p.init_state) + o + 8, f + 8);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            Vec16<float>::load(reinterpret_cast<const float*>(p.init_state) + o + i, f + i);
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) hv[i] = __float_as_uint(f[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) hv[i] = 0u;
                }
                const float dl = ex2(rlast[k]);
                const f32x2 dl2v = f2_pack(dl, dl);
                uint32_t sc[16], hw[8], lw[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const f32x2 h2 = f2_pack_u(hv[2 * i], hv[2 * i + 1]);
                    float a, b;
                    f2_unpack(f2_mul(dl2v, h2), a, b);
                    sc[2 * i] = __float_as_uint(a);
                    sc[2 * i + 1] = __float_as_uint(b);
                    split2(h2, hw[i], lw[i]);
                }
                tmem_st16(tmem + lo16 + COL_ST + 64 * k + 16 * kq, sc);
                uint8_t* wt = sm + OFF_W + k * 2 * TILE;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const uint32_t o = swz(row, 2 * kq + qq);
                    *reinterpret_cast<uint4*>(wt + o) = make_uint4(hw[4 * qq], hw[4 * qq + 1], hw[4 * qq + 2], hw[4 * qq + 3]);
                    *reinterpret_cast<uint4*>(wt + TILE + o) =
                        make_uint4(lw[4 * qq], lw[4 * qq + 1], lw[4 * qq + 2], lw[4 * qq + 3]);
                }
            }
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(bar(B_H));
        };

        // this thread's per-token data of a block, read from the workspace one block
        // ahead: the cumsum of its row's token for both heads; for the table threads
        // (kq < 2: head kq, token = row) also dt and the cumsum of the token before
        // (Mamba-3 form: also the weight of its row's own term for both heads)
        struct Pre { float2 row[2]; float dt; float2 prev; float dg[M3 ? 2 : 1]; };
        auto fetch = [&](const Item& dd, int jb, Pre& r) {
            const long long bh = (long long)dd.b * p.H + dd.h0;
            const long long t = (long long)jb * SUB + row;
            r.row[0] = cum(bh, t);
            r.row[1] = cum(bh + 1, t);
            if (M3 && p.dgw) {
                r.dg[0] = __ldcg(p.dgw + bh * p.Lpad + t);
                r.dg[M3 ? 1 : 0] = __ldcg(p.dgw + (bh + 1) * p.Lpad + t);
            }
            if (kq < 2) {
                r.dt = __ldcg(p.dtw + (bh + kq) * p.Lpad + t);
                r.prev = row ? cum(bh + kq, t - 1) : make_float2(0.f, 0.f);
            }
        };

        // Mamba-3 form (whose epilogue holds more registers): w o X by quarters 0 and 1,
        // one token row of one head per thread, read from the x tiles
        auto do_wx = [&](uint32_t ph) {
            wait(B_X, ph);
            const int t = kq * 64 + q * 32 + lane;
            const int s_ = t & (SUB - 1), k = t >> 7;
            const float wv = ex2(dl2(s_ge[k * 8 + 7], s_ge[k * 8 + (s_ >> 4)]) + s_v[k * SUB + s_]);
            const f32x2 w2 = f2_pack(wv, wv);
            const uint8_t* xt = sm + OFF_X + k * TILE;
            uint8_t* wt = sm + OFF_W + k * 2 * TILE;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t o = swz(s_, c);
                const uint4 xv = *reinterpret_cast<const uint4*>(xt + o);
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) split2(f2_mul(bf16x2_to_f2(xw[e]), w2), hw[e], lw[e]);
                *reinterpret_cast<uint4*>(wt + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(wt + TILE + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            fence_proxy_async();
            mbar_arrive(bar(B_WX));
        };

        float2 ref[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};   // cumsum at the previous block's end
        int it = 0, j = 0;
        Item d = total > 0 ? item_of(0) : Item{};
        Pre cur{};
        if (total > 0) fetch(d, 0, cur);
        for (int jj = 0; jj < total; ++jj) {
            const uint32_t ph = jj & 1;
            const bool chunk_start = ((j * SUB) & (p.Q - 1)) == 0;   // the cumsum restarts at every chunk
            const long long bh0 = (long long)d.b * p.H + d.h0;
            int it_n = it, j_n = j + 1;
            if (j_n == p.nblk) { j_n = 0; ++it_n; }
            const bool has_next = jj + 1 < total;
            const Item d_n = has_next ? (j_n == 0 ? item_of(it_n) : d) : d;
            const long long bh0_n = (long long)d_n.b * p.H + d_n.h0;

            // ---- per-token tables of the block.  Token s of head k: v_s = log2(dt_s)
            // + log2 exp(acs_J - acs_s) with J the last token of s's 16-token group,
            // and 2^(v_s); the cumsum pairs at the group ends
            float2 r0[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) r0[k] = chunk_start ? make_float2(0.f, 0.f) : ref[k];
            uint32_t inc = 0;                 // a log-decay that increases somewhere in the block
            if (kq < 2) {
                // head kq; selected, not indexed, so that the registers stay registers
                const int k = kq;
                const float2 me = k ? cur.row[1] : cur.row[0];
                const float2 r0k = k ? r0[1] : r0[0];
                inc = dl2(me, row ? cur.prev : r0k) > 0.f;
                const float2 ge = make_float2(__shfl_sync(0xffffffffu, me.x, lane | 15),
                                              __shfl_sync(0xffffffffu, me.y, lane | 15));
                const float v = (cur.dt > 0.f ? __log2f(cur.dt) : NEG_INF) + dl2(ge, me);
                s_v[k * SUB + row] = v;
                if (row < NFAC) s_fac[k * NFAC + row] = ex2(v);
                if ((row & 15) == 15) s_ge[k * 8 + (row >> 4)] = me;
            }
            uint32_t direct;
            asm volatile("{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.or.pred po, 1, %2, pi;\n"
                         " selp.u32 %0, 1, 0, po;\n}\n"
                         : "=r"(direct) : "r"(inc), "n"(NCT) : "memory");
            float rl[2], rlast[2];            // log2 decay of this row / of the whole block from its start
            float2 g127[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                g127[k] = s_ge[k * 8 + 7];
                rl[k] = dl2(cur.row[k], r0[k]);
                rlast[k] = dl2(g127[k], r0[k]);
            }
            if (jj == 0) h_enter(true, bh0, rlast);   // later blocks: entered during the previous one

            // ---- M_k = S o [s<=l] 2^(r_l - r_s) dt_s, written as bf16 hi/lo per K step:
            // hi to columns [16g, 16g+8), lo to [16g+8, 16g+16) of R0 (head 0, in place
            // over S) and R1 (head 1).  Quarter q needs column groups g < 2q+2; the
            // rest is zero.  Groups g < 2q lie before every row of the quarter:
            // factor 2^(r_l - r_J) 2^(v_s); the others 2^(r_l - r_J + v_s), masked.
            wait(B_S, ph);
            tc_fence_after();
#pragma unroll
            for (int gi = 0; gi < 2; ++gi) {
                const int g = kq + 4 * gi;
                const uint32_t c0 = 16u * (uint32_t)g;
                if (g >= 2 * q + 2) {
                    uint32_t z[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) z[i] = 0u;
                    tmem_st16(tmem + lo16 + COL_R0 + c0, z);
                    tmem_st16(tmem + lo16 + COL_R1 + c0, z);
                    continue;
                }
                uint32_t v[16];
                tmem_ld16(tmem + lo16 + COL_R0 + c0, v);
                tmem_wait_ld();
                const bool before = g < 2 * q && !direct;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float lf = dl2(cur.row[k], s_ge[k * 8 + g]);   // log2 decay from the group end to the row
                    uint32_t o[16];
                    if (before) {
                        const float f = ex2(lf);
                        const f32x2 ff = f2_pack(f, f);
                        const float4* fb = reinterpret_cast<const float4*>(s_fac + k * NFAC + c0);
#pragma unroll
                        for (int i4 = 0; i4 < 4; ++i4) {
                            const float4 bv = fb[i4];
                            const f32x2 w01 = f2_mul(ff, f2_pack(bv.x, bv.y)), w23 = f2_mul(ff, f2_pack(bv.z, bv.w));
                            split2(f2_mul(f2_pack_u(v[4 * i4], v[4 * i4 + 1]), w01), o[2 * i4], o[8 + 2 * i4]);
                            split2(f2_mul(f2_pack_u(v[4 * i4 + 2], v[4 * i4 + 3]), w23), o[2 * i4 + 1], o[9 + 2 * i4]);
                        }
                    } else {
                        const float4* vv = reinterpret_cast<const float4*>(s_v + k * SUB + c0);
#pragma unroll
                        for (int i4 = 0; i4 < 4; ++i4) {
                            const float4 uv = vv[i4];
                            const float ub[4] = {uv.x, uv.y, uv.z, uv.w};
                            float e[4];
#pragma unroll
                            for (int t = 0; t < 4; ++t)
                                e[t] = ex2((int)c0 + 4 * i4 + t <= row ? lf + ub[t] : NEG_INF);
                            if (M3 && p.dgw) {
                                // the row's own token: lam dt in place of the scan weight
#pragma unroll
                                for (int t = 0; t < 4; ++t)
                                    if ((int)c0 + 4 * i4 + t == row) e[t] = cur.dg[M3 ? k : 0];
                            }
                            split2(f2_mul(f2_pack_u(v[4 * i4], v[4 * i4 + 1]), f2_pack(e[0], e[1])),
                                   o[2 * i4], o[8 + 2 * i4]);
                            split2(f2_mul(f2_pack_u(v[4 * i4 + 2], v[4 * i4 + 3]), f2_pack(e[2], e[3])),
                                   o[2 * i4 + 1], o[9 + 2 * i4]);
                        }
                    }
                    tmem_st16(tmem + lo16 + (k ? COL_R1 : COL_R0) + c0, o);
                }
            }

            // ---- after C h: w o X of this thread's row and 16 columns (both heads, from
            // the x it keeps for D x) into the W tiles; then Yoff scaled by 2^(r_l)
            wait(B_OFF, ph);
            tc_fence_after();
            if (M3 && q < 2) do_wx(ph);
            if (!M3 || q >= 2) wait(B_X, ph);
            uint32_t xr[2][8];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const uint4 xv = *reinterpret_cast<const uint4*>(sm + OFF_X + k * TILE + swz(row, 2 * kq + qq));
                    xr[k][4 * qq] = xv.x; xr[k][4 * qq + 1] = xv.y; xr[k][4 * qq + 2] = xv.z; xr[k][4 * qq + 3] = xv.w;
                }
            }
#pragma unroll
            for (int k = 0; k < 2 && !M3; ++k) {
                // w_s = 2^(r_last - r_s) dt_s for the row's token s
                const float wv = ex2(dl2(s_ge[k * 8 + 7], s_ge[k * 8 + (row >> 4)]) + s_v[k * SUB + row]);
                const f32x2 w2 = f2_pack(wv, wv);
                uint8_t* wt = sm + OFF_W + k * 2 * TILE;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) split2(f2_mul(bf16x2_to_f2(xr[k][4 * qq + e]), w2), hw[e], lw[e]);
                    const uint32_t o = swz(row, 2 * kq + qq);
                    *reinterpret_cast<uint4*>(wt + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4*>(wt + TILE + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
            if (!M3) {
                fence_proxy_async();
                mbar_arrive(bar(B_WX));
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                uint32_t v[16];
                tmem_ld16(tmem + lo16 + COL_Y + 64 * k + 16 * kq, v);
                tmem_wait_ld();
                const float el = ex2(rl[k]);
                const f32x2 e2 = f2_pack(el, el);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float a, b;
                    f2_unpack(f2_mul(e2, f2_pack_u(v[2 * i], v[2 * i + 1])), a, b);
                    v[2 * i] = __float_as_uint(a);
                    v[2 * i + 1] = __float_as_uint(b);
                }
                tmem_st16(tmem + lo16 + COL_Y + 64 * k + 16 * kq, v);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_M));
            // the next block's per-token data, while this block's MMAs run
            Pre nxt{};
            if (has_next) fetch(d_n, j_n, nxt);
            float2 t127n[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            if (has_next) {
                t127n[0] = cum(bh0_n, (long long)j_n * SUB + SUB - 1);
                t127n[1] = cum(bh0_n + 1, (long long)j_n * SUB + SUB - 1);
            }

            // ---- once this block's state MMAs are done: the final state (last block of
            // an item), then the next block's entering state -- ahead of this block's
            // output, so that its C h can follow Y at once
            if (has_next || j == p.nblk - 1) wait(B_ST, ph);
            tc_fence_after();
            if (j == p.nblk - 1 && p.final_state) {
                uint32_t sv[2][16];
                tmem_ld16(tmem + lo16 + COL_ST + 16 * kq, sv[0]);
                tmem_ld16(tmem + lo16 + COL_ST + 64 + 16 * kq, sv[1]);
                tmem_wait_ld();
                float2 cs = make_float2(1.f, 0.f);
                if (M3) cs = p.rot[((long long)d.b * p.G + d.g) * (NS / 2) + (row >> 1)];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float ho[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) ho[i] = __uint_as_float(sv[k][i]);
                    if (M3) {
                        // h = R(Theta_last) ~h: row 2k' -> c u - s w, row 2k'+1 -> s u + c w
                        // (u, w the rows 2k', 2k'+1 of the turned state: this lane and its neighbour)
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float other = __shfl_xor_sync(0xffffffffu, ho[i], 1);
                            ho[i] = (row & 1) ? fmaf(cs.y, other, cs.x * ho[i]) : fmaf(-cs.y, other, cs.x * ho[i]);
                        }
                    }
                    const long long o = ((bh0 + k) * NS + row) * PD + 16 * kq;
                    if (M3 ? (p.state_bf16 & 1) : p.state_bf16) {
                        bf16* fs = reinterpret_cast<bf16*>(p.final_state) + o;
                        Vec16<bf16>::store(fs, ho);
                        Vec16<bf16>::store(fs + 8, ho + 8);
                    } else {
                        float* fs = reinterpret_cast<float*>(p.final_state) + o;
#pragma unroll
                        for (int i = 0; i < 16; i += 4) Vec16<float>::store(fs + i, ho + i);
                    }
                }
            }
            if (has_next) {
                const bool cs_n = j_n == 0 || ((j_n * SUB) & (p.Q - 1)) == 0;
                float rlast_n[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) rlast_n[k] = dl2(t127n[k], cs_n ? make_float2(0.f, 0.f) : g127[k]);
                h_enter(j_n == 0, bh0_n, rlast_n);
            }

            // ---- after Y: y = Y + D x staged in the block's C/B stage (dead once every
            // MMA of the block is done) for the TMA store
            wait(B_Y, ph);
            tc_fence_after();
            uint32_t yv[2][16];
            tmem_ld16(tmem + lo16 + COL_Y + 16 * kq, yv[0]);
            tmem_ld16(tmem + lo16 + COL_Y + 64 + 16 * kq, yv[1]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(B_EPI));          // the Y accumulators may be reused
            const float Dk[2] = {p.D ? __ldg(p.D + d.h0) : 0.f, p.D ? __ldg(p.D + d.h0 + 1) : 0.f};
            if (M3) {
                // y = Y + D x straight from the registers (16 columns of the row per head).
                // fp32: the 16-byte pieces are first transposed within lane quads
                // (lane 4i+c then holds piece c of rows 4i..4i+3 of the warp), so that
                // each store instruction writes 8 rows of 64 contiguous bytes, not 32
                // rows of 16
                const long long t = (long long)j * SUB + row;
                const long long tq = (long long)j * SUB + 32 * q + (lane & ~3);
                const int jq = lane & 3;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float out[16];
                    const f32x2 dd = f2_pack(Dk[k], Dk[k]);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        f2_unpack(f2_fma(dd, bf16x2_to_f2(xr[k][e]), f2_pack_u(yv[k][2 * e], yv[k][2 * e + 1])),
                                  out[2 * e], out[2 * e + 1]);
                    if (p.y_bf16) {
                        if (t < p.L) {
                            bf16* yo = reinterpret_cast<bf16*>(p.y) + (((long long)d.b * p.L + t) * p.H + d.h0 + k) * PD +
                                       16 * kq;
                            Vec16<bf16>::store(yo, out);
                            Vec16<bf16>::store(yo + 8, out + 8);
                        }
                    } else {
                        float4 ch[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            ch[c] = make_float4(out[4 * c], out[4 * c + 1], out[4 * c + 2], out[4 * c + 3]);
                        // swap 2x2 blocks of pieces with lane ^ 2, then single pieces with lane ^ 1
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const bool hi = jq & 2;
                            const float4 v = hi ? ch[u] : ch[2 + u];
                            const float4 r = make_float4(__shfl_xor_sync(0xffffffffu, v.x, 2),
                                                         __shfl_xor_sync(0xffffffffu, v.y, 2),
                                                         __shfl_xor_sync(0xffffffffu, v.z, 2),
                                                         __shfl_xor_sync(0xffffffffu, v.w, 2));
                            if (hi) ch[u] = r; else ch[2 + u] = r;
                        }
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const bool odd = jq & 1;
                            const float4 v = odd ? ch[2 * u] : ch[2 * u + 1];
                            const float4 r = make_float4(__shfl_xor_sync(0xffffffffu, v.x, 1),
                                                         __shfl_xor_sync(0xffffffffu, v.y, 1),
                                                         __shfl_xor_sync(0xffffffffu, v.z, 1),
                                                         __shfl_xor_sync(0xffffffffu, v.w, 1));
                            if (odd) ch[2 * u] = r; else ch[2 * u + 1] = r;
                        }
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            if (tq + m < p.L) {
                                float* yo = reinterpret_cast<float*>(p.y) +
                                            (((long long)d.b * p.L + tq + m) * p.H + d.h0 + k) * PD + 16 * kq + 4 * jq;
                                *reinterpret_cast<float4*>(yo) = ch[m];
                            }
                        }
                    }
                }
                ref[0] = g127[0];
                ref[1] = g127[1];
                cur = nxt;
                it = it_n;
                j = j_n;
                d = d_n;
                continue;
            }
            uint8_t* stg = sm + (jj & 1) * STAGE;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                float out[16];
                const f32x2 dd = f2_pack(Dk[k], Dk[k]);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    f2_unpack(f2_fma(dd, bf16x2_to_f2(xr[k][e]), f2_pack_u(yv[k][2 * e], yv[k][2 * e + 1])),
                              out[2 * e], out[2 * e + 1]);
                uint8_t* tile = stg + k * 2 * TILE;
                if (p.y_bf16) {
#pragma unroll
                    for (int qq = 0; qq < 2; ++qq)
                        *reinterpret_cast<uint4*>(tile + swz(row, 2 * kq + qq)) = Vec16<bf16>::pack(out + 8 * qq);
                } else {
                    uint8_t* bx = tile + (kq >> 1) * TILE;     // columns 0-31 / 32-63: one box each
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(bx + swz(row, (kq & 1) * 4 + c)) = Vec16<float>::pack(out + 4 * c);
                }
            }
            fence_proxy_async();
            mbar_arrive(bar(B_STG0 + (jj & 1)));
            ref[0] = g127[0];
            ref[1] = g127[1];
            cur = nxt;
            it = it_n;
            j = j_n;
            d = d_n;
        }
    }

    if (err) atomicOr(p.dev_err, err);
    tc_fence_before();
    __syncthreads();
    // after a wait gave up, copies or MMAs issued before it may still be in flight:
    // let them drain (1 ms) before the shared memory and TMEM are released
    if (*s_abort) {
        const unsigned long long t_end = gtimer() + 1000000ull;
        while (gtimer() < t_end) __nanosleep(1000);
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

}  // namespace pair

bool pair_path_supports(int64_t batch, int64_t H, int64_t P, int64_t N, int64_t G, int64_t Q, bool io_bf16) {
    // enough head pairs for every item to be a whole sequence on a part of 148 SMs
    return io_bf16 && P == pair::PD && N == pair::NS && (Q == 128 || Q == 256) && (H / G) % 2 == 0 &&
           batch * H >= 148;
}

// m3: the Mamba-3 form, B and C then [b][L][G][2][N] (hi, lo of the turned operands)
static cudaError_t launch_pair(const PrefillArgs& a, bool m3, const float* dgw, const float2* rot, bool init_bf16,
                               cudaStream_t s) {
    using namespace pair;
    if (!pair_path_supports(a.batch, a.H, a.P, a.N, a.G, a.Q, a.io_bf16)) return cudaErrorNotSupported;
    CUtensorMap mx, mb, mc, my;
    const uint64_t gops = (uint64_t)a.G * (m3 ? 2 : 1);    // groups of the B, C arrays
    if (!tc::make_map(&my, a.y, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.batch, !a.y_bf16) ||
        !tc::make_map(&mx, a.x, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.batch) ||
        !tc::make_map(&mb, a.B, (uint64_t)a.N, gops, (uint64_t)a.L, (uint64_t)a.batch) ||
        !tc::make_map(&mc, a.C, (uint64_t)a.N, gops, (uint64_t)a.L, (uint64_t)a.batch))
        return cudaErrorInvalidValue;
    static std::mutex mu;
    static int sms_of[64][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!sms_of[dev][m3]) {
            e = cudaFuncSetAttribute(m3 ? ssd_pair_kernel<true> : ssd_pair_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
            if (e != cudaSuccess) return e;
            int sms = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            sms_of[dev][m3] = sms;
        }
    }
    Params p{};
    p.dtw = (const float*)(a.ws + a.lay.off_dt);
    p.acsw = (const float*)(a.ws + a.lay.off_acs);
    p.acslo = a.lay.has_lo ? (const float*)(a.ws + a.lay.off_acs_lo) : nullptr;
    p.init_state = a.init_state;
    p.final_state = a.final_state;
    p.D = a.D;
    p.dev_err = a.dev_err;
    p.Lpad = a.lay.Lpad;
    p.H = (int)a.H;
    p.G = (int)a.G;
    p.Q = (int)a.Q;
    p.nblk = (int)((a.L + SUB - 1) / SUB);
    const long long pairs = a.batch * a.H / 2;
    const long long blocks = pairs * p.nblk;
    if (pairs > 0x7fffffffLL || blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.npairs = (int)pairs;
    p.state_bf16 = m3 ? (a.state_bf16 ? 1 : 0) | (init_bf16 ? 2 : 0) : a.state_bf16;
    p.y_bf16 = a.y_bf16;
    p.dgw = dgw;
    p.rot = rot;
    p.y = a.y;
    if (a.L > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.L = (int)a.L;
    const unsigned grid = (unsigned)(pairs < sms_of[dev][m3] ? pairs : sms_of[dev][m3]);
    // a programmatic dependent of the decay-cumsum kernel before it on the stream:
    // the prologue and the first operand loads overlap that kernel; the producer
    // waits for it (griddepcontrol.wait) before it reads dt and the cumsum
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return m3 ? cudaLaunchKernelEx(&cfg, ssd_pair_kernel<true>, mx, mb, mc, my, p)
              : cudaLaunchKernelEx(&cfg, ssd_pair_kernel<false>, mx, mb, mc, my, p);
}

cudaError_t launch_prefill_pair(const PrefillArgs& a, cudaStream_t s) {
    return launch_pair(a, false, nullptr, nullptr, a.state_bf16, s);
}

cudaError_t launch_prefill_pair_mamba3(const PrefillArgs& a, const float* dgw, const float2* rot, bool init_bf16,
                                       cudaStream_t s) {
    if (a.final_state && !rot) return cudaErrorInvalidValue;
    return launch_pair(a, true, dgw, rot, init_bf16, s);
}

}  // namespace ssd
