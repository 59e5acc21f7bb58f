// Tensor-core prefill of the SSD layer core for sm_100a: tcgen05 MMAs with
// TMEM accumulators, operands staged by TMA, fp32 state passing between
// runs of chunks through a chained (ticketed) hand-off.
//
// The chunked contraction of the semiseparable matrix ("Mamba-2 vs
// Transformers / SSD", section "Mamba-2 and the SSD paper: what changed in
// practice": chunks processed in parallel, per-chunk states recombined; its
// table: "Blocked two-pass contraction ... tensor-core-friendly tiled
// execution").  One CTA handles one work item = (batch b, chunk c, head h);
// the chunk's Q tokens are walked in blocks of 128 (the MMA M dimension).
// Per 128-token block, with r_l = (chunk-local decay cumsum) * log2(e)
// relative to the block start:
//
//   S    = C B^T                      (tcgen05, A=C K-major, B=B K-major, fp32 in TMEM)
//   M    = S o [s<=l] 2^(r_l-r_s) dt_s   (CUDA cores, TMEM -> regs -> TMEM in place)
//   Y    = M X                        (tcgen05, A=M from TMEM, B=X MN-major)
//   S_c  = B^T (w o X), w_s = 2^(r_last-r_s) dt_s     (tcgen05, A=B MN-major)
//   h'   = 2^(r_last) h + S_c          (fp32, CUDA cores; the inter-chunk scan)
//   Yoff = C h                         (tcgen05, A=C K-major, B=h MN-major)
//   y    = Y + 2^(r_l) Yoff + D x      (fp32 epilogue, staged in smem, TMA store)
//
// Precision: the operands computed in-kernel (M, w o X, h) are split into a
// bf16 pair hi + lo (hi = bf16(v), lo = bf16(v - hi)) and contracted with two
// MMAs against the exact bf16 input operand, accumulating in fp32.  That keeps
// about 16 significant bits in every product; a single bf16 rounding of those
// operands gives max|err|/rms(y) of ~0.14 on the 1.3B-shaped workload, whose
// outputs reach 60x their rms (tokens with large dt).  C B^T uses the exact
// inputs and needs one pass.
//
// Work items and state passing: a work item is one (b, h) sequence, or a run of
// K consecutive chunks of it when there are too few sequences to fill the
// block pipelines.  With runs, every run after the first needs the state that
// enters it, so the ticket stream first hands out state items (run r < nruns-1
// of a sequence: only the chunk-state MMAs, from a zero state, giving the
// run's own contribution dS_r and its total decay R_r), then output items (run
// r: the whole block chain from the entry state h_in(r)).  A state item ends
// with the one sequential step, h_in(r+1) = 2^(R_r) h_in(r) + dS_r, for which
// it waits (bounded) until flags[b,h] >= r, i.e. until state item r-1 has
// published h_in(r); it then writes h_in(r+1) to its fp32 slot and sets
// flags[b,h] = r+1.  An output item r > 0 waits for flags[b,h] >= r before its
// first block.  Tickets are handed out in order and an item only ever waits for
// an item with an earlier ticket, which is running or done and waits only on
// earlier ones: no cycle.  A CTA allocates TMEM before taking a ticket, so a
// ticket holder never waits for TMEM.  Every wait is bounded by a 2 s
// globaltimer deadline.  A hand-off wait that expires sets the device error
// word and a launch-wide abort word that ends every other hand-off wait at
// once; the CTA then finishes its (in-bounds) work -- still waiting for its own
// TMA and MMA completions -- and frees its TMEM.  Nothing traps.
#include "ssd_internal.h"
#include "ssd_tc_common.cuh"

namespace ssd {
namespace tc {

constexpr int PD = 64;          // headdim handled by this path
constexpr int NCOMPUTE = 256;   // compute threads of a pipeline: 8 warps; warps w and w+4 share TMEM lanes 32*(w%4)..+31
// thread layout: warps 8p..8p+7 compute for pipeline p, then one control warp per
// pipeline.  A warp may only touch TMEM lanes 32*(warp % 4), so compute warps
// must start at a multiple of 4 warps: they come first.

// TMEM columns of a pipeline
constexpr uint32_t COL_R = 0;     // S (fp32 128) -> M hi|lo (bf16x2 64+64)
constexpr uint32_t COL_Y = 128;   // Yoff, then Y (fp32 64)
constexpr uint32_t COL_ST = 192;  // chunk-state accumulator: fp32 64 per 128 state rows (lane = n % 128)

// control words after the per-(b,h) flags
constexpr int CTRL_TICKET = 0;
constexpr int CTRL_ABORT = 1;

// dstate N = 64, 128 or 256.  dstate 64 keeps the layout of 128 with B
// zero-padded: its chunk state is an M=128 MMA whose upper 64 rows stay zero,
// while C B^T and C h take only the 4 valid K steps.  dstate 256 needs 208 KB of
// tiles, so it runs one pipeline per CTA, with the state in two 128-row halves.
template <int N>
struct Cfg {
    static constexpr int NP = N < 128 ? 128 : N;            // state rows held (padded)
    static constexpr int KB = NP / 64;                      // 64-wide K blocks of C, B in smem
    static constexpr int KBV = N / 64;                      // ... of them loaded (the rest stays zero)
    static constexpr int NB = NP / 128;                     // 128-row blocks of the state
    static constexpr int PIPES = N > 128 ? 1 : 2;           // block pipelines per CTA (one CTA per SM)
    static constexpr int THREADS = PIPES * (NCOMPUTE + 32);
    static constexpr uint32_t PIPE_COLS = COL_ST + 64 * NB <= 256 ? 256 : 512;   // TMEM columns of a pipeline
    static constexpr uint32_t TMEM_COLS = PIPES * PIPE_COLS;
    static_assert(TMEM_COLS <= 512, "TMEM");
    // tiles of one pipeline (1024-byte aligned, 128-byte swizzle)
    static constexpr uint32_t OFF_C = 0;
    static constexpr uint32_t OFF_B = OFF_C + KB * TILE;
    static constexpr uint32_t OFF_X = OFF_B + KB * TILE;
    // W1/W2: hi/lo halves of w o X, then of h (MN-major operands), then the y staging tile
    static constexpr uint32_t W_BYTES = NP * 128;
    static constexpr uint32_t OFF_W1 = OFF_X + TILE;
    static constexpr uint32_t OFF_W2 = OFF_W1 + W_BYTES;
    static constexpr uint32_t TILES = OFF_W2 + W_BYTES;
    // small area of one pipeline (after the tiles of all pipelines)
    static constexpr uint32_t OFF_ACS = 0;                   // chunk-local cumsum of the block [128] (TMA)
    static constexpr uint32_t OFF_DTCS = OFF_ACS + 512;      // dt [128] (TMA), turned into log2(dt_s) - r_s
    static constexpr uint32_t OFF_BAR = OFF_DTCS + 512;      // mbarriers (10)
    static constexpr uint32_t OFF_MISC = OFF_BAR + 80;       // tmem base, block coordinates
    static constexpr uint32_t SMALL = OFF_MISC + 64;
    static constexpr uint32_t SMEM = PIPES * (TILES + SMALL);
    static constexpr uint32_t TX = (2 * KBV + 1) * TILE + 2 * SUB * 4;   // TMA bytes per block
    static constexpr uint32_t TX_ST = (KBV + 1) * TILE + 2 * SUB * 4;    // ... of a state item (no C)
    static_assert(TILES % 1024 == 0 && SMALL % 16 == 0, "alignment");
    static_assert(SMEM <= 232448, "shared memory per CTA");
};

struct Params {
    const float* dtw;       // [BH][Lpad]
    const float* acsw;      // [BH][Lpad] chunk-local inclusive cumsum of dt*A
    float* slots;           // [BH][nruns-1][N][PD] fp32 entry states of runs 1..nruns-1
    int* flags;             // [BH] chunks published, then control words
    const void* init_state; // [BH][N][PD] state dtype or NULL
    void* final_state;      // [BH][N][PD] state dtype or NULL
    void* y;                // [b][L][H][PD] y dtype
    const float* D;         // [H] or NULL
    unsigned* dev_err;
    long long L, Lpad;
    int H, G, Q, nchunks, BH;
    int K, nruns;           // a run = K consecutive chunks of one (b, h)
    int nstate;             // state items ((nruns - 1) * BH), ahead of the nruns * BH output items
    int state_bf16, y_bf16;
    int drop_publish;       // test hook: state items never publish (their successors time out)
};


// ---------------------------------------------------------------- the kernel
// Persistent, one CTA per SM, Cfg::PIPES independent block pipelines per CTA.  A
// pipeline = 8 compute warps (256 threads; thread = one TMEM lane/tile row and
// one half of its columns) + 1 control warp, converged, whose elected lane
// takes tickets, issues every TMA and MMA, waits for run-entry states and
// publishes them.  Compute and control meet only at mbarriers; a state item
// still completes every barrier once per block, so phases stay in step.
//
// Per 128-token block the state accumulator (TMEM) is first loaded with
// 2^(r_last) h and the chunk-state MMAs accumulate onto it, so h' stays in
// TMEM for the next block of the item; C h is computed first into the Y
// accumulator, scaled by 2^(r_l) in place, and M X accumulates on top.  Region
// R only holds S/M, so the next block's loads and C B^T start as soon as Y is
// done, overlapping this block's epilogue.
// RUNS: sequences are cut into runs (state items and run hand-offs present)
template <int N, bool RUNS>
__global__ void __launch_bounds__(Cfg<N>::THREADS, 1)
ssd_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY, const Params p) {
    using K = Cfg<N>;
    static_assert(N == 64 || N == 128 || N == 256, "dstate 64, 128 or 256");
    constexpr int PIPES = K::PIPES;
    extern __shared__ __align__(1024) uint8_t smem_all[];
    const bool control = threadIdx.x >= PIPES * NCOMPUTE;   // a pipeline's control warp
    const int pipe = control ? (threadIdx.x - PIPES * NCOMPUTE) / 32 : threadIdx.x / NCOMPUTE;
    uint8_t* sm = smem_all + pipe * K::TILES;         // the pipeline's own tiles
    uint8_t* ss = smem_all + PIPES * K::TILES + pipe * K::SMALL;   // and its small area
    const uint32_t base = smem_u32(sm);
    const uint32_t sbase = smem_u32(ss);
    const uint32_t base_all = smem_u32(smem_all);
    const int tid = threadIdx.x % NCOMPUTE;           // compute thread index within its pipeline
    const int warp = tid >> 5, lane = threadIdx.x & 31;
    const int half = (warp >> 2) & 1;                 // column half of the tiles
    const int row = (warp & 3) * 32 + lane;           // TMEM lane = tile row; warp % 4 == CTA warp % 4
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

    float* scs = reinterpret_cast<float*>(ss + K::OFF_DTCS);           // dt, then log2(dt) - r
    const float* s_acs = reinterpret_cast<const float*>(ss + K::OFF_ACS);
    volatile int* s_item = reinterpret_cast<volatile int*>(ss + K::OFF_MISC + 4);
    volatile int* s_j = reinterpret_cast<volatile int*>(ss + K::OFF_MISC + 8);
    uint8_t* s_tmem_slot = smem_all + PIPES * K::TILES + K::OFF_MISC;    // pipeline 0's misc word
    enum { BAR_TMA = 0, BAR_S, BAR_CHAIN, BAR_H, BAR_OFF, BAR_WX, BAR_M, BAR_Y, BAR_PUB, BAR_EPI, NBAR };
    auto bar = [&](int i) -> uint32_t { return sbase + K::OFF_BAR + 8u * (uint32_t)i; };
    volatile int* g_abort = reinterpret_cast<volatile int*>(p.flags + p.BH + CTRL_ABORT);
    const int total = p.nstate + p.nruns * p.BH;
    unsigned err = 0;

    // the 128-byte swizzle of TMA and of the MMA descriptors assumes 1024-byte
    // aligned tiles; refuse to run (and say so) if the runtime did not align
    if (base_all & 1023u) {
        if (threadIdx.x == 0) atomicOr(p.dev_err, kErrAsyncTimeout);
        return;
    }
    // TMEM first, then tickets (a ticket holder never waits for TMEM)
    if (threadIdx.x < 32) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(s_tmem_slot)), "r"(K::TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // dstate 64: the B tile of state rows 64..127 is never loaded; zero it once
    if (K::KBV < K::KB && !control) {
        uint4* z = reinterpret_cast<uint4*>(sm + K::OFF_B + K::KBV * TILE);
        for (int i = tid; i < (K::KB - K::KBV) * (int)TILE / 16; i += NCOMPUTE) z[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async();
    }
    if (!control && tid == 0) {
        //                        TMA S  CHAIN H         OFF WX        M         Y  PUB       EPI
        const uint32_t cnt[NBAR] = {1, 1, 1, NCOMPUTE, 1, NCOMPUTE, NCOMPUTE, 1, NCOMPUTE, NCOMPUTE};
        for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), cnt[i]);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the pipeline's 256 columns of the CTA's allocation (address = lane << 16 | column)
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(s_tmem_slot) + K::PIPE_COLS * pipe;
    auto wait = [&](int i, uint32_t ph) {
        if (!mbar_wait(bar(i), ph)) err |= kErrAsyncTimeout;
    };
    // ticket -> (state item?, run r (chunks [rK, rK+K)), sequence bh); both kinds
    // are run-major, so item r-1 of a sequence holds an earlier ticket than item r
    struct Item { int st, r, bh; };
    auto decode = [&](int it) -> Item {
        Item d;
        d.st = RUNS && it < p.nstate;
        const int k = d.st ? it : it - p.nstate;
        d.r = k / p.BH;
        d.bh = k % p.BH;
        return d;
    };
    auto nblocks = [&](int it) -> int {       // 128-token blocks of the run (never straddle a chunk)
        const long long t_first = (long long)decode(it).r * p.K * p.Q;
        const long long len = p.L - t_first < (long long)p.K * p.Q ? p.L - t_first : (long long)p.K * p.Q;
        return (int)((len + SUB - 1) / SUB);
    };
    auto slot_of = [&](int bh, int r) -> float* {   // entry state of run r >= 1
        return p.slots + (long long)(bh * (p.nruns - 1) + r - 1) * N * PD;
    };

    if (control) {
        // ==================================================== control warp
        {
            const uint32_t lead = elect_one();
            constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);   // C (K-major) x B^T (K-major)
            constexpr uint32_t ID_ST = idesc_bf16(128, PD, true, true);     // B^T (MN-major) x wX (MN-major)
            constexpr uint32_t ID_Y = idesc_bf16(128, PD, false, true);     // M (TMEM) x X (MN-major)
            constexpr uint32_t ID_OFF = idesc_bf16(128, PD, false, true);   // C (K-major) x h (MN-major)
            // Shared-memory descriptors, built once: a K step of a K-major operand
            // advances the start address by 32 B (+2 in the descriptor), a 64-wide
            // K block by one tile (+TILE/16); a K step of an MN-major operand by 16
            // rows of 128 B (+128).  The 14-bit address field cannot overflow:
            // every shared address is below 2^18.
            const uint64_t dC = sdesc(base + K::OFF_C, 16, 1024);       // K-major (S, Yoff)
            const uint64_t dBk = sdesc(base + K::OFF_B, 16, 1024);      // K-major (S)
            const uint64_t dBm = sdesc(base + K::OFF_B, TILE, 1024);    // MN-major (state)
            const uint64_t dX = sdesc(base + K::OFF_X, TILE, 1024);     // MN-major (Y)
            const uint64_t dW1 = sdesc(base + K::OFF_W1, TILE, 1024);   // MN-major (state, Yoff)
            const uint64_t dW2 = sdesc(base + K::OFF_W2, TILE, 1024);
            constexpr uint32_t KSTEP_K = 2, KBLOCK_K = TILE >> 4, KSTEP_MN = 2048 >> 4;
            // chunk-state MMAs: onto the state accumulator, B^T (w o X)_hi and
            // B^T (w o X)_lo (K = 128 tokens), one M=128 MMA per 128 state rows
            auto issue_state = [&]() {
#pragma unroll
                for (int nb = 0; nb < K::NB; ++nb) {
                    const uint64_t a0 = dBm + (uint64_t)((2u * TILE * nb) >> 4);   // B tiles 2nb, 2nb+1
#pragma unroll
                    for (int k = 0; k < SUB / 16; ++k)
                        if (lead) mma_ss<ID_ST, 1>(tmem + COL_ST + 64 * nb, a0 + k * KSTEP_MN, dW1 + k * KSTEP_MN);
#pragma unroll
                    for (int k = 0; k < SUB / 16; ++k)
                        if (lead) mma_ss<ID_ST, 1>(tmem + COL_ST + 64 * nb, a0 + k * KSTEP_MN, dW2 + k * KSTEP_MN);
                }
            };
            // publish the block's coordinates, then load its operands and per-token terms
            auto load_block = [&](int it, int j) {
                __syncwarp();
                if (lead) {
                    *s_item = it;
                    *s_j = j;
                }
                __syncwarp();
                if (it >= total) {                      // no more work: release the compute warps
                    if (lead) mbar_arrive(bar(BAR_TMA));
                    return;
                }
                if (!lead) return;
                const Item d_ = decode(it);
                const int bh_ = d_.bh;
                const int b_ = bh_ / p.H, h_ = bh_ % p.H, g_ = h_ / (p.H / p.G);
                const int t0_ = d_.r * p.K * p.Q + j * SUB;
                fence_proxy_async();
                mbar_expect_tx(bar(BAR_TMA), d_.st ? K::TX_ST : K::TX);   // a state item needs no C
#pragma unroll
                for (int kb = 0; kb < K::KBV; ++kb) {
                    if (!d_.st) tma_load_4d(base + K::OFF_C + kb * TILE, &tmC, kb * 64, g_, t0_, b_, bar(BAR_TMA));
                    tma_load_4d(base + K::OFF_B + kb * TILE, &tmB, kb * 64, g_, t0_, b_, bar(BAR_TMA));
                }
                tma_load_4d(base + K::OFF_X, &tmX, 0, h_, t0_, b_, bar(BAR_TMA));
                const long long o = (long long)bh_ * p.Lpad + t0_;
                bulk_load(sbase + K::OFF_ACS, p.acsw + o, SUB * 4, bar(BAR_TMA));
                bulk_load(sbase + K::OFF_DTCS, p.dtw + o, SUB * 4, bar(BAR_TMA));
                // the next block of the item into L2 while this one is processed
                if (j + 1 < nblocks(it)) {
#pragma unroll
                    for (int kb = 0; kb < K::KBV; ++kb) {
                        if (!d_.st) tma_prefetch_4d(&tmC, kb * 64, g_, t0_ + SUB, b_);
                        tma_prefetch_4d(&tmB, kb * 64, g_, t0_ + SUB, b_);
                    }
                    tma_prefetch_4d(&tmX, 0, h_, t0_ + SUB, b_);
                }
            };
            // this launch may start while the decay-cumsum kernel before it is still
            // running (programmatic dependent launch): wait for it to finish -- its
            // dt, cumsum and reset flags -- before the first ticket
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int item = 0;
            if (lead) item = atomicAdd(p.flags + p.BH + CTRL_TICKET, 1);
            item = __shfl_sync(0xffffffffu, item, __ffs(__ballot_sync(0xffffffffu, lead)) - 1);
            int j = 0;
            load_block(item, 0);
            uint32_t blk = 0;
            // bounded wait until sequence bh has published the entry state of run r
            auto chain_wait = [&](int bh, int r) {
                const int* f = p.flags + bh;
                const unsigned long long deadline = gtimer() + WAIT_NS;
                uint32_t spins = 0;
                while (true) {
                    int v;
                    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
                    if (v >= r) break;
                    if (*g_abort) { err |= kErrChainAborted; break; }
                    if ((++spins & 255u) == 0 && gtimer() > deadline) {
                        err |= kErrChainTimeout;
                        atomicExch(p.flags + p.BH + CTRL_ABORT, 1);
                        break;
                    }
                    __nanosleep(64);
                }
            };
            while (item < total) {
                const uint32_t ph = blk & 1u;
                const Item d = decode(item);
                const bool last_block = (j == nblocks(item) - 1);
                wait(BAR_TMA, ph);
                tc_fence_after();
                __syncwarp();
                if (d.st) {
                    // ---- state item: only the chunk-state MMAs (no S, Yoff, M, Y or y);
                    // the barriers of the skipped steps still complete once per block
                    if (lead) mbar_arrive(bar(BAR_S));
                    if (blk > 0) wait(BAR_EPI, ph ^ 1u);
                    wait(BAR_H, ph);
                    if (lead) mbar_arrive(bar(BAR_OFF));
                    wait(BAR_WX, ph);
                    tc_fence_after();
                    __syncwarp();
                    issue_state();
                    wait(BAR_M, ph);
                    if (lead) mma_commit(bar(BAR_Y));
                    // the combine of the last block needs h_in(r), published by state
                    // item r-1 (this item's MMAs are already issued)
                    if (last_block && d.r > 0 && lead) chain_wait(d.bh, d.r);
                    __syncwarp();
                    if (lead) mbar_arrive(bar(BAR_CHAIN));
                } else {
                    // ---- S = C B^T (K = N) into region R (free: the previous Y is done)
#pragma unroll
                    for (int k = 0; k < N / 16; ++k) {
                        const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                        if (k == 0) { if (lead) mma_ss<ID_S, 0>(tmem + COL_R, dC + o, dBk + o);
                        } else if (lead) mma_ss<ID_S, 1>(tmem + COL_R, dC + o, dBk + o);
                    }
                    if (lead) mma_commit(bar(BAR_S));
                    // ---- an output item starts from the entry state of its run
                    if (RUNS && j == 0 && d.r > 0 && lead) chain_wait(d.bh, d.r);
                    __syncwarp();
                    if (lead) mbar_arrive(bar(BAR_CHAIN));
                    // ---- Yoff = C h_hi + C h_lo into the Y accumulator (once the previous
                    // block's epilogue has read it)
                    if (blk > 0) wait(BAR_EPI, ph ^ 1u);
                    wait(BAR_H, ph);
                    tc_fence_after();
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < N / 16; ++k) {
                        const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                        if (k == 0) { if (lead) mma_ss<ID_OFF, 0>(tmem + COL_Y, dC, dW1);
                        } else if (lead) mma_ss<ID_OFF, 1>(tmem + COL_Y, dC + o, dW1 + k * KSTEP_MN);
                    }
#pragma unroll
                    for (int k = 0; k < N / 16; ++k) {
                        const uint32_t o = (uint32_t)(k >> 2) * KBLOCK_K + (uint32_t)(k & 3) * KSTEP_K;
                        if (lead) mma_ss<ID_OFF, 1>(tmem + COL_Y, dC + o, dW2 + k * KSTEP_MN);
                    }
                    if (lead) mma_commit(bar(BAR_OFF));
                    // ---- state: onto 2^(r_last) h (written by the compute warps) accumulate
                    // B^T (w o X)_hi and B^T (w o X)_lo (K = 128 tokens)
                    wait(BAR_WX, ph);
                    tc_fence_after();
                    __syncwarp();
                    issue_state();
                    // ---- Y += M_hi X + M_lo X onto the scaled Yoff (A from TMEM)
                    wait(BAR_M, ph);
                    tc_fence_after();
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < SUB / 16; ++k)
                        if (lead) mma_ts<ID_Y, 1>(tmem + COL_Y, tmem + COL_R + 16 * k, dX + k * KSTEP_MN);
#pragma unroll
                    for (int k = 0; k < SUB / 16; ++k)
                        if (lead) mma_ts<ID_Y, 1>(tmem + COL_Y, tmem + COL_R + 16 * k + 8, dX + k * KSTEP_MN);
                    if (lead) mma_commit(bar(BAR_Y));
                }
                // ---- next block: C, B, X, dt and the cumsum are free once Y is done
                wait(BAR_Y, ph);
                if (!last_block) {
                    ++j;
                } else {
                    int nx = 0;
                    if (lead) nx = atomicAdd(p.flags + p.BH + CTRL_TICKET, 1);
                    item = __shfl_sync(0xffffffffu, nx, __ffs(__ballot_sync(0xffffffffu, lead)) - 1);
                    j = 0;
                }
                load_block(item, j);
                // ---- a state item publishes h_in(r+1) once the compute warps stored it
                wait(BAR_PUB, ph);
                if (d.st && last_block && lead && !p.drop_publish) {
                    __threadfence();
                    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p.flags + d.bh), "r"(d.r + 1)
                                 : "memory");
                }
                ++blk;
            }
        }
    } else {
        // ==================================================== compute warps
        const float NEG_INF = __int_as_float(0xff800000u);
        auto csync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + pipe), "r"(NCOMPUTE) : "memory"); };
        uint32_t blk = 0;
        float prev_last = 0.f;   // raw cumsum at the end of the previous block of the same item
        float run_decay = 0.f;   // log2 decay over a state item's blocks so far (its R_r at the end)
        while (true) {
            const uint32_t ph = blk & 1u;
            wait(BAR_TMA, ph);
            const int item = *s_item, j = *s_j;
            if (item >= total) break;
            const Item d = decode(item);
            const int c = d.r, bh = d.bh;
            const int b = bh / p.H, h = bh % p.H;
            const bool last_block = (j == nblocks(item) - 1);
            const long long t0 = (long long)c * p.K * p.Q + (long long)j * SUB;
            const bool chunk_start = (t0 % p.Q) == 0;    // the decay cumsum restarts at every chunk

            // ---- per-token decay terms (r relative to the block start, log2 units)
            const float r0 = chunk_start ? 0.f : prev_last;
            const float rl = (s_acs[row] - r0) * LOG2E;
            const float rlast = (s_acs[SUB - 1] - r0) * LOG2E;
            if (half == 0) {
                // dt folded into the exponent: dt_s 2^(x - r_s) = 2^(x + log2(dt_s) - r_s); dt_s = 0
                // gives 0.  In place: this thread alone reads and writes element `row`.
                const float dtv = scs[row];
                scs[row] = (dtv > 0.f ? __log2f(dtv) : NEG_INF) - rl;
            }
            if (tid == 0) bulk_wait_read0();          // previous y store has read W1/W2
            csync();
            prev_last = s_acs[SUB - 1];

            // h_in(r) of state row n = row + 128 nb and 16 of this thread's columns:
            // the initial state (r = 0) or the run's entry-state slot; 0 for the
            // padding rows n >= N
            auto load_entry = [&](int r, int nb, int pc, float (&hv)[16]) {
                const int n = row + 128 * nb;
                if (N < 128 && n >= N) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) hv[i] = 0.f;
                } else if (RUNS && r > 0) {
                    const float* slot = slot_of(bh, r) + n * PD + half * 32 + pc * 16;
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        const float4 v = __ldcg(reinterpret_cast<const float4*>(slot + i));
                        hv[i] = v.x; hv[i + 1] = v.y; hv[i + 2] = v.z; hv[i + 3] = v.w;
                    }
                } else if (p.init_state) {
                    const long long o = ((long long)bh * N + n) * PD + half * 32 + pc * 16;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        hv[i] = p.state_bf16 ? __bfloat162float(reinterpret_cast<const bf16*>(p.init_state)[o + i])
                                             : reinterpret_cast<const float*>(p.init_state)[o + i];
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) hv[i] = 0.f;
                }
            };
            // w o X split hi -> W1, lo -> W2; the raw x words are returned for D x
            auto write_wx = [&](uint32_t (&xr)[16]) {
                const float w = ex2(rlast + scs[row]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t o = swz(row, half * 4 + q);
                    const uint4 xv = *reinterpret_cast<const uint4*>(sm + K::OFF_X + o);
                    xr[4 * q] = xv.x; xr[4 * q + 1] = xv.y; xr[4 * q + 2] = xv.z; xr[4 * q + 3] = xv.w;
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float v0 = bf16_lo(xr[4 * q + e]) * w, v1 = bf16_hi(xr[4 * q + e]) * w;
                        hw[e] = pack_bf16(v0, v1);
                        lw[e] = pack_bf16(v0 - bf16_lo(hw[e]), v1 - bf16_hi(hw[e]));
                    }
                    *reinterpret_cast<uint4*>(sm + K::OFF_W1 + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4*>(sm + K::OFF_W2 + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            };

            if (d.st) {
                // ==== state item: the run's own state from zero, dS_r, and its
                // log2 decay R_r; the last block combines h_in(r+1) = 2^(R_r) h_in(r) + dS_r
                run_decay = (j == 0 ? 0.f : run_decay) + rlast;
                {
                    const float dl = ex2(rlast);
#pragma unroll
                    for (int q = 0; q < 2 * K::NB; ++q) {   // (row block, 16-column part)
                        const uint32_t col = COL_ST + 64 * (q >> 1) + half * 32 + (q & 1) * 16;
                        uint32_t v[16];
                        if (j > 0) {
                            tmem_ld16(tmem + lane_off + col, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(dl * __uint_as_float(v[i]));
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i) v[i] = 0u;
                        }
                        tmem_st16(tmem + lane_off + col, v);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar(BAR_H));
                }
                wait(BAR_S, ph);
                wait(BAR_OFF, ph);
                {
                    uint32_t xr[16];
                    write_wx(xr);
                }
                fence_proxy_async();
                mbar_arrive(bar(BAR_WX));
                mbar_arrive(bar(BAR_M));
                wait(BAR_Y, ph);
                tc_fence_after();
                if (last_block) {
                    wait(BAR_CHAIN, ph);              // h_in(r) is published
                    const float dr = ex2(run_decay);
#pragma unroll
                    for (int q = 0; q < 2 * K::NB; ++q) {
                        const int nb = q >> 1, pc = q & 1;
                        if (N < 128 && row + 128 * nb >= N) continue;   // padding rows (warp-uniform: N % 32 == 0)
                        uint32_t sv[16];
                        tmem_ld16(tmem + lane_off + COL_ST + 64 * nb + half * 32 + pc * 16, sv);
                        tmem_wait_ld();
                        float hin[16];
                        load_entry(c, nb, pc, hin);
                        float* slot = slot_of(bh, c + 1) + (row + 128 * nb) * PD + half * 32 + pc * 16;
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            __stcg(reinterpret_cast<float4*>(slot + i),
                                   make_float4(fmaf(dr, hin[i], __uint_as_float(sv[i])),
                                               fmaf(dr, hin[i + 1], __uint_as_float(sv[i + 1])),
                                               fmaf(dr, hin[i + 2], __uint_as_float(sv[i + 2])),
                                               fmaf(dr, hin[i + 3], __uint_as_float(sv[i + 3]))));
                    }
                }
                mbar_arrive(bar(BAR_PUB));
                tc_fence_before();
                mbar_arrive(bar(BAR_EPI));            // no output: the Y accumulator is free
                ++blk;
                continue;
            }

            // ==== output item
            // ---- h entering the block: the run's entry state (first block), else the
            // state the previous block left in the TMEM accumulator.  Split hi -> W1,
            // lo -> W2 for C h; 2^(r_last) h -> the state accumulator.
            {
                const float dl = ex2(rlast);
                if (j == 0) wait(BAR_CHAIN, ph);
#pragma unroll
                for (int qq = 0; qq < 2 * K::NB; ++qq) {   // (row block, 16-column part)
                    const int nb = qq >> 1, pc = qq & 1;
                    const uint32_t col = COL_ST + 64 * nb + half * 32 + pc * 16;
                    float hv[16];
                    if (j > 0) {
                        uint32_t v[16];
                        tmem_ld16(tmem + lane_off + col, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) hv[i] = __uint_as_float(v[i]);
                    } else {
                        load_entry(c, nb, pc, hv);
                    }
                    uint32_t sc[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) sc[i] = __float_as_uint(dl * hv[i]);
                    tmem_st16(tmem + lane_off + col, sc);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float v0 = hv[q * 8 + 2 * e], v1 = hv[q * 8 + 2 * e + 1];
                            hw[e] = pack_bf16(v0, v1);
                            lw[e] = pack_bf16(v0 - bf16_lo(hw[e]), v1 - bf16_hi(hw[e]));
                        }
                        const uint32_t o = swz(row + 128 * nb, half * 4 + pc * 2 + q);
                        *reinterpret_cast<uint4*>(sm + K::OFF_W1 + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                        *reinterpret_cast<uint4*>(sm + K::OFF_W2 + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                    }
                }
                tmem_wait_st();
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(bar(BAR_H));
            }

            // ---- M = S o [s<=l] 2^(r_l - r_s) dt_s, split hi/lo, written back in place:
            // for every 16-column K step k of the MMA, hi goes to columns [16k, 16k+8)
            // and lo to [16k+8, 16k+16) -- the S columns this thread just read.
            // Column parts entirely above the diagonal for the whole warp are zero.
            wait(BAR_S, ph);
            tc_fence_after();
            const int row_lo = (warp & 3) * 32;       // first row of this warp
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int c0 = half * 64 + g * 16;    // one K step of the MMA: 16 columns
                uint32_t v[16], o[16];
                tmem_ld16(tmem + lane_off + COL_R + c0, v);
                tmem_wait_ld();
                if (c0 > row_lo + 31) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = 0u;
                } else {
                    const float4* cs4 = reinterpret_cast<const float4*>(scs + c0);
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const float4 cv = cs4[i4];
                        const float cvv[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int i = i4 * 2 + hh;
                            const int s0 = c0 + 2 * i;
                            const float e0 = ex2(s0 <= row ? rl + cvv[2 * hh] : NEG_INF);
                            const float e1 = ex2(s0 + 1 <= row ? rl + cvv[2 * hh + 1] : NEG_INF);
                            const float m0 = __uint_as_float(v[2 * i]) * e0;
                            const float m1 = __uint_as_float(v[2 * i + 1]) * e1;
                            const uint32_t hi = pack_bf16(m0, m1);
                            o[i] = hi;
                            o[8 + i] = pack_bf16(m0 - bf16_lo(hi), m1 - bf16_hi(hi));
                        }
                    }
                }
                tmem_st16(tmem + lane_off + COL_R + c0, o);
            }

            // ---- scale Yoff by 2^(r_l) in place (the Y MMAs accumulate on top)
            const float el = ex2(rl);
            wait(BAR_OFF, ph);
            tc_fence_after();
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
                uint32_t v[16];
                tmem_ld16(tmem + lane_off + COL_Y + half * 32 + pc * 16, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(el * __uint_as_float(v[i]));
                tmem_st16(tmem + lane_off + COL_Y + half * 32 + pc * 16, v);
            }
            // ---- w o X (free: C h is done); x kept for D x
            uint32_t xr[16];
            write_wx(xr);
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(bar(BAR_WX));
            mbar_arrive(bar(BAR_M));

            // ---- after Y (and the state MMAs before it): the final state after the
            // last block of the last run, then y = (2^(r_l) Yoff + M X) + D x, staged
            // in W1/W2, TMA store
            wait(BAR_Y, ph);
            tc_fence_after();
            if (last_block && c == p.nruns - 1 && p.final_state) {
#pragma unroll
                for (int q = 0; q < 2 * K::NB; ++q) {
                    const int nb = q >> 1, pc = q & 1;
                    const int n = row + 128 * nb;
                    if (N < 128 && n >= N) continue;     // padding rows (warp-uniform: N % 32 == 0)
                    const long long fo = ((long long)bh * N + n) * PD + half * 32;
                    uint32_t sv[16];
                    tmem_ld16(tmem + lane_off + COL_ST + 64 * nb + half * 32 + pc * 16, sv);
                    tmem_wait_ld();
                    float ho[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) ho[i] = __uint_as_float(sv[i]);
                    if (p.state_bf16) {
                        bf16* fs = reinterpret_cast<bf16*>(p.final_state) + fo + pc * 16;
                        Vec16<bf16>::store(fs, ho);
                        Vec16<bf16>::store(fs + 8, ho + 8);
                    } else {
                        float* fs = reinterpret_cast<float*>(p.final_state) + fo + pc * 16;
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            *reinterpret_cast<float4*>(fs + i) = make_float4(ho[i], ho[i + 1], ho[i + 2], ho[i + 3]);
                    }
                }
            }
            mbar_arrive(bar(BAR_PUB));
            {
                const float dsk = p.D ? p.D[h] : 0.f;
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    uint32_t yv[16];
                    tmem_ld16(tmem + lane_off + COL_Y + half * 32 + pc * 16, yv);
                    tmem_wait_ld();
                    if (pc == 1) {
                        tc_fence_before();
                        mbar_arrive(bar(BAR_EPI));    // the Y accumulator may be reused
                    }
                    float out[16];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t xw = xr[pc * 8 + e];
                        out[2 * e] = __uint_as_float(yv[2 * e]) + dsk * bf16_lo(xw);
                        out[2 * e + 1] = __uint_as_float(yv[2 * e + 1]) + dsk * bf16_hi(xw);
                    }
                    if (p.y_bf16) {
#pragma unroll
                        for (int q = 0; q < 2; ++q)
                            *reinterpret_cast<uint4*>(sm + K::OFF_W1 + swz(row, half * 4 + pc * 2 + q)) =
                                Vec16<bf16>::pack(out + 8 * q);
                    } else {
                        uint8_t* tile = sm + (half ? K::OFF_W2 : K::OFF_W1);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<float4*>(tile + swz(row, pc * 4 + q)) =
                                make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
                    }
                }
            }
            fence_proxy_async();
            csync();
            if (tid == 0) {
                tma_store_4d(&tmY, base + K::OFF_W1, 0, h, (int)t0, b);
                if (!p.y_bf16) tma_store_4d(&tmY, base + K::OFF_W2, 32, h, (int)t0, b);
                bulk_commit();
            }
            ++blk;
        }
        if (tid == 0) bulk_wait0();   // the last y store is complete before the CTA leaves
    }

    if (err) atomicOr(p.dev_err, err);
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        const uint32_t tmem_all = *reinterpret_cast<volatile uint32_t*>(s_tmem_slot);
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_all), "r"(K::TMEM_COLS) : "memory");
    }
}


template <int N>
static cudaError_t launch_n(const PrefillArgs& a, cudaStream_t s) {
    using K = Cfg<N>;
    CUtensorMap mx, mb, mc, my;
    if (!make_map(&my, a.y, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.batch, !a.y_bf16) ||
        !make_map(&mx, a.x, (uint64_t)a.P, (uint64_t)a.H, (uint64_t)a.L, (uint64_t)a.batch) ||
        !make_map(&mb, a.B, (uint64_t)a.N, (uint64_t)a.G, (uint64_t)a.L, (uint64_t)a.batch) ||
        !make_map(&mc, a.C, (uint64_t)a.N, (uint64_t)a.G, (uint64_t)a.L, (uint64_t)a.batch))
        return cudaErrorInvalidValue;
    // persistent grid: as many CTAs as can be resident (one per SM), never more than items
    static std::mutex mu;
    static int resident[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!resident[dev]) {
            e = cudaFuncSetAttribute(ssd_tc_kernel<N, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::SMEM);
            if (e != cudaSuccess) return e;
            e = cudaFuncSetAttribute(ssd_tc_kernel<N, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::SMEM);
            if (e != cudaSuccess) return e;
            int per_sm = 0, sms = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ssd_tc_kernel<N, false>, K::THREADS, K::SMEM);
            if (e != cudaSuccess) return e;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            resident[dev] = (per_sm > 0 ? per_sm : 1) * sms;
        }
    }
    Params p{};
    p.dtw = (const float*)(a.ws + a.lay.off_dt);
    p.acsw = (const float*)(a.ws + a.lay.off_acs);
    p.slots = (float*)(a.ws + a.lay.off_states);
    p.flags = (int*)(a.ws + a.lay.off_flags);
    p.init_state = a.init_state;
    p.final_state = a.final_state;
    p.y = a.y;
    p.D = a.D;
    p.dev_err = a.dev_err;
    p.L = a.L;
    p.Lpad = a.lay.Lpad;
    p.H = (int)a.H;
    p.G = (int)a.G;
    p.Q = (int)a.Q;
    p.nchunks = (int)a.lay.nchunks;
    p.BH = (int)(a.batch * a.H);
    const long long nruns = tc_runs(p.BH, p.nchunks, N);
    p.nruns = (int)nruns;
    p.K = (int)((p.nchunks + nruns - 1) / nruns);
    p.nstate = (int)((nruns - 1) * p.BH);
    p.state_bf16 = a.state_bf16;
    p.y_bf16 = a.y_bf16;
    p.drop_publish = a.drop_publish;
    const long long items = (long long)p.nstate + (long long)p.nruns * p.BH;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    const long long want = (items + K::PIPES - 1) / K::PIPES;   // each CTA runs PIPES ticket streams
    const unsigned grid = (unsigned)(want < resident[dev] ? want : resident[dev]);
    // whole sequences (one run each) take the instantiation without state items
    // or hand-off waits: the code of the block loop is then that alone.  The
    // launch is a programmatic dependent of the decay-cumsum kernel before it on
    // the stream: its prologue overlaps that kernel, and its control warps wait
    // for it (griddepcontrol.wait) before reading what it wrote.
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(K::THREADS);
    cfg.dynamicSmemBytes = K::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (p.nruns > 1) return cudaLaunchKernelEx(&cfg, ssd_tc_kernel<N, true>, mx, mb, mc, my, p);
    return cudaLaunchKernelEx(&cfg, ssd_tc_kernel<N, false>, mx, mb, mc, my, p);
}

}  // namespace tc

// Runs per sequence.  With at least half as many sequences as the block
// pipelines of a 148-SM part (1 or 2 per SM), every item is a whole sequence and the
// state never leaves the SM.  Otherwise sequences are cut into runs so that
// about 3 output items fall to each pipeline: fewer, longer items measured
// faster than finer balance (each item pays a pipeline fill and drain, and
// every run but the last one extra, light state item).  A pure function of the
// shape, so that the workspace size does not depend on the device.
int64_t tc_runs(int64_t BH, int64_t nchunks, int64_t N) {
    const int64_t kPipes = 148 * (N > 128 ? tc::Cfg<256>::PIPES : tc::Cfg<128>::PIPES);
    if (nchunks <= 1 || 2 * BH >= kPipes) return 1;
    int64_t k = (nchunks * BH + 3 * kPipes - 1) / (3 * kPipes);   // chunks per run
    if (k < 1) k = 1;
    return (nchunks + k - 1) / k;
}

bool tc_path_supports(int64_t P, int64_t N, int64_t Q, bool io_bf16) {
    return io_bf16 && P == tc::PD && (N == 64 || N == 128 || N == 256) && (Q == 128 || Q == 256);
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
    if (!tc_path_supports(a.P, a.N, a.Q, a.io_bf16)) return cudaErrorNotSupported;
    // pairs of heads sharing B and C, every item a whole sequence
    if (pair_path_supports(a.batch, a.H, a.P, a.N, a.G, a.Q, a.io_bf16)) return launch_prefill_pair(a, s);
    switch (a.N) {
        case 64: return tc::launch_n<64>(a, s);
        case 128: return tc::launch_n<128>(a, s);
        default: return tc::launch_n<256>(a, s);
    }
}

}  // namespace ssd
