// libssd C ABI: argument validation, workspace layout and dispatch.
// Declarations and the contract of every entry point are in include/ssd.h.
#include <atomic>
#include <mutex>

#include "../../include/ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

// Device-side error word (bits kErr*), one per device that loads the library.
__device__ unsigned g_device_error;

static std::mutex g_err_mutex;
static std::atomic<uint32_t> g_debug_faults{0};

uint32_t debug_faults() { return g_debug_faults.load(std::memory_order_relaxed); }
static unsigned* g_err_ptr[64];

static cudaError_t device_error_ptr(unsigned** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_err_mutex);
    if (!g_err_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_error);
        if (e != cudaSuccess) return e;
        g_err_ptr[dev] = (unsigned*)p;
    }
    *out = g_err_ptr[dev];
    return cudaSuccess;
}

static inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

static bool valid_dtype(int32_t d) { return d == SSD_F32 || d == SSD_BF16; }
static size_t dsize(int32_t d) { return d == SSD_BF16 ? 2 : 4; }

static bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

static ssd_status_t check_prefill_desc(const ssd_prefill_desc_t* d) {
    if (!d) return SSD_ERR_INVALID_ARG;
    if (d->batch < 0 || d->seqlen < 0 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 ||
        d->ngroups < 1 || d->chunk < 1)
        return SSD_ERR_INVALID_ARG;
    if (d->nheads % d->ngroups != 0) return SSD_ERR_INVALID_ARG;
    if (!valid_dtype(d->io_dtype) || !valid_dtype(d->y_dtype) || !valid_dtype(d->state_dtype))
        return SSD_ERR_INVALID_ARG;
    if (!is_pow2(d->chunk) || d->chunk < 16 || d->chunk > 256) return SSD_ERR_UNSUPPORTED;
    if (d->headdim % 8 != 0 || d->dstate % 8 != 0 || d->headdim > 256 || d->dstate > 256)
        return SSD_ERR_UNSUPPORTED;
    if (d->nheads > (1 << 20) || d->batch > (1 << 24) || d->seqlen > ((int64_t)1 << 31))
        return SSD_ERR_UNSUPPORTED;
    // 1-D grids: blocks over (batch*heads) x chunks x tiles must stay below 2^31
    const int64_t nchunks = (d->seqlen + d->chunk - 1) / d->chunk;
    const int64_t tiles = ((d->dstate + 63) / 64) * ((d->headdim + 63) / 64) * ((d->chunk + 63) / 64);
    if (d->batch * d->nheads * nchunks * tiles >= ((int64_t)1 << 31)) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

static PrefillLayout prefill_layout(const ssd_prefill_desc_t* d, bool tc) {
    PrefillLayout lay{};
    const int64_t BH = d->batch * d->nheads;
    lay.nchunks = (d->seqlen + d->chunk - 1) / d->chunk;
    lay.Lpad = lay.nchunks * d->chunk;
    size_t off = 0;
    lay.off_dt = off;
    off = align256(off + sizeof(float) * (size_t)BH * lay.Lpad);
    lay.off_acs = off;
    off = align256(off + sizeof(float) * (size_t)BH * lay.Lpad);
    lay.off_acs_lo = off;
    lay.has_lo = true;
    off = align256(off + sizeof(float) * (size_t)BH * lay.Lpad);
    lay.off_states = off;
    const size_t state_elems = (size_t)d->dstate * d->headdim;
    // CUDA-core path: one state per chunk; tensor-core path: the entry state of
    // every run after the first
    const int64_t nstates = tc ? tc_runs(BH, lay.nchunks, d->dstate) - 1 : lay.nchunks;
    off = align256(off + sizeof(float) * state_elems * (size_t)BH * (size_t)nstates);
    lay.off_flags = off;
    off = align256(off + sizeof(int) * ((size_t)BH + 64));
    lay.total = off;
    return lay;
}

static int prefill_path(const ssd_prefill_desc_t* d) {
    const bool bf = d->io_dtype == SSD_BF16;
    if (!tc_path_supports(d->headdim, d->dstate, d->chunk, bf)) return 1;
    return pair_path_supports(d->batch, d->nheads, d->headdim, d->dstate, d->ngroups, d->chunk, bf) ? 2 : 0;
}

// replay descriptor checks shared by ssd_replay_buffer_size and ssd_replay_step
static ssd_status_t check_replay_desc(const ssd_replay_desc_t* d) {
    if (!d) return SSD_ERR_INVALID_ARG;
    if (d->batch < 0 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 || d->ngroups < 1 ||
        d->nheads % d->ngroups != 0 || d->capacity < 1)
        return SSD_ERR_INVALID_ARG;
    if (!valid_dtype(d->io_dtype) || !valid_dtype(d->y_dtype) || !valid_dtype(d->state_dtype))
        return SSD_ERR_INVALID_ARG;
    // a lane owns 4 columns of a state row and the lanes of a warp cover whole rows
    const int64_t P = d->headdim;
    if (!(P == 8 || P == 16 || P == 32 || P == 64 || P == 128)) return SSD_ERR_UNSUPPORTED;
    if (d->dstate % 8 != 0 || d->dstate > 256 || d->capacity > 16) return SSD_ERR_UNSUPPORTED;
    if (d->batch * d->nheads > (int64_t)0x7fffffff) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

static ReplayLayout replay_layout(const ssd_replay_desc_t* d) {
    ReplayLayout l{};
    const size_t K = (size_t)d->capacity, e = dsize(d->io_dtype);
    const size_t bh = (size_t)d->batch * d->nheads, bg = (size_t)d->batch * d->ngroups;
    l.off_x = 0;
    l.off_B = align256(l.off_x + bh * K * d->headdim * e);
    l.off_dt = align256(l.off_B + bg * K * d->dstate * e);
    l.off_cum = align256(l.off_dt + bh * K * sizeof(float));
    l.off_cb = align256(l.off_cum + bh * K * sizeof(float));
    l.total = align256(l.off_cb + bg * 16 * sizeof(float));
    return l;
}

// copies (or zero-fills) init_state into final_state for seqlen == 0
template <typename S, typename D>
__global__ void copy_state_kernel(const S* __restrict__ src, D* __restrict__ dst, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = from_f32<D>(src ? to_f32(src[i]) : 0.f);
}

}  // namespace ssd

using namespace ssd;

extern "C" {

int ssd_version(void) { return 100; }

const char* ssd_status_string(ssd_status_t s) {
    switch (s) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: invalid argument";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape or dtype not implemented";
        case SSD_ERR_ALIGNMENT: return "SSD_ERR_ALIGNMENT: tensor base not 16-byte aligned";
        case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA call failed";
        case SSD_ERR_DEVICE_TIMEOUT: return "SSD_ERR_DEVICE_TIMEOUT: a device-side wait gave up";
    }
    return "SSD_ERR_UNKNOWN";
}

ssd_status_t ssd_chunk_scan_workspace_size(const ssd_prefill_desc_t* desc, size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    const ssd_status_t st = check_prefill_desc(desc);
    if (st != SSD_OK) return st;
    *bytes = prefill_layout(desc, prefill_path(desc) != 1).total;
    return SSD_OK;
}

ssd_status_t ssd_chunk_scan_path(const ssd_prefill_desc_t* desc, int32_t* path) {
    if (!path) return SSD_ERR_INVALID_ARG;
    const ssd_status_t st = check_prefill_desc(desc);
    if (st != SSD_OK) return st;
    *path = prefill_path(desc);
    return SSD_OK;
}

// ssd_chunk_scan_fwd and its variable-length form (pad_left NULL = no padding)
static ssd_status_t prefill(const ssd_prefill_desc_t* d, const void* x, const void* dt_raw,
                            const float* dt_bias, const float* A, const void* B, const void* C,
                            const float* D, const void* init_state, const int32_t* pad_left, void* y,
                            void* final_state, void* workspace, size_t workspace_bytes, void* stream) {
    ssd_status_t st = check_prefill_desc(d);
    if (st != SSD_OK) return st;
    const bool empty = d->batch == 0 || d->seqlen == 0;   // token tensors may then be NULL
    if (!A || (!empty && (!x || !dt_raw || !B || !C || !y))) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt_raw, dt_bias, A, B, C, D, init_state, y, final_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGNMENT;
    const size_t tok = (size_t)d->batch * d->seqlen;
    const size_t x_bytes = tok * d->nheads * d->headdim * dsize(d->io_dtype);
    const size_t y_bytes = tok * d->nheads * d->headdim * dsize(d->y_dtype);
    const size_t s_bytes = (size_t)d->batch * d->nheads * d->dstate * d->headdim * dsize(d->state_dtype);
    const size_t bc_bytes = tok * d->ngroups * d->dstate * dsize(d->io_dtype);
    if (overlaps(y, y_bytes, x, x_bytes) || overlaps(y, y_bytes, B, bc_bytes) ||
        overlaps(y, y_bytes, C, bc_bytes) || overlaps(final_state, s_bytes, y, y_bytes) ||
        overlaps(final_state, s_bytes, x, x_bytes))
        return SSD_ERR_INVALID_ARG;
    const bool tc = prefill_path(d) != 1;
    const PrefillLayout lay = prefill_layout(d, tc);
    if (d->batch == 0) return SSD_OK;
    if (d->seqlen > 0 && (!workspace || workspace_bytes < lay.total)) return SSD_ERR_WORKSPACE;
    if (workspace && ((uintptr_t)workspace & 255u)) return SSD_ERR_ALIGNMENT;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (d->seqlen == 0) {
        if (!final_state) return SSD_OK;
        const int64_t n = (int64_t)d->batch * d->nheads * d->dstate * d->headdim;
        const unsigned grid = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
        const bool sb = d->state_dtype == SSD_BF16;
        if (sb) copy_state_kernel<bf16, bf16><<<grid, 256, 0, s>>>((const bf16*)init_state, (bf16*)final_state, n);
        else copy_state_kernel<float, float><<<grid, 256, 0, s>>>((const float*)init_state, (float*)final_state, n);
        return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
    }
    PrefillArgs a{};
    a.batch = d->batch; a.L = d->seqlen; a.H = d->nheads; a.P = d->headdim; a.N = d->dstate;
    a.G = d->ngroups; a.Q = d->chunk;
    a.io_bf16 = d->io_dtype == SSD_BF16; a.y_bf16 = d->y_dtype == SSD_BF16;
    a.state_bf16 = d->state_dtype == SSD_BF16;
    a.x = x; a.dt_raw = dt_raw; a.B = B; a.C = C; a.dt_bias = dt_bias; a.A = A; a.D = D;
    a.init_state = init_state; a.y = y; a.final_state = final_state;
    a.pad_left = pad_left;
    a.ws = (char*)workspace; a.lay = lay;
    a.drop_publish = (debug_faults() & SSD_FAULT_DROP_RUN_PUBLISH) ? 1 : 0;
    e = device_error_ptr(&a.dev_err);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    e = launch_dt_cumsum(a, s);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    e = tc ? launch_prefill_tc(a, s) : launch_prefill_simt(a, s);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status_t ssd_chunk_scan_fwd(const ssd_prefill_desc_t* d, const void* x, const void* dt_raw,
                                const float* dt_bias, const float* A, const void* B, const void* C,
                                const float* D, const void* init_state, void* y, void* final_state,
                                void* workspace, size_t workspace_bytes, void* stream) {
    return prefill(d, x, dt_raw, dt_bias, A, B, C, D, init_state, nullptr, y, final_state, workspace,
                   workspace_bytes, stream);
}

ssd_status_t ssd_chunk_scan_fwd_varlen(const ssd_prefill_desc_t* d, const void* x, const void* dt_raw,
                                       const float* dt_bias, const float* A, const void* B, const void* C,
                                       const float* D, const void* init_state, const int32_t* pad_left, void* y,
                                       void* final_state, void* workspace, size_t workspace_bytes,
                                       void* stream) {
    if (!pad_left && d && d->batch > 0) return SSD_ERR_INVALID_ARG;
    if (pad_left && ((uintptr_t)pad_left & 3u)) return SSD_ERR_ALIGNMENT;
    return prefill(d, x, dt_raw, dt_bias, A, B, C, D, init_state, pad_left, y, final_state, workspace,
                   workspace_bytes, stream);
}

static Mamba3Layout m3_layout(const ssd_prefill_desc_t* d) {
    return mamba3_layout(d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->ngroups, d->chunk,
                         d->io_dtype == SSD_BF16, prefill_path(d) != 1);
}

static ssd_status_t check_mamba3_desc(const ssd_prefill_desc_t* d) {
    const ssd_status_t st = check_prefill_desc(d);
    if (st != SSD_OK) return st;
    // the rotation kernel's grid: (b, g, chunk, 4 pairs)
    const int64_t nchunks = (d->seqlen + d->chunk - 1) / d->chunk;
    if (d->batch * d->ngroups * nchunks * ((d->dstate / 2 + 3) / 4) >= ((int64_t)1 << 31)) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

ssd_status_t ssd_chunk_scan_mamba3_workspace_size(const ssd_prefill_desc_t* desc, size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    const ssd_status_t st = check_mamba3_desc(desc);
    if (st != SSD_OK) return st;
    *bytes = m3_layout(desc).total;
    return SSD_OK;
}

ssd_status_t ssd_chunk_scan_fwd_mamba3(const ssd_prefill_desc_t* d, const void* x, const void* dt_raw,
                                       const float* dt_bias, const float* A, const void* B, const void* C,
                                       const float* D, const float* lam, const float* theta, const void* init_state,
                                       void* y, void* final_state, void* workspace, size_t workspace_bytes,
                                       void* stream) {
    ssd_status_t st = check_mamba3_desc(d);
    if (st != SSD_OK) return st;
    if ((lam && !aligned16(lam)) || (theta && !aligned16(theta))) return SSD_ERR_ALIGNMENT;
    const size_t tok = (size_t)d->batch * d->seqlen;
    const size_t y_bytes = tok * d->nheads * d->headdim * dsize(d->y_dtype);
    const size_t s_bytes = (size_t)d->batch * d->nheads * d->dstate * d->headdim * dsize(d->state_dtype);
    if (overlaps(y, y_bytes, lam, tok * d->nheads * sizeof(float)) ||
        overlaps(y, y_bytes, theta, tok * d->ngroups * (d->dstate / 2) * sizeof(float)) ||
        overlaps(final_state, s_bytes, lam, tok * d->nheads * sizeof(float)) ||
        overlaps(final_state, s_bytes, theta, tok * d->ngroups * (d->dstate / 2) * sizeof(float)))
        return SSD_ERR_INVALID_ARG;
    // empty problems, argument checks and the plain recurrence's cases: the
    // forward call (with seqlen 0 the final state is the initial one either way)
    if (d->batch == 0 || d->seqlen == 0 || (!lam && !theta))
        return prefill(d, x, dt_raw, dt_bias, A, B, C, D, init_state, nullptr, y, final_state, workspace,
                       workspace_bytes, stream);
    if (!A || !x || !dt_raw || !B || !C || !y) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt_raw, dt_bias, A, B, C, D, init_state, y, final_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGNMENT;
    const size_t x_bytes = tok * d->nheads * d->headdim * dsize(d->io_dtype);
    const size_t bc_bytes = tok * d->ngroups * d->dstate * dsize(d->io_dtype);
    if (overlaps(y, y_bytes, x, x_bytes) || overlaps(y, y_bytes, B, bc_bytes) || overlaps(y, y_bytes, C, bc_bytes) ||
        overlaps(final_state, s_bytes, y, y_bytes) || overlaps(final_state, s_bytes, x, x_bytes))
        return SSD_ERR_INVALID_ARG;
    const Mamba3Layout lay = m3_layout(d);
    if (!workspace || workspace_bytes < lay.total) return SSD_ERR_WORKSPACE;
    if ((uintptr_t)workspace & 255u) return SSD_ERR_ALIGNMENT;
    Mamba3Args a{};
    a.batch = d->batch; a.L = d->seqlen; a.H = d->nheads; a.P = d->headdim; a.N = d->dstate;
    a.G = d->ngroups; a.Q = d->chunk;
    a.io_bf16 = d->io_dtype == SSD_BF16; a.y_bf16 = d->y_dtype == SSD_BF16;
    a.state_bf16 = d->state_dtype == SSD_BF16; a.tc = prefill_path(d) != 1;
    a.x = x; a.dt_raw = dt_raw; a.B = B; a.C = C; a.dt_bias = dt_bias; a.A = A; a.D = D;
    a.lam = lam; a.theta = theta; a.init_state = init_state; a.y = y; a.final_state = final_state;
    a.ws = (char*)workspace; a.lay = lay;
    cudaError_t e = device_error_ptr(&a.dev_err);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    e = launch_mamba3(a, (cudaStream_t)stream);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status_t ssd_chunk_scan_mamba3_launches(const ssd_prefill_desc_t* desc, int32_t has_lam, int32_t has_theta,
                                            int32_t has_final_state, int32_t* launches) {
    if (!launches) return SSD_ERR_INVALID_ARG;
    const ssd_status_t st = check_mamba3_desc(desc);
    if (st != SSD_OK) return st;
    const bool tc = prefill_path(desc) != 1;
    if (desc->batch == 0) *launches = 0;
    else if (desc->seqlen == 0) *launches = has_final_state ? 1 : 0;
    else if (!has_lam && !has_theta) *launches = 1 + (tc ? 1 : 3);
    else *launches = mamba3_launches(tc, desc->io_dtype == SSD_BF16, has_lam != 0, has_theta != 0,
                                     has_final_state != 0, m3_layout(desc).fused);
    return SSD_OK;
}

// the descriptor of the transposed scans of the backward (headdim and dstate
// swapped, one group per head, N cut into column slices)
static ssd_prefill_desc_t transposed_desc(const ssd_prefill_desc_t* d, int64_t pw) {
    ssd_prefill_desc_t t = *d;
    t.headdim = pw;
    t.dstate = d->headdim;
    t.ngroups = d->nheads;
    t.y_dtype = SSD_F32;
    t.state_dtype = SSD_F32;
    return t;
}

static ssd_status_t check_backward_desc(const ssd_prefill_desc_t* d, BackwardLayout* lay) {
    ssd_status_t st = check_prefill_desc(d);
    if (st != SSD_OK) return st;
    const BackwardLayout l = backward_layout(d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->ngroups,
                                             d->chunk, d->io_dtype == SSD_BF16);
    if (l.mode == 0) {
        const ssd_prefill_desc_t t = transposed_desc(d, l.pw);
        st = check_prefill_desc(&t);
        if (st != SSD_OK) return st;
    }
    if (d->batch * d->seqlen * d->nheads > ((int64_t)1 << 31) / 8) return SSD_ERR_UNSUPPORTED;
    if (lay) *lay = l;
    return SSD_OK;
}

ssd_status_t ssd_chunk_scan_bwd_workspace_size(const ssd_prefill_desc_t* desc, size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    BackwardLayout l;
    const ssd_status_t st = check_backward_desc(desc, &l);
    if (st != SSD_OK) return st;
    *bytes = l.total;
    return SSD_OK;
}

ssd_status_t ssd_chunk_scan_bwd(const ssd_prefill_desc_t* d, const void* x, const void* dt_raw,
                                const float* dt_bias, const float* A, const void* B, const void* C,
                                const float* D, const void* init_state, const void* dy,
                                const void* dfinal_state, void* dx, void* ddt_raw, float* ddt_bias, float* dA,
                                void* dB, void* dC, float* dD, void* dinit_state, void* workspace,
                                size_t workspace_bytes, void* stream) {
    BackwardLayout lay;
    ssd_status_t st = check_backward_desc(d, &lay);
    if (st != SSD_OK) return st;
    const bool empty = d->batch == 0 || d->seqlen == 0;
    if (!A || !dA) return SSD_ERR_INVALID_ARG;
    if (!empty && (!x || !dt_raw || !B || !C || !dy || !dx || !ddt_raw || !dB || !dC)) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt_raw, dt_bias, A, B, C, D, init_state, dy, dfinal_state,
                          dx, ddt_raw, ddt_bias, dA, dB, dC, dD, dinit_state};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGNMENT;
    const size_t tok = (size_t)d->batch * d->seqlen;
    const size_t ei = dsize(d->io_dtype), eg = dsize(d->y_dtype), es = dsize(d->state_dtype);
    const size_t hp = (size_t)d->nheads * d->headdim, gn = (size_t)d->ngroups * d->dstate;
    const size_t sb = (size_t)d->batch * d->nheads * d->dstate * d->headdim * es, hb = sizeof(float) * d->nheads;
    // no output may overlap an input or another output
    const struct { const void* p; size_t n; } in[] = {
        {x, tok * hp * ei}, {dt_raw, tok * d->nheads * ei}, {dt_bias, hb}, {A, hb}, {B, tok * gn * ei},
        {C, tok * gn * ei}, {D, hb}, {init_state, sb}, {dy, tok * hp * ei}, {dfinal_state, sb}};
    const struct { const void* p; size_t n; } out[] = {
        {dx, tok * hp * eg}, {ddt_raw, tok * d->nheads * eg}, {ddt_bias, hb}, {dA, hb}, {dB, tok * gn * eg},
        {dC, tok * gn * eg}, {dD, hb}, {dinit_state, sb}};
    for (size_t i = 0; i < sizeof(out) / sizeof(out[0]); ++i) {
        for (const auto& r : in)
            if (overlaps(out[i].p, out[i].n, r.p, r.n)) return SSD_ERR_INVALID_ARG;
        for (size_t j = i + 1; j < sizeof(out) / sizeof(out[0]); ++j)
            if (overlaps(out[i].p, out[i].n, out[j].p, out[j].n)) return SSD_ERR_INVALID_ARG;
    }
    if (!empty && (!workspace || workspace_bytes < lay.total)) return SSD_ERR_WORKSPACE;
    if (workspace && ((uintptr_t)workspace & 255u)) return SSD_ERR_ALIGNMENT;
    BackwardArgs a{};
    a.batch = d->batch; a.L = d->seqlen; a.H = d->nheads; a.P = d->headdim; a.N = d->dstate;
    a.G = d->ngroups; a.Q = d->chunk;
    a.io_bf16 = d->io_dtype == SSD_BF16; a.grad_bf16 = d->y_dtype == SSD_BF16;
    a.state_bf16 = d->state_dtype == SSD_BF16;
    a.x = x; a.dt_raw = dt_raw; a.B = B; a.C = C; a.dy = dy;
    a.dt_bias = dt_bias; a.A = A; a.D = D; a.init_state = init_state; a.dfinal = dfinal_state;
    a.dx = dx; a.ddt_raw = ddt_raw; a.dB = dB; a.dC = dC; a.dinit = dinit_state;
    a.ddt_bias = ddt_bias; a.dA = dA; a.dD = dD;
    a.ws = (char*)workspace; a.lay = lay;
    cudaError_t e = device_error_ptr(&a.dev_err);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    e = empty ? launch_backward_empty(a, s) : launch_backward(a, s);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status_t ssd_chunk_scan_bwd_launches(const ssd_prefill_desc_t* desc, int32_t has_states, int32_t* launches) {
    if (!launches) return SSD_ERR_INVALID_ARG;
    BackwardLayout l;
    const ssd_status_t st = check_backward_desc(desc, &l);
    if (st != SSD_OK) return st;
    *launches = (desc->batch == 0 || desc->seqlen == 0) ? 1 : backward_launches(l, has_states != 0);
    return SSD_OK;
}

ssd_status_t ssd_state_update(const ssd_decode_desc_t* d, void* state, const void* x, const void* dt_raw,
                              const float* dt_bias, const float* A, const void* B, const void* C,
                              const float* D, void* y, void* stream) {
    if (!d) return SSD_ERR_INVALID_ARG;
    if (d->batch < 0 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 || d->ngroups < 1 ||
        d->nheads % d->ngroups != 0)
        return SSD_ERR_INVALID_ARG;
    if (!valid_dtype(d->io_dtype) || !valid_dtype(d->y_dtype) || !valid_dtype(d->state_dtype))
        return SSD_ERR_INVALID_ARG;
    if (d->headdim % 8 != 0 || d->dstate % 8 != 0 || d->headdim > 256 || d->dstate > 256)
        return SSD_ERR_UNSUPPORTED;
    if (d->batch * d->nheads > (int64_t)0x7fffffff) return SSD_ERR_UNSUPPORTED;
    if (!state || !x || !dt_raw || !A || !B || !C || !y) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {state, x, dt_raw, dt_bias, A, B, C, D, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGNMENT;
    const size_t bh = (size_t)d->batch * d->nheads;
    const size_t s_bytes = bh * d->dstate * d->headdim * dsize(d->state_dtype);
    const size_t y_bytes = bh * d->headdim * dsize(d->y_dtype);
    const size_t x_bytes = bh * d->headdim * dsize(d->io_dtype);
    if (overlaps(y, y_bytes, state, s_bytes) || overlaps(y, y_bytes, x, x_bytes) ||
        overlaps(state, s_bytes, x, x_bytes))
        return SSD_ERR_INVALID_ARG;
    if (d->batch == 0) return SSD_OK;
    DecodeArgs a{};
    a.batch = d->batch; a.H = d->nheads; a.P = d->headdim; a.N = d->dstate; a.G = d->ngroups;
    a.io_bf16 = d->io_dtype == SSD_BF16; a.y_bf16 = d->y_dtype == SSD_BF16;
    a.state_bf16 = d->state_dtype == SSD_BF16;
    a.state = state; a.x = x; a.dt_raw = dt_raw; a.B = B; a.C = C;
    a.dt_bias = dt_bias; a.A = A; a.D = D; a.y = y;
    const cudaError_t e = launch_state_update(a, (cudaStream_t)stream);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status_t ssd_state_update_mamba3(const ssd_decode_desc_t* d, void* state, const void* x, const void* x_prev,
                                     const void* dt_raw, const float* dt_bias, const float* A, const void* B,
                                     const void* B_prev, const void* C, const float* D, const float* lam,
                                     const float* theta, void* y, void* stream) {
    if (!d) return SSD_ERR_INVALID_ARG;
    if (d->batch < 0 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 || d->ngroups < 1 ||
        d->nheads % d->ngroups != 0)
        return SSD_ERR_INVALID_ARG;
    if (!valid_dtype(d->io_dtype) || !valid_dtype(d->y_dtype) || !valid_dtype(d->state_dtype))
        return SSD_ERR_INVALID_ARG;
    if (d->headdim % 8 != 0 || d->dstate % 8 != 0 || d->headdim > 256 || d->dstate > 256)
        return SSD_ERR_UNSUPPORTED;
    if (!mamba3_step_supports(d->headdim, d->dstate, d->state_dtype == SSD_BF16)) return SSD_ERR_UNSUPPORTED;
    if (d->batch * d->nheads > (int64_t)0x7fffffff) return SSD_ERR_UNSUPPORTED;
    if (!state || !x || !dt_raw || !A || !B || !C || !y) return SSD_ERR_INVALID_ARG;
    if ((x_prev == nullptr) != (B_prev == nullptr)) return SSD_ERR_INVALID_ARG;   // both or neither
    const void* ptrs[] = {state, x, x_prev, dt_raw, dt_bias, A, B, B_prev, C, D, lam, theta, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGNMENT;
    const size_t bh = (size_t)d->batch * d->nheads;
    const size_t s_bytes = bh * d->dstate * d->headdim * dsize(d->state_dtype);
    const size_t y_bytes = bh * d->headdim * dsize(d->y_dtype);
    const size_t x_bytes = bh * d->headdim * dsize(d->io_dtype);
    if (overlaps(y, y_bytes, state, s_bytes) || overlaps(y, y_bytes, x, x_bytes) ||
        overlaps(state, s_bytes, x, x_bytes) || overlaps(y, y_bytes, x_prev, x_bytes) ||
        overlaps(state, s_bytes, x_prev, x_bytes))
        return SSD_ERR_INVALID_ARG;
    if (d->batch == 0) return SSD_OK;
    Mamba3StepArgs a{};
    a.batch = d->batch; a.H = d->nheads; a.P = d->headdim; a.N = d->dstate; a.G = d->ngroups;
    a.io_bf16 = d->io_dtype == SSD_BF16; a.y_bf16 = d->y_dtype == SSD_BF16;
    a.state_bf16 = d->state_dtype == SSD_BF16;
    a.state = state; a.x = x; a.x_prev = x_prev; a.dt_raw = dt_raw; a.B = B; a.B_prev = B_prev; a.C = C;
    a.dt_bias = dt_bias; a.A = A; a.D = D; a.lam = lam; a.theta = theta; a.y = y;
    const cudaError_t e = launch_mamba3_step(a, (cudaStream_t)stream);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status_t ssd_state_update_mimo(const ssd_mimo_desc_t* d, void* state, const void* x, const void* dt_raw,
                                   const float* dt_bias, const float* A, const void* B, const void* C,
                                   const float* D, void* y, void* stream) {
    if (!d) return SSD_ERR_INVALID_ARG;
    if (d->batch < 0 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 || d->ngroups < 1 || d->rank < 1 ||
        d->nheads % d->ngroups != 0)
        return SSD_ERR_INVALID_ARG;
    if (!valid_dtype(d->io_dtype) || !valid_dtype(d->y_dtype) || !valid_dtype(d->state_dtype))
        return SSD_ERR_INVALID_ARG;
    const int64_t P = d->headdim, R = d->rank;
    if (!(P == 8 || P == 16 || P == 32 || P == 64 || P == 128)) return SSD_ERR_UNSUPPORTED;
    if (!(R == 1 || R == 2 || R == 4 || R == 8)) return SSD_ERR_UNSUPPORTED;
    if (d->dstate % 8 != 0 || d->dstate > 256) return SSD_ERR_UNSUPPORTED;
    if (d->batch * d->nheads > (int64_t)0x7fffffff) return SSD_ERR_UNSUPPORTED;
    if (!state || !x || !dt_raw || !A || !B || !C || !y) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {state, x, dt_raw, dt_bias, A, B, C, D, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGNMENT;
    const size_t bh = (size_t)d->batch * d->nheads;
    const size_t s_bytes = bh * d->dstate * P * dsize(d->state_dtype);
    const size_t y_bytes = bh * R * P * dsize(d->y_dtype);
    const size_t x_bytes = bh * R * P * dsize(d->io_dtype);
    if (overlaps(y, y_bytes, state, s_bytes) || overlaps(y, y_bytes, x, x_bytes) ||
        overlaps(state, s_bytes, x, x_bytes))
        return SSD_ERR_INVALID_ARG;
    if (d->batch == 0) return SSD_OK;
    MimoArgs a{};
    a.batch = d->batch; a.H = d->nheads; a.P = P; a.N = d->dstate; a.G = d->ngroups; a.R = R;
    a.io_bf16 = d->io_dtype == SSD_BF16; a.y_bf16 = d->y_dtype == SSD_BF16;
    a.state_bf16 = d->state_dtype == SSD_BF16;
    a.state = state; a.x = x; a.dt_raw = dt_raw; a.B = B; a.C = C;
    a.dt_bias = dt_bias; a.A = A; a.D = D; a.y = y;
    const cudaError_t e = launch_mimo_step(a, (cudaStream_t)stream);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status_t ssd_replay_buffer_size(const ssd_replay_desc_t* desc, size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    const ssd_status_t st = check_replay_desc(desc);
    if (st != SSD_OK) return st;
    *bytes = replay_layout(desc).total;
    return SSD_OK;
}

ssd_status_t ssd_replay_step(const ssd_replay_desc_t* d, void* checkpoint, void* buffer, int32_t fill,
                             const void* x, const void* dt_raw, const float* dt_bias, const float* A,
                             const void* B, const void* C, const float* D, void* y, void* stream) {
    ssd_status_t st = check_replay_desc(d);
    if (st != SSD_OK) return st;
    if (fill < 0 || fill >= d->capacity) return SSD_ERR_INVALID_ARG;
    if (!checkpoint || !buffer || !x || !dt_raw || !A || !B || !C || !y) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {checkpoint, x, dt_raw, dt_bias, A, B, C, D, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGNMENT;
    if ((uintptr_t)buffer & 255u) return SSD_ERR_ALIGNMENT;
    const ReplayLayout lay = replay_layout(d);
    const size_t bh = (size_t)d->batch * d->nheads;
    const size_t s_bytes = bh * d->dstate * d->headdim * dsize(d->state_dtype);
    const size_t y_bytes = bh * d->headdim * dsize(d->y_dtype);
    const size_t x_bytes = bh * d->headdim * dsize(d->io_dtype);
    if (overlaps(y, y_bytes, checkpoint, s_bytes) || overlaps(y, y_bytes, x, x_bytes) ||
        overlaps(checkpoint, s_bytes, x, x_bytes) || overlaps(buffer, lay.total, checkpoint, s_bytes) ||
        overlaps(buffer, lay.total, y, y_bytes) || overlaps(buffer, lay.total, x, x_bytes))
        return SSD_ERR_INVALID_ARG;
    if (d->batch == 0) return SSD_OK;
    ReplayArgs a{};
    a.batch = d->batch; a.H = d->nheads; a.P = d->headdim; a.N = d->dstate; a.G = d->ngroups;
    a.K = d->capacity; a.fill = fill;
    a.io_bf16 = d->io_dtype == SSD_BF16; a.y_bf16 = d->y_dtype == SSD_BF16;
    a.state_bf16 = d->state_dtype == SSD_BF16;
    a.ckpt = checkpoint;
    a.xb = (char*)buffer + lay.off_x;
    a.Bb = (char*)buffer + lay.off_B;
    a.dtb = (float*)((char*)buffer + lay.off_dt);
    a.cumb = (float*)((char*)buffer + lay.off_cum);
    a.cb = (float*)((char*)buffer + lay.off_cb);
    a.x = x; a.dt_raw = dt_raw; a.B = B; a.C = C; a.dt_bias = dt_bias; a.A = A; a.D = D; a.y = y;
    const cudaError_t e = launch_replay_step(a, (cudaStream_t)stream);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status_t ssd_debug_inject(uint32_t faults) {
    if (faults & ~(uint32_t)SSD_FAULT_DROP_RUN_PUBLISH) return SSD_ERR_INVALID_ARG;
    g_debug_faults.store(faults, std::memory_order_relaxed);
    return SSD_OK;
}

ssd_status_t ssd_get_device_error(void* stream, uint32_t* detail) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return SSD_ERR_CUDA;
    if (v) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return SSD_ERR_CUDA;
    }
    if (detail) *detail = v;
    return v ? SSD_ERR_DEVICE_TIMEOUT : SSD_OK;
}

}  // extern "C"
