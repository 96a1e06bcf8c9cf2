// m3_api.cu -- the C ABI of include/m3.h: argument checks, the launch plan,
// the workspace layout and the dispatch to the kernels.
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <vector>

#define M3_BOUNDS_FILE 9
#include "m3_bounds.cuh"
#include "m3_common.cuh"
#include "m3_kernels.h"
#include "m3_nvtx.h"

namespace m3 {

#if M3_DEBUG_BOUNDS
// readers of the per-file check records (each kernel file defines its own)
cudaError_t bounds_take_scan_tc(BoundsRecord* out, bool clear);
cudaError_t bounds_take_scan_simt(BoundsRecord* out, bool clear);
cudaError_t bounds_take_step(BoundsRecord* out, bool clear);
cudaError_t bounds_take_rope(BoundsRecord* out, bool clear);
cudaError_t bounds_take_seq(BoundsRecord* out, bool clear);
cudaError_t bounds_take_bwd(BoundsRecord* out, bool clear);
cudaError_t bounds_take_phase(BoundsRecord* out, bool clear);
cudaError_t bounds_take_scan_ws(BoundsRecord* out, bool clear);
cudaError_t bounds_take_api(BoundsRecord* out, bool clear);

// the check itself, on one index the caller chose (m3_selftest_bounds_check)
__global__ void bounds_selftest_kernel(float* buf, long long index, long long limit) {
    if (M3_IN(1, index, limit)) buf[index] = 1.f;
}
#endif

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static m3_status check_dims(const m3_dims* d, bool need_seq) {
    if (!d) return M3_ERR_INVALID_ARG;
    if (d->batch < 0 || d->nheads < 1 || d->ngroups < 1 || d->headdim < 1 || d->dstate < 2 ||
        d->rank < 1)
        return M3_ERR_INVALID_ARG;
    if (need_seq && (d->seqlen < 0 || d->chunk < 1)) return M3_ERR_INVALID_ARG;
    if (d->dstate % 2 != 0 || d->nheads % d->ngroups != 0) return M3_ERR_INVALID_ARG;
    if (d->io_dtype != M3_F32 && d->io_dtype != M3_BF16) return M3_ERR_INVALID_ARG;
    // sizes whose element counts would overflow the kernels' 32-bit per-head indexing
    if ((long long)d->dstate * d->headdim > (1LL << 24) || d->rank > 64 || d->dstate > 1024)
        return M3_ERR_UNSUPPORTED;
    return M3_OK;
}

static bool ptrs_ok(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (!p || !aligned16(p)) return false;
    return true;
}

static bool opt_ptrs_ok(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (p && !aligned16(p)) return false;
    return true;
}

static size_t io_bytes(const m3_dims& d) { return d.io_dtype == M3_BF16 ? 2 : 4; }

// ---------------------------------------------------------------- plan --
struct Plan {
    int path;    // 0 = SIMT float32, 1 = tcgen05
    int qs;      // chunk length the kernels use (tokens)
    int nseg;    // segments per (b, h)
    int cps;     // chunks per segment
    int kernel;  // tcgen05 path: 1 = tile kernel (k_scan_tc.cu), 2 = persistent kernel (k_scan_ws.cu)
    int wmode;   // persistent kernel: 0 = ranges with hand-off, 1 = one segment per CTA
    int grid;    // persistent kernel: CTAs
    int M;       // persistent kernel, mode 0: tiles per CTA
    int nt;      // tiles (chunks) per sequence
};

static int env_int(const char* name, int dflt) {
    const char* v = getenv(name);
    if (!v || !*v) return dflt;
    return atoi(v);
}

static bool env_is(const char* name, const char* val) {
    const char* v = getenv(name);
    return v && strcmp(v, val) == 0;
}

// SM count of the current device: a device attribute cached per device
// (atomics: calls may come from several host threads); 148, the B200's
// count, when no device can be queried
int device_sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Path and chunking.  tcgen05 path: a chunk is one 128-row UMMA tile
// (128/R tokens).  SIMT path: the kernel keeps one chunk of rotated B, C, X,
// the masked Gram and the state in shared memory, so it uses the caller's
// chunk when that fits, else halves it until it does.  The chunked result
// does not depend on the chunk length except through rounding.
// Segments: a (b, h) sequence is cut into segments only when there are too
// few sequences to give every SM work (two resident CTAs per SM).
static m3_status make_plan(const m3_dims& d, Plan* pl) {
    const size_t kMaxSmem = 200 * 1024;
    const bool tc = tc_eligible(d) && !env_is("M3_SCAN_PATH", "simt");
    // tcgen05 path: the tile kernel (two CTAs per SM, one sequence or
    // segment each) unless M3_TC_KERNEL=persistent asks for the persistent
    // warp-specialised kernel (one CTA per SM; measured slower on every layer
    // workload, kept as an option)
    pl->kernel = tc ? (env_is("M3_TC_KERNEL", "persistent") ? 2 : 1) : 0;
    pl->wmode = 0;
    pl->grid = 0;
    pl->M = 0;
    if (pl->kernel == 2) {
        // persistent kernel: one CTA per SM.  With at least as many (b, h)
        // sequences as SMs the concatenated tiles are cut into one range per
        // CTA (a sequence split by a range boundary hands its state from its
        // head to its tail); with fewer, each sequence is cut into segments
        // (at most one CTA each, all resident) whose incoming states come from
        // a summary pass.  M3_SCAN_NSEG forces segments.
        const int qs = tc_tile_tokens(d.rank);
        const long long nt = d.seqlen > 0 ? (d.seqlen + qs - 1) / qs : 0;
        const long long units = (long long)d.batch * d.nheads;
        const long long sms = device_sm_count();
        const int forced = env_int("M3_SCAN_NSEG", 0);
        pl->path = 1;
        pl->qs = qs;
        pl->nt = (int)nt;
        if (forced <= 0 && units >= sms && nt > 0) {
            const long long total = units * nt;
            if (total > (1LL << 30)) return M3_ERR_UNSUPPORTED;
            pl->wmode = 0;
            pl->M = (int)((total + sms - 1) / sms);
            pl->grid = (int)sms;
            pl->nseg = 1;
            pl->cps = (int)nt;
            return M3_OK;
        }
        long long nseg = 1;
        if (forced > 0) {
            nseg = forced;
        } else if (units > 0) {
            nseg = sms / units;
            if (nseg > nt / 2) nseg = nt / 2;
        }
        if (nseg < 1) nseg = 1;
        if (nt > 0 && nseg > nt) nseg = nt;
        const long long cps = nt > 0 ? (nt + nseg - 1) / nseg : 1;
        if (nt > 0) nseg = (nt + cps - 1) / cps;
        if (units * nseg > 0x7fffffffLL) return M3_ERR_UNSUPPORTED;
        pl->wmode = 1;
        pl->nseg = (int)nseg;
        pl->cps = (int)cps;
        pl->grid = (int)(units * nseg);
        return M3_OK;
    }
    int qs;
    if (tc) {
        qs = tc_tile_tokens(d.rank);
    } else {
        qs = d.chunk;
        if (d.seqlen > 0 && qs > d.seqlen) qs = d.seqlen;
        while (qs > 1 && simt_smem_bytes(qs, d.rank, d.dstate, d.headdim, false) > kMaxSmem) qs = (qs + 1) / 2;
        if (simt_smem_bytes(qs, d.rank, d.dstate, d.headdim, false) > kMaxSmem) return M3_ERR_UNSUPPORTED;
    }
    const long long nchunks = d.seqlen > 0 ? (d.seqlen + qs - 1) / qs : 0;
    const long long units = (long long)d.batch * d.nheads;
    const long long sms = device_sm_count();
    int nseg = 1;
    if (units > 0 && units < sms && nchunks >= 4) {
        long long want = (2 * sms) / units;
        long long cap = nchunks / 2;
        nseg = (int)(want < cap ? want : cap);
        if (nseg < 1) nseg = 1;
    }
    const int forced = env_int("M3_SCAN_NSEG", 0);   // tuning / test knob
    if (forced > 0) nseg = (int)(forced < nchunks ? forced : (nchunks > 0 ? nchunks : 1));
    int cps = nchunks > 0 ? (int)((nchunks + nseg - 1) / nseg) : 1;
    if (nchunks > 0) nseg = (int)((nchunks + cps - 1) / cps);   // drop empty segments
    pl->path = tc ? 1 : 0;
    pl->qs = qs;
    pl->nseg = nseg;
    pl->cps = cps;
    return M3_OK;
}

struct WsLayout {
    size_t sloc, decay, phase, sin, ho_state, ho_flag, total;
};

static size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

static WsLayout ws_layout(const m3_dims& d, const Plan& pl) {
    WsLayout w;
    size_t off = kWorkspaceHeaderBytes;
    const size_t units = (size_t)d.batch * d.nheads * (pl.nseg > 1 ? pl.nseg : 0);
    const size_t NP = (size_t)d.dstate * d.headdim;
    w.sloc = off;  off = round256(off + units * NP * sizeof(float));
    w.decay = off; off = round256(off + units * sizeof(float));
    w.phase = off; off = round256(off + units * (d.dstate / 2) * sizeof(float));
    w.sin = off;   off = round256(off + units * NP * sizeof(float));
    const size_t slots = (pl.kernel == 2 && pl.wmode == 0) ? (size_t)pl.grid : 0;
    w.ho_state = off; off = round256(off + slots * NP * sizeof(float));
    w.ho_flag = off;  off = round256(off + slots * sizeof(int));
    w.total = off;
    return w;
}

}  // namespace m3

using namespace m3;

extern "C" {

const char* m3_status_string(m3_status s) {
    switch (s) {
        case M3_OK: return "ok";
        case M3_ERR_INVALID_ARG: return "invalid argument (null, misaligned or bad size)";
        case M3_ERR_UNSUPPORTED: return "shape not supported by the kernels";
        case M3_ERR_WORKSPACE: return "workspace missing or too small";
        case M3_ERR_CUDA: return "CUDA runtime error";
        case M3_ERR_DEVICE_TIMEOUT: return "a bounded on-chip wait expired on the device";
    }
    return "unknown status";
}

m3_status m3_scan_workspace_size(const m3_dims* d, size_t* bytes) {
    if (!bytes) return M3_ERR_INVALID_ARG;
    m3_status s = check_dims(d, true);
    if (s != M3_OK) return s;
    Plan pl;
    s = make_plan(*d, &pl);
    if (s != M3_OK) return s;
    *bytes = ws_layout(*d, pl).total;
    return M3_OK;
}

m3_status m3_scan_plan(const m3_dims* d, int* launches, int* segments, int* chunk_used, int* path) {
    m3_status s = check_dims(d, true);
    if (s != M3_OK) return s;
    Plan pl;
    s = make_plan(*d, &pl);
    if (s != M3_OK) return s;
    const bool work = d->batch > 0 && d->seqlen > 0;
    if (launches) *launches = work ? (pl.nseg > 1 ? 3 : 1) : 0;   // summary, combine, main
    if (segments) *segments = pl.nseg;
    if (chunk_used) *chunk_used = pl.qs;
    if (path) *path = pl.path;
    return M3_OK;
}

m3_status m3_scan_fwd(const m3_dims* d, const void* x, const void* B, const void* C, const float* dt,
                      const float* A, const float* lambda, const float* theta, const m3_carry* init,
                      void* y, m3_carry* fin, void* workspace, size_t ws_bytes, void* stream) {
    const NvtxRange range("m3_scan_fwd");
    m3_status s = check_dims(d, true);
    if (s != M3_OK) return s;
    const bool work = d->batch > 0 && d->seqlen > 0;
    if (work && !ptrs_ok({x, B, C, dt, A, lambda, theta, y})) return M3_ERR_INVALID_ARG;
    if (init && !opt_ptrs_ok({init->h, init->prev_B, init->prev_x})) return M3_ERR_INVALID_ARG;
    if (fin && !opt_ptrs_ok({fin->h, fin->prev_B, fin->prev_x})) return M3_ERR_INVALID_ARG;
    Plan pl;
    s = make_plan(*d, &pl);
    if (s != M3_OK) return s;
    const WsLayout w = ws_layout(*d, pl);
    if (!workspace || !aligned16(workspace) || ws_bytes < w.total) return M3_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t NP = (size_t)d->dstate * d->headdim;
    const size_t units = (size_t)d->batch * d->nheads;

    if (!work) {
        // no tokens: the carry passes through unchanged
        if (fin && d->batch > 0) {
            const size_t hb = units * NP * sizeof(float);
            const size_t bb = units * d->rank * d->dstate * io_bytes(*d);
            const size_t xb = units * d->rank * d->headdim * io_bytes(*d);
            cudaError_t e = cudaSuccess;
            if (fin->h)
                e = (init && init->h) ? cudaMemcpyAsync(fin->h, init->h, hb, cudaMemcpyDeviceToDevice, st)
                                      : cudaMemsetAsync(fin->h, 0, hb, st);
            if (e == cudaSuccess && fin->prev_B)
                e = (init && init->prev_B)
                        ? cudaMemcpyAsync(fin->prev_B, init->prev_B, bb, cudaMemcpyDeviceToDevice, st)
                        : cudaMemsetAsync(fin->prev_B, 0, bb, st);
            if (e == cudaSuccess && fin->prev_x)
                e = (init && init->prev_x)
                        ? cudaMemcpyAsync(fin->prev_x, init->prev_x, xb, cudaMemcpyDeviceToDevice, st)
                        : cudaMemsetAsync(fin->prev_x, 0, xb, st);
            if (e != cudaSuccess) return M3_ERR_CUDA;
        }
        return M3_OK;
    }

    ScanParams q;
    memset(&q, 0, sizeof(q));
    q.batch = d->batch; q.seqlen = d->seqlen; q.nheads = d->nheads; q.ngroups = d->ngroups;
    q.headdim = d->headdim; q.dstate = d->dstate; q.rank = d->rank;
    q.qs = pl.qs; q.nseg = pl.nseg; q.cps = pl.cps;
    q.x = x; q.B = B; q.C = C; q.dt = dt; q.A = A; q.lam = lambda; q.theta = theta;
    if (init) { q.init_h = init->h; q.init_pB = init->prev_B; q.init_pX = init->prev_x; }
    q.y = y;
    if (fin) { q.fin_h = fin->h; q.fin_pB = fin->prev_B; q.fin_pX = fin->prev_x; }
    char* ws = static_cast<char*>(workspace);
    q.ws_sloc = reinterpret_cast<float*>(ws + w.sloc);
    q.ws_decay = reinterpret_cast<float*>(ws + w.decay);
    q.ws_phase = reinterpret_cast<float*>(ws + w.phase);
    q.ws_sin = reinterpret_cast<float*>(ws + w.sin);
    int* status = reinterpret_cast<int*>(workspace);
    cudaError_t e;
    if (pl.kernel == 2) {
        e = cudaSuccess;
        if (pl.wmode == 1 && pl.nseg > 1) e = launch_scan_tc_summary(*d, q, status, st);
        if (e == cudaSuccess) {
            static std::atomic<int> calls{0};
            int id = calls.fetch_add(1, std::memory_order_relaxed) + 1;
            id = (id & 0x3fffffff) + 1;            // never 0: a cleared flag never matches
            WsPlanArgs pa;
            pa.mode = pl.wmode;
            pa.nt = pl.nt;
            pa.M = pl.M;
            pa.total = pl.nt * (int)units;
            pa.grid = pl.grid;
            pa.call_id = id;
            pa.ho_state = reinterpret_cast<float*>(ws + w.ho_state);
            pa.ho_flag = reinterpret_cast<int*>(ws + w.ho_flag);
            e = launch_scan_ws(*d, q, pa, status, st);
        }
    } else {
        e = pl.path == 1 ? launch_scan_tc(*d, q, status, st) : launch_scan_simt(*d, q, st);
    }
    return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

m3_status m3_step(const m3_dims* d, m3_carry* state, const void* x, const void* B, const void* C,
                  const float* dt, const float* A, const float* lambda, const float* theta, void* y,
                  void* stream) {
    const NvtxRange range("m3_step");
    m3_status s = check_dims(d, false);
    if (s != M3_OK) return s;
    if (!state) return M3_ERR_INVALID_ARG;
    if (d->batch > 0 &&
        !ptrs_ok({state->h, state->prev_B, state->prev_x, x, B, C, dt, A, lambda, theta, y}))
        return M3_ERR_INVALID_ARG;
    StepParams q;
    q.batch = d->batch; q.nheads = d->nheads; q.ngroups = d->ngroups;
    q.headdim = d->headdim; q.dstate = d->dstate;
    q.h = state->h; q.prev_B = state->prev_B; q.prev_x = state->prev_x;
    q.x = x; q.B = B; q.C = C; q.dt = dt; q.A = A; q.lam = lambda; q.theta = theta; q.y = y;
    return launch_step(*d, q, (cudaStream_t)stream);
}

m3_status m3_rope_bc(const m3_dims* d, const void* B, const void* C, const float* dt, const float* theta,
                     void* B_rot, void* C_rot, float* phase, void* stream) {
    const NvtxRange range("m3_rope_bc");
    m3_status s = check_dims(d, false);
    if (s != M3_OK) return s;
    if (d->seqlen < 0) return M3_ERR_INVALID_ARG;
    if (d->batch > 0 && d->seqlen > 0 && !ptrs_ok({B, C, dt, theta, B_rot, C_rot}))
        return M3_ERR_INVALID_ARG;
    if (!opt_ptrs_ok({phase})) return M3_ERR_INVALID_ARG;
    RopeParams q;
    q.batch = d->batch; q.seqlen = d->seqlen; q.nheads = d->nheads; q.ngroups = d->ngroups;
    q.dstate = d->dstate; q.rank = d->rank;
    q.B = B; q.C = C; q.dt = dt; q.theta = theta; q.B_rot = B_rot; q.C_rot = C_rot; q.phase = phase;
    return launch_rope(*d, q, (cudaStream_t)stream);
}

static size_t bwd_ws_bytes(const m3_dims& d) {
    const size_t kBwdCkpt = (size_t)bwd_block_tokens(d);     // tokens between checkpoints
    const size_t units = (size_t)d.batch * d.nheads, NP = (size_t)d.dstate * d.headdim;
    const size_t nck = d.seqlen > 0 ? (size_t)(d.seqlen + kBwdCkpt - 1) / kBwdCkpt : 0;
    size_t off = kWorkspaceHeaderBytes;
    off += (units * nck * NP * sizeof(float) + 255) & ~(size_t)255;
    off += (units * kBwdCkpt * NP * sizeof(float) + 255) & ~(size_t)255;
    return off;
}

m3_status m3_scan_bwd_workspace_size(const m3_dims* d, size_t* bytes) {
    m3_status s = check_dims(d, true);
    if (s != M3_OK) return s;
    if (!bytes) return M3_ERR_INVALID_ARG;
    if (!bwd_supported(*d)) return M3_ERR_UNSUPPORTED;
    *bytes = bwd_ws_bytes(*d);
    return M3_OK;
}

m3_status m3_scan_bwd(const m3_dims* d, const void* x, const void* B, const void* C, const float* dt,
                      const float* A, const float* lambda, const float* theta, const m3_carry* init,
                      const void* dy, const m3_grad_carry* d_final, float* dx, float* dB, float* dC, float* ddt,
                      float* dA, float* dlambda, float* dtheta, m3_grad_carry* d_init, void* workspace,
                      size_t ws_bytes, void* stream) {
    const NvtxRange range("m3_scan_bwd");
    m3_status s = check_dims(d, true);
    if (s != M3_OK) return s;
    if (!bwd_supported(*d)) return M3_ERR_UNSUPPORTED;
    const bool work = d->batch > 0 && d->seqlen > 0;
    if (!ptrs_ok({A, dA})) return M3_ERR_INVALID_ARG;
    if (work && !ptrs_ok({x, B, C, dt, lambda, theta, dy, dx, dB, dC, ddt, dlambda, dtheta}))
        return M3_ERR_INVALID_ARG;
    if (init && !opt_ptrs_ok({init->h, init->prev_B, init->prev_x})) return M3_ERR_INVALID_ARG;
    if (d_final && !opt_ptrs_ok({d_final->h, d_final->prev_B, d_final->prev_x})) return M3_ERR_INVALID_ARG;
    if (d_init && !opt_ptrs_ok({d_init->h, d_init->prev_B, d_init->prev_x})) return M3_ERR_INVALID_ARG;
    const size_t need = bwd_ws_bytes(*d);
    if (!workspace || !aligned16(workspace) || ws_bytes < need) return M3_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t tokg = (size_t)d->batch * d->seqlen * d->ngroups;
    // the accumulated outputs start at zero
    if (cudaMemsetAsync(dA, 0, sizeof(float) * d->nheads, st) != cudaSuccess) return M3_ERR_CUDA;
    if (work) {
        if (cudaMemsetAsync(dB, 0, sizeof(float) * tokg * d->rank * d->dstate, st) != cudaSuccess ||
            cudaMemsetAsync(dC, 0, sizeof(float) * tokg * d->rank * d->dstate, st) != cudaSuccess ||
            cudaMemsetAsync(dtheta, 0, sizeof(float) * tokg * (d->dstate / 2), st) != cudaSuccess)
            return M3_ERR_CUDA;
    }
    BwdParams q;
    q.batch = d->batch; q.seqlen = d->seqlen; q.nheads = d->nheads; q.ngroups = d->ngroups;
    const int kBwdCkpt = bwd_block_tokens(*d);
    q.headdim = d->headdim; q.dstate = d->dstate; q.rank = d->rank; q.K = kBwdCkpt;
    q.x = x; q.B = B; q.C = C; q.dt = dt; q.A = A; q.lam = lambda; q.theta = theta;
    q.init_h = init ? init->h : nullptr;
    q.init_pB = init ? init->prev_B : nullptr;
    q.init_pX = init ? init->prev_x : nullptr;
    q.dy = dy;
    q.d_fin_h = d_final ? d_final->h : nullptr;
    q.d_fin_pB = d_final ? d_final->prev_B : nullptr;
    q.d_fin_pX = d_final ? d_final->prev_x : nullptr;
    q.dx = dx; q.dB = dB; q.dC = dC; q.ddt = ddt; q.dA = dA; q.dlam = dlambda; q.dtheta = dtheta;
    q.d_init_h = d_init ? d_init->h : nullptr;
    q.d_init_pB = d_init ? d_init->prev_B : nullptr;
    q.d_init_pX = d_init ? d_init->prev_x : nullptr;
    const size_t units = (size_t)d->batch * d->nheads, NP = (size_t)d->dstate * d->headdim;
    const size_t nck = d->seqlen > 0 ? (size_t)(d->seqlen + kBwdCkpt - 1) / kBwdCkpt : 0;
    char* base = static_cast<char*>(workspace);
    q.ws_ckpt = reinterpret_cast<float*>(base + kWorkspaceHeaderBytes);
    q.ws_scratch = reinterpret_cast<float*>(base + kWorkspaceHeaderBytes +
                                            ((units * nck * NP * sizeof(float) + 255) & ~(size_t)255));
    if (d->batch == 0) return M3_OK;
    return launch_bwd(*d, q, st) == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

// ------------------------------------------------------- phase interventions
struct PhaseLayout {
    size_t inner, perm, freq, theta, brot, crot, expd, total;
};

static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

static m3_status phase_layout(const m3_dims& d, int mode, PhaseLayout* l) {
    if (mode < M3_PHASE_NATIVE || mode > M3_PHASE_READ_ONLY) return M3_ERR_INVALID_ARG;
    const bool onesided = mode == M3_PHASE_WRITE_ONLY || mode == M3_PHASE_READ_ONLY;
    m3_dims di = d;
    if (onesided) di.ngroups = d.nheads;
    size_t inner = 0;
    m3_status s = m3_scan_workspace_size(&di, &inner);
    if (s != M3_OK) return s;
    const size_t NH = d.dstate / 2, tok = (size_t)d.batch * d.seqlen;
    const size_t io = d.io_dtype == M3_BF16 ? 2 : 4;
    l->inner = 0;
    size_t off = up256(inner);
    l->perm = off;  off = up256(off + (mode == M3_PHASE_SHUFFLE ? NH * sizeof(int) : 0));
    l->freq = off;  off = up256(off + (mode == M3_PHASE_FIXED ? (size_t)d.ngroups * NH * sizeof(float) : 0));
    const size_t th_groups = onesided ? (size_t)d.nheads : (size_t)d.ngroups;
    l->theta = off; off = up256(off + (mode == M3_PHASE_NATIVE ? 0 : tok * th_groups * NH * sizeof(float)));
    const size_t per_head = onesided ? tok * d.nheads * (size_t)d.rank * d.dstate * io : 0;
    l->brot = off;  off = up256(off + per_head);
    l->crot = off;  off = up256(off + per_head);
    l->expd = off;  off = up256(off + (onesided && d.ngroups != d.nheads ? per_head : 0));
    l->total = off;
    return M3_OK;
}

m3_status m3_scan_phase_workspace_size(const m3_dims* d, int mode, size_t* bytes) {
    m3_status s = check_dims(d, true);
    if (s != M3_OK) return s;
    if (!bytes) return M3_ERR_INVALID_ARG;
    PhaseLayout l;
    s = phase_layout(*d, mode, &l);
    if (s != M3_OK) return s;
    *bytes = l.total;
    return M3_OK;
}

m3_status m3_scan_fwd_phase(const m3_dims* d, int mode, const int* perm, const float* freq, const void* x,
                            const void* B, const void* C, const float* dt, const float* A, const float* lambda,
                            const float* theta, const m3_carry* init, void* y, m3_carry* final_state,
                            void* workspace, size_t ws_bytes, void* stream) {
    const NvtxRange range("m3_scan_fwd_phase");
    m3_status s = check_dims(d, true);
    if (s != M3_OK) return s;
    PhaseLayout l;
    s = phase_layout(*d, mode, &l);
    if (s != M3_OK) return s;
    const int NH = d->dstate / 2;
    if (mode == M3_PHASE_SHUFFLE) {
        if (!perm) return M3_ERR_INVALID_ARG;
        std::vector<char> seen(NH, 0);
        for (int i = 0; i < NH; ++i) {
            if (perm[i] < 0 || perm[i] >= NH || seen[perm[i]]) return M3_ERR_INVALID_ARG;
            seen[perm[i]] = 1;
        }
    }
    if (mode == M3_PHASE_FIXED && !freq) return M3_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || ws_bytes < l.total) return M3_ERR_WORKSPACE;
    const bool work = d->batch > 0 && d->seqlen > 0;
    if (work && !ptrs_ok({x, B, C, dt, A, lambda, theta, y})) return M3_ERR_INVALID_ARG;
    if (mode == M3_PHASE_NATIVE)
        return m3_scan_fwd(d, x, B, C, dt, A, lambda, theta, init, y, final_state, workspace, ws_bytes, stream);
    cudaStream_t st = (cudaStream_t)stream;
    char* base = static_cast<char*>(workspace);
    const size_t tok = (size_t)d->batch * d->seqlen;
    const size_t inner_bytes = l.perm;            // the inner scan's workspace comes first
    if (mode == M3_PHASE_WRITE_ONLY || mode == M3_PHASE_READ_ONLY) {
        m3_dims di = *d;
        di.ngroups = d->nheads;
        void* brot = base + l.brot;
        void* crot = base + l.crot;
        float* th0 = reinterpret_cast<float*>(base + l.theta);
        if (work) {
            s = m3_rope_bc(d, B, C, dt, theta, brot, crot, nullptr, stream);
            if (s != M3_OK) return s;
            if (cudaMemsetAsync(th0, 0, tok * d->nheads * NH * sizeof(float), st) != cudaSuccess) return M3_ERR_CUDA;
        }
        // the side that keeps no rotation, one copy per head
        const void* plain = mode == M3_PHASE_WRITE_ONLY ? C : B;
        const void* plain_h = plain;
        if (work && d->ngroups != d->nheads) {
            const size_t row = (size_t)d->rank * d->dstate * (d->io_dtype == M3_BF16 ? 2 : 4);
            if (launch_expand_heads(plain, base + l.expd, tok, d->nheads, d->ngroups, row, st) != cudaSuccess)
                return M3_ERR_CUDA;
            plain_h = base + l.expd;
        }
        const void* Bp = mode == M3_PHASE_WRITE_ONLY ? brot : plain_h;
        const void* Cp = mode == M3_PHASE_WRITE_ONLY ? plain_h : crot;
        return m3_scan_fwd(&di, x, work ? Bp : B, work ? Cp : C, dt, A, lambda, work ? th0 : theta, init, y,
                           final_state, workspace, inner_bytes, stream);
    }
    // zero / reverse / shuffle / fixed: rewrite theta, then the ordinary scan
    int* dperm = reinterpret_cast<int*>(base + l.perm);
    float* dfreq = reinterpret_cast<float*>(base + l.freq);
    float* th = reinterpret_cast<float*>(base + l.theta);
    if (mode == M3_PHASE_SHUFFLE &&
        cudaMemcpyAsync(dperm, perm, NH * sizeof(int), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return M3_ERR_CUDA;
    if (mode == M3_PHASE_FIXED &&
        cudaMemcpyAsync(dfreq, freq, (size_t)d->ngroups * NH * sizeof(float), cudaMemcpyHostToDevice, st) !=
            cudaSuccess)
        return M3_ERR_CUDA;
    if (work && launch_theta_transform(mode, theta, dperm, dfreq, th, tok * d->ngroups, d->ngroups, NH, st) !=
                    cudaSuccess)
        return M3_ERR_CUDA;
    return m3_scan_fwd(d, x, B, C, dt, A, lambda, work ? th : theta, init, y, final_state, workspace, inner_bytes,
                       stream);
}

// ------------------------------------------------- transition variants --
// carry pass-through of an empty call (no tokens): shared by the variants
static m3_status carry_passthrough(const m3_dims* d, const m3_carry* init, m3_carry* fin, cudaStream_t st) {
    if (!fin || d->batch == 0) return M3_OK;
    const size_t units = (size_t)d->batch * d->nheads;
    const size_t hb = units * d->dstate * d->headdim * sizeof(float);
    const size_t bb = units * d->rank * d->dstate * io_bytes(*d);
    const size_t xb = units * d->rank * d->headdim * io_bytes(*d);
    cudaError_t e = cudaSuccess;
    if (fin->h)
        e = (init && init->h) ? cudaMemcpyAsync(fin->h, init->h, hb, cudaMemcpyDeviceToDevice, st)
                              : cudaMemsetAsync(fin->h, 0, hb, st);
    if (e == cudaSuccess && fin->prev_B)
        e = (init && init->prev_B) ? cudaMemcpyAsync(fin->prev_B, init->prev_B, bb, cudaMemcpyDeviceToDevice, st)
                                   : cudaMemsetAsync(fin->prev_B, 0, bb, st);
    if (e == cudaSuccess && fin->prev_x)
        e = (init && init->prev_x) ? cudaMemcpyAsync(fin->prev_x, init->prev_x, xb, cudaMemcpyDeviceToDevice, st)
                                   : cudaMemsetAsync(fin->prev_x, 0, xb, st);
    return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

static m3_status scan_variant(const m3_dims* d, int regime, const void* u, const void* x, const void* B,
                              const void* C, const float* dt, const float* A, const float* lambda,
                              const float* theta, const m3_carry* init, void* y, m3_carry* fin, void* stream) {
    m3_status s = check_dims(d, true);
    if (s != M3_OK) return s;
    if (regime < 0 || regime > 2) return M3_ERR_INVALID_ARG;
    if (!seq_supported(*d)) return M3_ERR_UNSUPPORTED;
    const bool work = d->batch > 0 && d->seqlen > 0;
    if (work && !ptrs_ok({x, B, C, dt, A, lambda, theta, y})) return M3_ERR_INVALID_ARG;
    if (init && !opt_ptrs_ok({init->h, init->prev_B, init->prev_x})) return M3_ERR_INVALID_ARG;
    if (fin && !opt_ptrs_ok({fin->h, fin->prev_B, fin->prev_x})) return M3_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (!work) return carry_passthrough(d, init, fin, st);
    SeqParams q;
    memset(&q, 0, sizeof(q));
    q.batch = d->batch; q.seqlen = d->seqlen; q.nheads = d->nheads; q.ngroups = d->ngroups;
    q.headdim = d->headdim; q.dstate = d->dstate; q.rank = d->rank; q.regime = regime;
    q.x = x; q.B = B; q.C = C; q.u = u; q.dt = dt; q.A = A; q.lam = lambda; q.theta = theta;
    if (init) { q.init_h = init->h; q.init_pB = init->prev_B; q.init_pX = init->prev_x; }
    q.y = y;
    if (fin) { q.fin_h = fin->h; q.fin_pB = fin->prev_B; q.fin_pX = fin->prev_x; }
    return launch_seq(*d, q, st) == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

m3_status m3_scan_fwd_damped(const m3_dims* d, int regime, const void* x, const void* B, const void* C,
                             const float* dt, const float* A, const float* lambda, const float* theta,
                             const m3_carry* init, void* y, m3_carry* final_state, void* stream) {
    const NvtxRange range("m3_scan_fwd_damped");
    return scan_variant(d, regime, nullptr, x, B, C, dt, A, lambda, theta, init, y, final_state, stream);
}

m3_status m3_scan_fwd_reflect(const m3_dims* d, const void* u, const void* x, const void* B, const void* C,
                              const float* dt, const float* A, const float* lambda, const float* theta,
                              const m3_carry* init, void* y, m3_carry* final_state, void* stream) {
    const NvtxRange range("m3_scan_fwd_reflect");
    // u is read only when there are tokens (like the other inputs)
    if (d && d->batch > 0 && d->seqlen > 0 && !ptrs_ok({u})) return M3_ERR_INVALID_ARG;
    return scan_variant(d, 0, u, x, B, C, dt, A, lambda, theta, init, y, final_state, stream);
}

m3_status m3_selftest_bounded_wait(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || !aligned16(workspace) || workspace_bytes < kWorkspaceHeaderBytes) return M3_ERR_WORKSPACE;
    return launch_wait_selftest(reinterpret_cast<int*>(workspace), (cudaStream_t)stream) == cudaSuccess
               ? M3_OK
               : M3_ERR_CUDA;
}

m3_status m3_debug_bounds_report(m3_bounds_report* out, int clear) {
    if (!out) return M3_ERR_INVALID_ARG;
    memset(out, 0, sizeof(*out));
#if M3_DEBUG_BOUNDS
    using Take = cudaError_t (*)(BoundsRecord*, bool);
    // in file order (site = file * 1000 + check)
    const Take takes[] = {bounds_take_scan_tc, bounds_take_scan_simt, bounds_take_step,
                          bounds_take_rope,    bounds_take_seq,       bounds_take_bwd,
                          bounds_take_phase,   bounds_take_scan_ws,   bounds_take_api};
    out->enabled = 1;
    if (cudaDeviceSynchronize() != cudaSuccess) return M3_ERR_CUDA;
    for (Take take : takes) {
        BoundsRecord r;
        if (take(&r, clear != 0) != cudaSuccess) return M3_ERR_CUDA;
        if (r.failures != 0u && out->failures == 0u) {
            out->site = r.site;
            out->index = r.index;
            out->limit = r.limit;
        }
        out->failures += r.failures;
    }
#else
    (void)clear;
#endif
    return M3_OK;
}

m3_status m3_selftest_bounds_check(float* buffer, long long capacity, long long index, long long limit,
                                   void* stream) {
    if (!buffer || capacity < 1 || index < 0 || index >= capacity || limit < 0 || limit > capacity)
        return M3_ERR_INVALID_ARG;
#if M3_DEBUG_BOUNDS
    bounds_selftest_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(buffer, index, limit);
    return cudaGetLastError() == cudaSuccess ? M3_OK : M3_ERR_CUDA;
#else
    (void)stream;
    return M3_ERR_UNSUPPORTED;
#endif
}

m3_status m3_device_status(void* workspace, void* stream) {
    if (!workspace) return M3_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return M3_ERR_CUDA;
    WorkspaceHeader hdr;
    if (cudaMemcpy(&hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost) != cudaSuccess) return M3_ERR_CUDA;
    if (hdr.status != 0) {
        if (cudaMemset(workspace, 0, sizeof(hdr)) != cudaSuccess) return M3_ERR_CUDA;
        return (m3_status)hdr.status;
    }
    return M3_OK;
}

}  // extern "C"

M3_BOUNDS_EXPORT(api)
