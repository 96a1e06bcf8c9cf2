// k_scan_ws.cu -- persistent, warp-specialised chunked prefill of the
// Mamba-3 SSM layer on the sm_100a tensor cores (tcgen05 + TMEM + TMA),
// bfloat16 io, N = 128, P = 64, rank R in {1, 2, 4, 8}.
//
// The algebra is that of the tile kernel (k_scan_tc.cu): with B and C
// rotated by their cumulative phase ("Mamba-3" summary, b-lab.team, section
// 2, Proposition 3) a 128-row tile (T = 128 / R tokens x R ranks) is the
// two-band masked matrix of section 1, and one float32 state is passed from
// tile to tile; the pending trapezoid term of a tile's last token rides in
// that state ("augmented" state).
//
// What differs is the schedule.  One CTA per SM runs for the whole call and
// overlaps consecutive tiles:
//   warp 0      TMA producer: B, C, X of tile k into a two-stage ring;
//   warp 1      MMA issuer (one thread):
//                 Y_inter = C~ S_bf, S_loc = B~^T (w X)  -> commit SL
//                 G = C~ B~^T (into G/P buffer k % 2)     -> commit G
//                 Y_intra = P X, P read from TMEM          -> commit YD, EMPTY
//   warps 2..5  epilogue (TMEM lane quarters 2, 3, 0, 1; thread = tile row or
//               state row): S = e^{a_last} S + S_loc and its bf16 copy S_bf,
//               P = (two-band decay mask) o G written back into TMEM as
//               bf16, y = Y_intra + e^{a_t} Y_inter stored as 128-byte rows;
//   warps 6..9  rotation: coefficients (a_t, gamma, c, w), the mask table,
//               the cumulative phase, B and C rotated in place (float32
//               arithmetic, one rounding to bf16), w X into its own buffer.
// So while the epilogue works on tile k, the rotation warps prepare tile k+1
// and the TMA engine loads tile k+2; the only per-tile chain left is
//   S_bf(k) -> Y_inter / S_loc (k+1) -> state update (k+1) -> S_bf(k+1).
//
// Work split.  Each (batch, head) sequence is a chain of nt tiles.  When
// there are at least as many chains as SMs, the chains are laid end to end
// and cut into equal ranges of M = ceil(total / #CTAs) tiles, one per CTA
// (McNaughton's wrap-around rule); a chain cut by a range boundary has its
// head at the end of one CTA's range and its tail at the start of the next
// one's.  Every CTA processes its head piece FIRST and its tail piece LAST,
// so a tail starts about M - nt tiles after its head has finished.  The head
// hands its final state (rotated back to the original frame, pending term
// included) to the tail through the workspace and a flag; the tail's
// epilogue warps wait for the flag (bounded).  The launch is cooperative, so
// every CTA is resident.  With fewer chains than SMs the sequences are cut
// into segments instead, whose incoming states come from the summary and
// combine passes (k_scan_tc.cu, k_scan_simt.cu), and this kernel runs one
// segment per CTA.
//
// Every mbarrier wait and the flag wait are bounded (1 s); on expiry the
// kernel records M3_ERR_DEVICE_TIMEOUT in the workspace status word, every
// role leaves its loop, in-flight copies and MMAs are drained (bounded) and
// the TMEM is freed.
#define M3_BOUNDS_FILE 8
#include "m3_bounds.cuh"
#include "m3_kernels.h"
#include "tc_ptx.cuh"

namespace m3 {
namespace wsk {

using namespace ptx;

constexpr int kRows = 128;
constexpr int kN = 128;
constexpr int kP = 64;
constexpr int kThreads = 512;      // 16 warps at 128 registers each
constexpr int kEW0 = 4;            // first epilogue warp (warps 4..7: TMEM lane quarters 0..3)
constexpr int kRW0 = 8;            // first rotation warp (warps 8..15)
constexpr int kEWT = 128;          // epilogue threads
constexpr int kRWT = 256;          // rotation threads
constexpr int kNE = 8;             // rotation warps = token groups per tile
constexpr int kTabs = 3;           // buffers of the per-tile tables (see the rotation warps)
constexpr unsigned kFull = 0xffffffffu;
constexpr int kPre = 2;            // tiles between a tile's L2 prefetch and its load

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int ST_B = 0, ST_C = 32768, ST_X = 65536, ST_BYTES = 81920;   // one ring stage
constexpr int OFF_WX = 2 * ST_BYTES;          // w X      (16 KB)
constexpr int OFF_SBF = OFF_WX + 16384;       // bf16 S   (16 KB)
constexpr int OFF_MISC = OFF_SBF + 16384;

// TMEM columns (512 allocated)
constexpr uint32_t TM_G = 0;        // G / P, two buffers of 128 columns
constexpr uint32_t TM_YX = 256;     // Y_inter, two buffers of 64
constexpr uint32_t TM_SL = 384;     // S_loc
constexpr uint32_t TM_YI = 448;     // Y_intra

struct Misc {
    uint64_t full_bc[2], full_x[2], empty_bc[2], empty_x[2], rot[2], g[2];
    uint64_t sl, sbf, p, yd, drain;
    uint64_t ho_w, ho_r, spare;     // hand-off: rows written, flag seen (once per launch each)
    uint64_t tf[3];                 // per-tile tables of buffer k % 3 consumed by the epilogue
    uint32_t tmem_base;
    int abort_flag;
    int drain_flag;
    int ho_ok;
    int pad[12];
    float2 qs[2][kNE][32];          // rotation warps: phase sums of each token group, by tile parity
    float2 phf[kTabs][32];          // phase of pairs (2l, 2l+1) at a piece's last token
    float ts[kTabs][132];           // a2 (log2 cumulative decay) per token; [128] = a2 of the last
    float4 xch[4][32];              // epilogue warps: partner-row exchange of the state export
    float cg[2][2][32];             // rotation warps: gamma and c per token (R >= 4), by tile parity
    union alignas(16) {
        float msk[32 * 36];         // R >= 4: decay mask per (token, token)
        float cs[6][128];           // R < 4: mask factors per token (see the rotation warps)
    } u[kTabs];
};
constexpr int SMEM_BYTES = OFF_MISC + (int)sizeof(Misc) + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory over the per-CTA limit");

// ------------------------------------------------------------------ work --
struct WsArgs {
    int mode;          // 0: ranges with hand-off (McNaughton), 1: one segment per CTA
    int nt;            // tiles per chain
    int M;             // tiles per CTA range (mode 0)
    int total;         // tiles of all chains (mode 0)
    int call_id;       // this call's flag value (never 0)
    float* ho_state;   // [slots][N][P] hand-off states (mode 0)
    int* ho_flag;      // [slots]
};

struct Piece {
    int unit, j0, j1;
    int init;          // 0 carry, 1 hand-off wait (slot_in), 2 segment input state
    int fin;           // 0 none, 1 final carry, 2 hand-off write (slot_out)
    int slot_in, slot_out, seg;
};

// The idx-th piece of this CTA in processing order; false past the last.
__device__ __forceinline__ bool piece_at(const WsArgs& a, const ScanParams& q, int idx, Piece& pc) {
    const int nt = a.nt;
    if (a.mode == 1) {
        if (idx > 0) return false;
        const int c = blockIdx.x;
        pc.seg = c % q.nseg;
        pc.unit = c / q.nseg;
        pc.j0 = pc.seg * q.cps;
        pc.j1 = min(nt, (pc.seg + 1) * q.cps);
        pc.init = pc.seg == 0 ? 0 : 2;
        pc.fin = pc.seg == q.nseg - 1 ? 1 : 0;
        pc.slot_in = pc.slot_out = 0;
        return pc.j0 < pc.j1;
    }
    const int i = blockIdx.x;
    const int s = i * a.M;
    const int e = min(s + a.M, a.total);
    if (s >= e) return false;
    const bool has_head = (e % nt) != 0;            // range ends inside a chain
    const bool has_tail = (s % nt) != 0;            // range starts inside a chain
    const int w0 = (s + nt - 1) / nt, w1 = e / nt;  // whole chains [w0, w1)
    pc.seg = 0;
    if (has_head) {
        if (idx == 0) {
            pc.unit = e / nt; pc.j0 = 0; pc.j1 = e % nt;
            pc.init = 0; pc.fin = 2; pc.slot_in = 0; pc.slot_out = i + 1;
            return true;
        }
        --idx;
    }
    if (idx < w1 - w0) {
        pc.unit = w0 + idx; pc.j0 = 0; pc.j1 = nt;
        pc.init = 0; pc.fin = 1; pc.slot_in = pc.slot_out = 0;
        return true;
    }
    idx -= w1 - w0;
    if (has_tail && idx == 0) {
        pc.unit = s / nt; pc.j0 = s % nt; pc.j1 = nt;
        pc.init = 1; pc.fin = 1; pc.slot_in = i; pc.slot_out = 0;
        return true;
    }
    return false;
}

// Walks this CTA's tiles in processing order (every role walks the same list).
struct Cursor {
    Piece pc;
    int pidx, j;
    int b, h, g;       // batch, head and group of the piece's sequence
    bool ok;
    __device__ __forceinline__ void set_unit(const ScanParams& q) {
        b = pc.unit / q.nheads;
        h = pc.unit - b * q.nheads;
        g = h / (q.nheads / q.ngroups);
    }
    __device__ __forceinline__ void start(const WsArgs& a, const ScanParams& q) {
        pidx = 0;
        ok = piece_at(a, q, 0, pc);
        j = ok ? pc.j0 : 0;
        if (ok) set_unit(q);
    }
    __device__ __forceinline__ void next(const WsArgs& a, const ScanParams& q) {
        if (++j < pc.j1) return;
        ok = piece_at(a, q, ++pidx, pc);
        j = ok ? pc.j0 : 0;
        if (ok) set_unit(q);
    }
};

// ------------------------------------------------------- small helpers --
__device__ __forceinline__ bool bwait(uint64_t* b, uint32_t parity, Misc* m, int* status, int where) {
    return mbar_wait_flag(b, parity, &m->abort_flag, status, where);
}
// OR of `cond` over the rotation warps (named barrier `id` with a reduction)
__device__ __forceinline__ int group_any(int id, int cond) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(cond), "r"(id), "n"(kRWT)
        : "memory");
    return r;
}

// rotation of one bf16 pair (x, y) -> (c x + s y, c y - s x) in float32,
// rounded once to bf16
__device__ __forceinline__ uint32_t rot_f32(uint32_t v, float c, float s) {
    const float x = __uint_as_float(v << 16), y = __uint_as_float(v & 0xffff0000u);
    const float2 r = __ffma2_rn(make_float2(c, c), make_float2(x, y), __fmul2_rn(make_float2(s, -s), make_float2(y, x)));
    return pack_bf16x2(r.x, r.y);
}
// a 16-byte chunk of 8 bf16 times a float32 weight, rounded once
__device__ __forceinline__ uint4 scale_chunk_f32(uint4 v, float w) {
    uint32_t* e = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(e[i] << 16), hi = __uint_as_float(e[i] & 0xffff0000u);
        e[i] = pack_bf16x2(lo * w, hi * w);
    }
    return v;
}

// ---------------------------------------------------------------- kernel --
template <int R>
__global__ void __launch_bounds__(kThreads, 1)
    scan_ws_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmX, ScanParams q, WsArgs wa, int* status) {
    constexpr int T = kRows / R;       // tokens per tile
    constexpr int NT = (T + 31) / 32;  // token slices per lane
    constexpr int TE = T / kNE;        // tokens per rotation warp
    constexpr float kLog2e = 1.4426950408889634f;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
    Misc* m = reinterpret_cast<Misc*>(smem + OFF_MISC);
    const uint32_t sbase = su32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = q.seqlen, H = q.nheads, G = q.ngroups;
    // the shared-memory map inside the launch's dynamic shared memory
    // (uniform over the CTA, before any barrier)
    if (!M3_SPAN(1, smem - smem_raw, OFF_MISC + (int)sizeof(Misc), dyn_smem_bytes())) return;
    const long long ext_ho = (long long)gridDim.x;                // hand-off slots (debug checks)
    const long long ext_ws = (long long)q.batch * H * q.nseg;     // segment inputs (debug checks)
    (void)ext_ho; (void)ext_ws;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m->full_bc[s], 1);
            mbar_init(&m->full_x[s], 1);
            mbar_init(&m->empty_bc[s], 1);
            mbar_init(&m->empty_x[s], 1);
            mbar_init(&m->rot[s], kRWT);
            mbar_init(&m->g[s], 1);
        }
        mbar_init(&m->sl, 1);
        mbar_init(&m->sbf, kEWT);
        mbar_init(&m->p, kEWT);
        mbar_init(&m->yd, 1);
        mbar_init(&m->drain, 1);
        mbar_init(&m->ho_w, kEWT);
        mbar_init(&m->ho_r, 1);
        for (int z = 0; z < kTabs; ++z) mbar_init(&m->tf[z], kEWT);
        m->abort_flag = 0;
        m->drain_flag = 0;
        m->ho_ok = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&m->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;

    if (warp == 0 || warp == 2) {
        // ----------------------------------------------------- TMA producers
        // warp 0 loads B and C, warp 2 loads X, each into its half of the
        // two-stage ring as soon as that half is free (B, C after tile k - 2's
        // G; X after its Y_intra), so neither waits behind the other
        if (lane == 0) {
            const bool bc = warp == 0;
            Cursor cu;
            cu.start(wa, q);
            int k = 0;
            int issued_last = -1;
            for (; cu.ok; cu.next(wa, q), ++k) {
                const int s = k & 1;
                const int t0 = cu.j * T;
                const uint32_t st = sbase + s * ST_BYTES;
                if (k >= 2 && !bwait(bc ? &m->empty_bc[s] : &m->empty_x[s], ((k - 2) >> 1) & 1, m, status, bc ? 1 : 5))
                    break;
                // tensor coordinates (the copy engine bounds them itself: only noted)
                M3_NOTE(2, t0, L);
                M3_NOTE(3, cu.b, q.batch);
                M3_NOTE(4, bc ? cu.g : cu.h, bc ? G : H);
                if (bc) {
                    uint64_t* fb = &m->full_bc[s];
                    mbar_expect_tx(fb, 65536u);
                    tma_load_5d(st + ST_B, &tmB, fb, 0, 0, cu.g, t0, cu.b);
                    tma_load_5d(st + ST_B + 16384, &tmB, fb, 64, 0, cu.g, t0, cu.b);
                    tma_load_5d(st + ST_C, &tmC, fb, 0, 0, cu.g, t0, cu.b);
                    tma_load_5d(st + ST_C + 16384, &tmC, fb, 64, 0, cu.g, t0, cu.b);
                } else {
                    uint64_t* fx = &m->full_x[s];
                    mbar_expect_tx(fx, 16384u);
                    tma_load_5d(st + ST_X, &tmX, fx, 0, 0, cu.h, t0, cu.b);
                }
                issued_last = k;
                // the tile kPre ahead into L2, so that DRAM has this SM's next
                // tiles in flight while the ring holds only two
                Cursor cp = cu;
                for (int z = 0; z < kPre && cp.ok; ++z) cp.next(wa, q);
                if (cp.ok) {
                    const int tp = cp.j * T;
                    if (bc) {
                        tma_prefetch_5d(&tmB, 0, 0, cp.g, tp, cp.b);
                        tma_prefetch_5d(&tmB, 64, 0, cp.g, tp, cp.b);
                        tma_prefetch_5d(&tmC, 0, 0, cp.g, tp, cp.b);
                        tma_prefetch_5d(&tmC, 64, 0, cp.g, tp, cp.b);
                    } else {
                        tma_prefetch_5d(&tmX, 0, 0, cp.h, tp, cp.b);
                    }
                }
            }
            // let every issued load land before the CTA can exit (bounded);
            // loads the rotation warps consumed complete immediately here
            for (int kk = max(0, issued_last - 1); kk <= issued_last; ++kk)
                mbar_wait_flag(bc ? &m->full_bc[kk & 1] : &m->full_x[kk & 1], (kk >> 1) & 1, &m->drain_flag, nullptr,
                               0);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            Cursor cu;
            cu.start(wa, q);
            constexpr uint32_t idG = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idY = idesc_bf16(128, 64, 0, 1);
            constexpr uint32_t idS = idesc_bf16(128, 64, 1, 1);
            constexpr uint32_t idI = idesc_bf16(128, 64, 0, 1);
            // Y_intra of tile k - 1 (P from TMEM) is issued after tile k's
            // first products, so the tensor pipe starts tile k while the
            // epilogue warps still compute P(k - 1)
            auto y_intra = [&](int kp) -> bool {
                const int sp = kp & 1;
                if (!bwait(&m->p, kp & 1, m, status, 4)) return false;
                tc_fence_after();
                const uint32_t sX = sbase + sp * ST_BYTES + ST_X;
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tmem + TM_YI, tmem + TM_G + 128 * sp + 8 * kk, sdesc(sX + kk * 2048, 8192, 1024), idI,
                            kk > 0);
                umma_commit(&m->yd);
                umma_commit(&m->empty_x[sp]);
                return true;
            };
            int k = 0;
            bool live = true;
            for (; cu.ok; cu.next(wa, q), ++k) {
                const int s = k & 1;
                if (!bwait(&m->rot[s], (k >> 1) & 1, m, status, 2)) { live = false; break; }
                if (!bwait(&m->sbf, k & 1, m, status, 3)) { live = false; break; }
                tc_fence_after();
                const uint32_t sB = sbase + s * ST_BYTES + ST_B, sC = sbase + s * ST_BYTES + ST_C;
                // Y_inter = C~ S_bf (K = n), S_loc = B~^T (w X) (K = tile rows)
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t offa = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma(tmem + TM_YX + 64 * s, sdesc(sC + offa, 16, 1024),
                         sdesc(sbase + OFF_SBF + kk * 2048, 8192, 1024), idY, kk > 0);
                }
                for (int kk = 0; kk < 8; ++kk)
                    umma(tmem + TM_SL, sdesc(sB + kk * 2048, 16384, 1024),
                         sdesc(sbase + OFF_WX + kk * 2048, 8192, 1024), idS, kk > 0);
                umma_commit(&m->sl);
                // G = C~ B~^T (K = n, both K-major)
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma(tmem + TM_G + 128 * s, sdesc(sC + off, 16, 1024), sdesc(sB + off, 16, 1024), idG, kk > 0);
                }
                umma_commit(&m->g[s]);
                umma_commit(&m->empty_bc[s]);         // B~ and C~ read for the last time
                if (k > 0 && !y_intra(k - 1)) { live = false; break; }
            }
            if (live && k > 0) y_intra(k - 1);
            // every MMA issued is complete before TMEM is freed
            umma_commit(&m->drain);
            mbar_wait_flag(&m->drain, 0, &m->drain_flag, nullptr, 0);
        }
        __syncwarp();
    } else if (warp < kEW0) {
        // warp 3 has no role; it waits at the final barrier
    } else if (warp < kRW0) {
        // ---------------------------------------------------------- epilogue
        const int e = tid - 32 * kEW0;                 // 0..127
        const int qd = warp & 3;                        // TMEM lane quarter
        const int row = qd * 32 + lane;                 // tile row / state row
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        const int tr = row / R;                         // token of this tile row
        const int rr = row % R;
        __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(q.y);
        float S[kP];
        Cursor cu;
        cu.start(wa, q);
        int k = 0;
        int cur_piece = -1;
        // y = Y_intra + e^{a_t} Y_inter of tile kp (thread = tile row (tr, rr))
        int pend_b = 0, pend_h = 0, pend_t0 = 0, pend_qc = 0;
        float pend_ea = 0.f;
        auto emit_prev = [&](int kp) -> bool {
            const bool yd_ok = bwait(&m->yd, kp & 1, m, status, 13);
            if (__any_sync(kFull, !yd_ok)) return false;
            tc_fence_after();
            const float2 ea2 = make_float2(pend_ea, pend_ea);
            __nv_bfloat16* yrow = yg + ((((size_t)pend_b * L + pend_t0 + tr) * H + pend_h) * R + rr) * kP;
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                float yi[16], yx[16];
                tmem_ld16x2(tl + TM_YI + 16 * hh, tl + TM_YX + 64 * (kp & 1) + 16 * hh, yi, yx);
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const float2 o2 = __ffma2_rn(ea2, make_float2(yx[j], yx[j + 1]), make_float2(yi[j], yi[j + 1]));
                    yi[j] = o2.x;
                    yi[j + 1] = o2.y;
                }
                if (tr < pend_qc &&
                    M3_SPAN(10, ((((size_t)pend_b * L + pend_t0 + tr) * H + pend_h) * R + rr) * kP + 16 * hh, 16, ext_x(q))) {
                    uint4* dst = reinterpret_cast<uint4*>(yrow + 16 * hh);
                    dst[0] = pack_chunk(yi);
                    dst[1] = pack_chunk(yi + 8);
                }
            }
            tc_fence_before();
            return true;
        };
        while (cu.ok) {
            const Piece pc = cu.pc;
            const int b = cu.b, h = cu.h;
            const size_t bh = (size_t)b * H + h;
            if (cur_piece != cu.pidx) {
                // ---- the piece's incoming state (thread = state row n)
                cur_piece = cu.pidx;
                const int n = row;
                if (pc.init == 1) {
                    // hand-off from the CTA that processed this chain's head.
                    // The first epilogue warp polls the flag as a whole (lane 0
                    // loads it and the warp decides together, so no lane spins
                    // apart from its warp), clears it for the next call (the
                    // state itself stays until the next call overwrites it) and
                    // releases the other three warps through an mbarrier.
                    if (e < 32) {
                        int ok = 1;
                        const uint64_t t0w = globaltimer_ns();
                        while (true) {
                            int seen = 0, stop = 0;
                            if (lane == 0) {
                                seen = M3_IN(11, pc.slot_in, ext_ho) && ld_acquire_gpu(wa.ho_flag + pc.slot_in) == wa.call_id;
                                stop = !seen && (*(volatile int*)&m->abort_flag || globaltimer_ns() - t0w > kWaitNs);
                            }
                            seen = __shfl_sync(kFull, seen, 0);
                            stop = __shfl_sync(kFull, stop, 0);
                            if (seen) break;
                            if (stop) { ok = 0; break; }
                        }
                        if (lane == 0) {
                            if (ok) {
                                wa.ho_flag[pc.slot_in] = 0;
                            } else {
                                m->abort_flag = 1;
                                if (atomicCAS(status, 0, (int)M3_ERR_DEVICE_TIMEOUT) == 0) status[1] = 20;
                            }
                            *(volatile int*)&m->ho_ok = ok;
                            mbar_arrive(&m->ho_r);
                        }
                        __syncwarp();
                        if (!ok) break;
                    } else {
                        const bool got = bwait(&m->ho_r, 0, m, status, 21);
                        if (__any_sync(kFull, !got || !*(volatile int*)&m->ho_ok)) break;
                    }
                    const float4* src = reinterpret_cast<const float4*>(wa.ho_state + ((size_t)pc.slot_in * kN + n) * kP);
                    const bool okh = M3_SPAN(12, ((size_t)pc.slot_in * kN + n) * kP, kP, ext_ho * kN * kP);
#pragma unroll
                    for (int c = 0; c < kP / 4; ++c) {
                        const float4 v = okh ? __ldcg(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                        S[4 * c] = v.x; S[4 * c + 1] = v.y; S[4 * c + 2] = v.z; S[4 * c + 3] = v.w;
                    }
                } else if (pc.init == 2) {
                    const size_t bhs = bh * q.nseg + pc.seg;
                    const float4* src = reinterpret_cast<const float4*>(q.ws_sin + (bhs * kN + n) * kP);
                    const bool oks = M3_SPAN(13, (bhs * kN + n) * kP, kP, ext_ws * kN * kP);
#pragma unroll
                    for (int c = 0; c < kP / 4; ++c) {
                        const float4 v = oks ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
                        S[4 * c] = v.x; S[4 * c + 1] = v.y; S[4 * c + 2] = v.z; S[4 * c + 3] = v.w;
                    }
                } else {
                    const bool oki = !q.init_h || M3_SPAN(14, (bh * kN + n) * kP, kP, ext_h(q));
#pragma unroll
                    for (int p = 0; p < kP; ++p) S[p] = (q.init_h && oki) ? q.init_h[(bh * kN + n) * kP + p] : 0.f;
                    if (q.init_pB && q.init_pX) {
                        const bool ok0 = M3_IN(15, (size_t)b * L * H + h, ext_tok(q));
                        const float w0 = ok0 ? (1.f - q.lam[(size_t)b * L * H + h]) * q.dt[(size_t)b * L * H + h] : 0.f;
                        const __nv_bfloat16* pB = static_cast<const __nv_bfloat16*>(q.init_pB) + bh * R * kN;
                        const __nv_bfloat16* pX = static_cast<const __nv_bfloat16*>(q.init_pX) + bh * R * kP;
                        for (int r = 0; r < R; ++r) {
                            if (!M3_IN(16, bh * R * kN + r * kN + n, ext_pB(q)) ||
                                !M3_SPAN(17, bh * R * kP + r * kP, kP, ext_pX(q)))
                                continue;
                            const float bv = w0 * __bfloat162float(pB[r * kN + n]);
#pragma unroll
                            for (int p = 0; p < kP; ++p) S[p] = fmaf(bv, __bfloat162float(pX[r * kP + p]), S[p]);
                        }
                    }
                }
#pragma unroll
                for (int c = 0; c < kP / 8; ++c)
                    if (M3_SPAN(18, sw128(n, c), 16, 16384))
                        *reinterpret_cast<uint4*>(smem + OFF_SBF + sw128(n, c)) = pack_chunk(S + 8 * c);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&m->sbf);
            }
            // ---- tile k of the piece
            const int s = k & 1, tb = k % kTabs;
            const int t0 = cu.j * T, qc = min(T, L - t0);
            const bool rot_ok = bwait(&m->rot[s], (k >> 1) & 1, m, status, 10);
            if (__any_sync(kFull, !rot_ok)) break;       // the warp leaves together
            const float a2_tr = m->ts[tb][tr];
            const float a2_last = m->ts[tb][128];
            // state: S = e^{a_last} S + S_loc
            const bool sl_ok = bwait(&m->sl, k & 1, m, status, 11);
            if (__any_sync(kFull, !sl_ok)) break;       // the warp leaves together
            tc_fence_after();
            {
                const float dec = exp2f(a2_last);
                const float2 dec2 = make_float2(dec, dec);
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
                    float va[16];
                    tmem_ld16(tl + TM_SL + 16 * hh, va);
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        const float2 s2 = __ffma2_rn(dec2, make_float2(S[16 * hh + j], S[16 * hh + j + 1]),
                                                     make_float2(va[j], va[j + 1]));
                        S[16 * hh + j] = s2.x;
                        S[16 * hh + j + 1] = s2.y;
                    }
                }
            }
            const bool last_of_piece = cu.j == pc.j1 - 1;
            if (!last_of_piece) {
#pragma unroll
                for (int c = 0; c < kP / 8; ++c)
                    if (M3_SPAN(19, sw128(row, c), 16, 16384))
                        *reinterpret_cast<uint4*>(smem + OFF_SBF + sw128(row, c)) = pack_chunk(S + 8 * c);
            } else if (pc.fin != 0) {
                // ---- the piece's outgoing state: h = R(Phi) S (original frame)
                const int n = row;
                const float2 cv2 = m->phf[tb][n >> 2];
                const float phn = ((n >> 1) & 1) ? cv2.y : cv2.x;
                float sv, cv;
                __sincosf(phn, &sv, &cv);         // phn is reduced to [-pi, pi]: error ~4e-7
                float* dst = pc.fin == 2 ? wa.ho_state + ((size_t)pc.slot_out * kN + n) * kP
                                         : (q.fin_h ? q.fin_h + (bh * kN + n) * kP : nullptr);
                // (the partner exchange below is warp-wide: a failed check
                // only drops this thread's stores)
                const bool okd = pc.fin == 2 ? M3_SPAN(20, ((size_t)pc.slot_out * kN + n) * kP, kP, ext_ho * kN * kP)
                                             : M3_SPAN(21, (bh * kN + n) * kP, kP, ext_h(q));
                (void)okd;
                if (dst) {
                    // rows n and n ^ 1 (one rotary pair) sit in adjacent lanes;
                    // four columns at a time go through a shared-memory slot
                    float4* xs = &m->xch[qd][0];
#pragma unroll
                    for (int p = 0; p < kP; p += 4) {
                        xs[lane] = make_float4(S[p], S[p + 1], S[p + 2], S[p + 3]);
                        __syncwarp();
                        const float4 ot = xs[lane ^ 1];
                        __syncwarp();
                        const float o4[4] = {ot.x, ot.y, ot.z, ot.w};
                        float o[4];
#pragma unroll
                        for (int z = 0; z < 4; ++z)
                            o[z] = (n & 1) ? (sv * o4[z] + cv * S[p + z]) : (cv * S[p + z] - sv * o4[z]);
                        if (okd) *reinterpret_cast<float4*>(dst + p) = make_float4(o[0], o[1], o[2], o[3]);
                    }
                }
                if (pc.fin == 2) {
                    // publish: every thread fences its row; the first epilogue
                    // warp waits (as a whole, bounded) for all of them and its
                    // lane 0 raises the flag
                    __threadfence();
                    mbar_arrive(&m->ho_w);
                    if (e < 32) {
                        const bool all = bwait(&m->ho_w, 0, m, status, 23);
                        __syncwarp();
                        if (all && lane == 0 && M3_IN(22, pc.slot_out, ext_ho))
                            st_release_gpu(wa.ho_flag + pc.slot_out, wa.call_id);
                        __syncwarp();
                    }
                } else if (L > 0) {
                    const int g = h / (H / G);
                    if (q.fin_pB) {
                        const __nv_bfloat16* sB = static_cast<const __nv_bfloat16*>(q.B) + (((size_t)b * L + L - 1) * G + g) * R * kN;
                        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(q.fin_pB) + bh * R * kN;
                        for (int z = e; z < R * kN; z += kEWT)
                            if (M3_IN(23, (((size_t)b * L + L - 1) * G + g) * R * kN + z, ext_bc(q)) &&
                                M3_IN(24, bh * R * kN + z, ext_pB(q)))
                                o[z] = sB[z];
                    }
                    if (q.fin_pX) {
                        const __nv_bfloat16* sX = static_cast<const __nv_bfloat16*>(q.x) + (((size_t)b * L + L - 1) * H + h) * R * kP;
                        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(q.fin_pX) + bh * R * kP;
                        for (int z = e; z < R * kP; z += kEWT)
                            if (M3_IN(25, (((size_t)b * L + L - 1) * H + h) * R * kP + z, ext_x(q)) &&
                                M3_IN(26, bh * R * kP + z, ext_pX(q)))
                                o[z] = sX[z];
                    }
                }
            }
            // ---- the previous tile's y, now that its Y_intra is done
            if (k > 0 && !emit_prev(k - 1)) break;
            if (!last_of_piece) {
                // S_bf for the next tile (the MMA then overwrites this tile's
                // Y_inter buffer's twin, which the emit above has read)
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&m->sbf);
            }
            // ---- P = mask o G into TMEM (bf16, packed in place over G)
            const bool g_ok = bwait(&m->g[s], (k >> 1) & 1, m, status, 12);
            if (__any_sync(kFull, !g_ok)) break;       // the warp leaves together
            tc_fence_after();
            {
                const uint32_t gcol = tl + TM_G + 128 * s;
                const auto& U = m->u[tb];
#pragma unroll 1
                for (int cg = 0; cg < 8; ++cg) {
                    const int col0 = cg * 16;
                    float v[16];
                    tmem_ld16(gcol + col0, v);
                    if (R >= 4) {
                        constexpr int LD = T + 4;
                        const float* mrow = U.msk + tr * LD + col0 / R;
                        float mk[16 / R];
                        if (!M3_SPAN(27, tr * LD + col0 / R, 16 / R, 32 * 36)) {
#pragma unroll
                            for (int i = 0; i < 16 / R; ++i) mk[i] = 0.f;
                        } else if (R == 4) {
                            const float4 f = *reinterpret_cast<const float4*>(mrow);
                            mk[0] = f.x; mk[1] = f.y; mk[2 % (16 / R)] = f.z; mk[3 % (16 / R)] = f.w;
                        } else {
                            const float2 f = *reinterpret_cast<const float2*>(mrow);
                            mk[0] = f.x; mk[1] = f.y;
                        }
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            const float2 g2 = __fmul2_rn(make_float2(mk[j / R], mk[(j + 1) / R]), make_float2(v[j], v[j + 1]));
                            v[j] = g2.x;
                            v[j + 1] = g2.y;
                        }
                    } else {
                        constexpr int GT = 16 / R;            // tokens per 16-column block
                        const int u0 = col0 / R;
                        // (u0 + 16 / R <= T <= 128 keeps the cs rows below inside their 128 floats)
                        const bool okc = M3_SPAN(28, u0, GT, 128);
                        const float aref = okc ? U.cs[2][u0 / GT] : 0.f;
                        if (u0 > tr || !okc) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) v[j] = 0.f;
                        } else if (aref != __int_as_float(0x7f800000)) {
                            const float rowf = exp2f(a2_tr - aref);
#pragma unroll
                            for (int i4 = 0; i4 < GT / 4; ++i4) {
                                const float4 fc = reinterpret_cast<const float4*>(U.cs[0] + u0)[i4];
                                const float4 fg = reinterpret_cast<const float4*>(U.cs[1] + u0)[i4];
                                const float mc[4] = {fc.x, fc.y, fc.z, fc.w}, mg[4] = {fg.x, fg.y, fg.z, fg.w};
#pragma unroll
                                for (int z = 0; z < 4; ++z) {
                                    const int uu = u0 + 4 * i4 + z;
                                    const float mkv = rowf * ((uu < tr) ? mc[z] : (uu == tr ? mg[z] : 0.f));
#pragma unroll
                                    for (int r2 = 0; r2 < R; ++r2) v[(4 * i4 + z) * R + r2] *= mkv;
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; j += R) {
                                const int uu = u0 + j / R;
                                const float au = U.cs[3][uu], gu = U.cs[4][uu], cu2 = U.cs[5][uu];
                                const float mkv = (uu <= tr) ? exp2f(a2_tr - au) * (uu == tr ? gu : cu2) : 0.f;
#pragma unroll
                                for (int r2 = 0; r2 < R; ++r2) v[j + r2] *= mkv;
                            }
                        }
                    }
                    uint32_t pk[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                    tmem_st8(gcol + 8 * cg, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&m->p);
                mbar_arrive(&m->tf[tb]);          // ts, u and phf of this tile are no longer read
            }
            // this tile's y waits for its Y_intra, which follows the next
            // tile's first products
            pend_b = b; pend_h = h; pend_t0 = t0; pend_qc = qc; pend_ea = exp2f(a2_tr);
            cu.next(wa, q);
            ++k;
        }
        if (k > 0) emit_prev(k - 1);
    } else {
        // ---------------------------------------------------------- rotation
        const int r = tid - 32 * kRW0;         // 0..255
        const int qe = warp - kRW0;            // token group of the phase / rotation pass
        const int xr = r & 127;                // tile row of the w X pass (two threads per row)
        const int xc0 = (r >> 7) * 4;          // its four 16-byte chunks
        const int g0 = qe * TE;
        const int gsl = g0 >> 5, gln = g0 & 31;
        const int rtk = xr / R;                // token of tile row xr
        const int rsl = rtk >> 5, rln = rtk & 31;
        Cursor cu;
        cu.start(wa, q);
        // inputs of the next tile, loaded a tile ahead of their use: dt,
        // lambda per token (lane l holds tokens l + 32 j), the token after the
        // tile, A of its head, and theta of this warp's tokens for pairs
        // (2 lane, 2 lane + 1); every load uses a clamped (valid) address
        float dt_n[NT], lam_n[NT], dx_n = 0.f, lx_n = 1.f, a_n = 0.f;
        float2 th_n[TE];
        auto load_tok = [&](const Cursor& c) {
            const int b = c.b, h = c.h;
            const int t0n = c.j * T, qcn = min(T, L - t0n);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const int t = min(lane + 32 * j, qcn - 1);
                const size_t o = ((size_t)b * L + t0n + t) * H + h;
                const bool ok = M3_IN(30, o, ext_tok(q));
                dt_n[j] = ok ? __ldg(q.dt + o) : 0.f;
                lam_n[j] = ok ? __ldg(q.lam + o) : 1.f;
            }
            const int tn = min(t0n + qcn, L - 1);
            const size_t o = ((size_t)b * L + tn) * H + h;
            const bool ok = M3_IN(31, o, ext_tok(q));
            dx_n = ok ? __ldg(q.dt + o) : 0.f;
            lx_n = ok ? __ldg(q.lam + o) : 1.f;
            a_n = M3_IN(32, h, H) ? __ldg(q.A + h) : 0.f;
        };
        // theta row of token kk of this warp's group in tile c (pairs 2 lane, 2 lane + 1)
        auto theta_row = [&](const Cursor& c, int& qcn) -> const float2* {
            const int b = c.b, g = c.g;
            const int t0n = c.j * T;
            qcn = min(T, L - t0n);
            return reinterpret_cast<const float2*>(q.theta + (((size_t)b * L + t0n) * G + g) * (kN / 2)) + lane;
        };
        const size_t th_tok = (size_t)G * (kN / 4);     // float2 stride between tokens
        // L2 prefetch of a tile's theta rows (256 B per token, two lines)
        auto prefetch_theta = [&](const Cursor& c) {
            const int b = c.b, g = c.g;
            const int t0n = c.j * T, qcn = min(T, L - t0n);
            for (int z = r; z < 2 * qcn; z += kRWT)
                if (M3_IN(33, (((size_t)b * L + t0n + (z >> 1)) * G + g) * (kN / 2) + (z & 1) * 32, ext_theta(q)))
                    prefetch_l2(q.theta + (((size_t)b * L + t0n + (z >> 1)) * G + g) * (kN / 2) + (z & 1) * 32);
        };
        if (cu.ok) {
            load_tok(cu);
            int qc0;
            const float2* tp = theta_row(cu, qc0);
#pragma unroll
            for (int kk = 0; kk < TE; ++kk)
                th_n[kk] = M3_SPAN(34, (((size_t)cu.b * L + cu.j * T) * G + cu.g) * (kN / 2) + 2 * lane +
                                           (size_t)min(g0 + kk, qc0 - 1) * 2 * th_tok, 2, ext_theta(q))
                               ? __ldg(tp + (size_t)min(g0 + kk, qc0 - 1) * th_tok) : make_float2(0.f, 0.f);
            Cursor c1 = cu;
            c1.next(wa, q);
            if (c1.ok) prefetch_theta(c1);
        }
        float2 carry = make_float2(0.f, 0.f);
        int cur_piece = -1;
        for (int k = 0; cu.ok; ++k) {
            const Piece pc = cu.pc;
            if (cur_piece != cu.pidx) {
                cur_piece = cu.pidx;
                carry = make_float2(0.f, 0.f);       // every piece has its own rotated frame
            }
            const int s = k & 1, tb = k % kTabs;
            const int t0 = cu.j * T, qc = min(T, L - t0);
            const float A2 = a_n * kLog2e;
            // this tile's inputs (tokens past the tile count as dt = 0, lambda = 1)
            float dtv[NT], lmv[NT];
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const bool in = lane + 32 * j < qc;
                dtv[j] = in ? dt_n[j] : 0.f;
                lmv[j] = in ? lam_n[j] : 1.f;
            }
            const bool nx_in = t0 + qc < L;
            const float dx = nx_in ? dx_n : 0.f, lx = nx_in ? lx_n : 1.f;
#pragma unroll
            for (int kk = 0; kk < TE; ++kk)
                if (g0 + kk >= qc) th_n[kk] = make_float2(0.f, 0.f);
            // coefficients (log2 units): a2 = inclusive scan of dt A, gamma =
            // lambda dt, c = gamma + (1 - lambda') dt' (' = the next token;
            // past the tile: the token after it, zero past the sequence)
            float a2v[NT], gmv[NT], cfv[NT];
            float a2_last;
            {
                float run = 0.f;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    float v = dtv[j] * A2;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const float u = __shfl_up_sync(kFull, v, o);
                        if (lane >= o) v += u;
                    }
                    a2v[j] = v + run;
                    run = __shfl_sync(kFull, a2v[j], 31);
                }
                a2_last = run;
                float up[NT];
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    gmv[j] = lmv[j] * dtv[j];
                    up[j] = (1.f - lmv[j]) * dtv[j];
                }
                const float ux = (1.f - lx) * dx;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    float nx = __shfl_down_sync(kFull, up[j], 1);
                    if (j + 1 < NT) {
                        const float first = __shfl_sync(kFull, up[j + 1 < NT ? j + 1 : j], 0);
                        if (lane == 31) nx = first;
                    }
                    if (lane + 32 * j + 1 == T) nx = ux;
                    cfv[j] = gmv[j] + nx;
                }
            }
            // the next tile's dt / lambda, a tile ahead of their use; theta of
            // the tile after it into L2
            Cursor nx1 = cu;
            nx1.next(wa, q);
            if (nx1.ok) {
                load_tok(nx1);
                Cursor nx2 = nx1;
                nx2.next(wa, q);
                if (nx2.ok) prefetch_theta(nx2);
            }
            // per-tile tables for the epilogue warps, in buffer tb once the
            // epilogue has consumed tile k - 3's (a wait that expires sets the
            // abort flag; the group then leaves together at its barrier)
            if (k >= kTabs) bwait(&m->tf[tb], ((k - kTabs) / kTabs) & 1, m, status, 33);
            if (qe == 0) {
#pragma unroll
                for (int j = 0; j < NT; ++j)
                    if (lane + 32 * j < T) m->ts[tb][lane + 32 * j] = a2v[j];
                if (lane == 0) m->ts[tb][128] = a2_last;
            }
            if (R >= 4) {
                // gamma and c of every token for the mask table built after
                // the group barrier (a2 is in ts)
                if (qe == 0 && lane < T) {
                    m->cg[s][0][lane] = gmv[0];
                    m->cg[s][1][lane] = cfv[0];
                }
            } else if (qe == 0) {
                // the mask of a 16-column block (GT tokens) factors as
                // e^{a_t - a_ref} x e^{a_ref - a_u} (gamma_u or c_u), a_ref = a at
                // the block's first token, when the block's own decay is small
                // enough that the second factor cannot overflow; other blocks
                // get a_ref = +inf (element-wise path)
                constexpr int GT = 16 / R;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const int t = lane + 32 * j;
                    const float aref = __shfl_sync(kFull, a2v[j], lane & ~(GT - 1));
                    const float aend = __shfl_sync(kFull, a2v[j], lane | (GT - 1));
                    const bool okb = aref - aend <= 60.f;
                    const float colf = exp2f(aref - a2v[j]);
                    if (!M3_IN(36, t, 128)) continue;
                    m->u[tb].cs[0][t] = okb ? cfv[j] * colf : 0.f;
                    m->u[tb].cs[1][t] = okb ? gmv[j] * colf : 0.f;
                    if ((lane & (GT - 1)) == 0) m->u[tb].cs[2][t / GT] = okb ? aref : __int_as_float(0x7f800000);
                    m->u[tb].cs[3][t] = a2v[j];
                    m->u[tb].cs[4][t] = gmv[j];
                    m->u[tb].cs[5][t] = cfv[j];
                }
            }
            // phase pass 1: this group's increments of pairs (2 lane, 2 lane + 1)
            const float dsl = pick<NT>(dtv, gsl);
            {
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int kk = 0; kk < TE; ++kk) {
                    const float d = __shfl_sync(kFull, dsl, gln + kk);
                    acc.x = fmaf(d, th_n[kk].x, acc.x);
                    acc.y = fmaf(d, th_n[kk].y, acc.y);
                }
                m->qs[s][qe][lane] = acc;
            }
            // one barrier of the group per tile: publishes qs; all agree to stop
            if (group_any(2, *(volatile int*)&m->abort_flag)) break;
            if (R >= 4) {
                // decay mask per (token t, token u) of the tile, shared by the
                // R x R rank block: e^{a_t - a_u} (gamma_u if u == t, c_u if
                // u < t), 0 above; thread = (row t, a run of T*T/128 columns)
                constexpr int LD = T + 4;
                constexpr int PER = T * T / kRWT;         // 4 (R = 4) or 1 (R = 8)
                const int t = r / (T / PER), u0 = (r % (T / PER)) * PER;
                const float at = m->ts[tb][t];
#pragma unroll
                for (int z = 0; z < PER; ++z) {
                    const int u = u0 + z;
                    const float mv = exp2f(at - m->ts[tb][u]) * (u == t ? m->cg[s][0][u] : m->cg[s][1][u]);
                    if (M3_IN(35, t * LD + u, 32 * 36)) m->u[tb].msk[t * LD + u] = (u <= t) ? mv : 0.f;
                }
            }
            float2 ph = carry;
            {
                float2 tot = make_float2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < kNE; ++j) {
                    const float2 v = m->qs[s][j][lane];
                    if (j < qe) { ph.x += v.x; ph.y += v.y; }
                    tot.x += v.x;
                    tot.y += v.y;
                }
                carry = make_float2(wrap_pi_f(carry.x + tot.x), wrap_pi_f(carry.y + tot.y));
            }
            if (qe == 0 && cu.j == pc.j1 - 1) m->phf[tb][lane] = carry;
            // phase pass 2: rotate rows (t, r) of B and C in place, float32
            // arithmetic, every token's phase reduced to [-pi, pi] first
            // a wait that expires sets the abort flag and the group leaves
            // together at the next tile's barrier: no thread leaves alone
            bwait(&m->full_bc[s], (k >> 1) & 1, m, status, 30);
            {
                // the next tile's theta is loaded token by token as this tile's
                // is consumed (no extra registers); row loads of token kk + 1
                // are issued before the stores of token kk
                Cursor cn = cu;
                cn.next(wa, q);
                int qcn = 1;
                const float2* tpn = cn.ok ? theta_row(cn, qcn) : nullptr;
                uint8_t* st = smem + s * ST_BYTES;
                const uint32_t atom = (uint32_t)(lane >> 4) * 16384u;
                const int chunk = (lane & 15) >> 1;
                const uint32_t inb = (uint32_t)(lane & 1) * 8u;
                // tokens in batches of KB: every row load of a batch first,
                // then the phases, then every rotation and store, so a warp
                // keeps many independent loads and rotations in flight
                constexpr int KB = (8 / R) < TE ? (8 / R > 0 ? 8 / R : 1) : TE;   // 8 rows of B and C per batch
#pragma unroll
                for (int k0 = 0; k0 < TE; k0 += KB) {
                    uint2 vv[KB][2][R];
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                        for (int rk = 0; rk < R; ++rk) {
                            const uint32_t off = atom + sw128((g0 + k0 + kb) * R + rk, chunk) + inb;
                            const bool okr = M3_SPAN(37, off, 8, 32768);
                            vv[kb][0][rk] = okr ? *reinterpret_cast<const uint2*>(st + ST_B + off) : make_uint2(0u, 0u);
                            vv[kb][1][rk] = okr ? *reinterpret_cast<const uint2*>(st + ST_C + off) : make_uint2(0u, 0u);
                        }
                    float cs[KB][4];
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb) {
                        const int kk = k0 + kb;
                        const float d = __shfl_sync(kFull, dsl, gln + kk);
                        ph.x = fmaf(d, th_n[kk].x, ph.x);
                        ph.y = fmaf(d, th_n[kk].y, ph.y);
                        ph = make_float2(wrap_pi_f(ph.x), wrap_pi_f(ph.y));
                        if (tpn && M3_SPAN(38, (((size_t)cn.b * L + cn.j * T) * G + cn.g) * (kN / 2) + 2 * lane +
                                                   (size_t)min(g0 + kk, qcn - 1) * 2 * th_tok, 2, ext_theta(q)))
                            th_n[kk] = __ldg(tpn + (size_t)min(g0 + kk, qcn - 1) * th_tok);
                        __sincosf(ph.x, &cs[kb][0], &cs[kb][1]);
                        __sincosf(ph.y, &cs[kb][2], &cs[kb][3]);
                    }
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                        for (int rk = 0; rk < R; ++rk) {
                            const uint32_t off = atom + sw128((g0 + k0 + kb) * R + rk, chunk) + inb;
#pragma unroll
                            for (int mt = 0; mt < 2; ++mt) {
                                uint2 v = vv[kb][mt][rk];
                                v.x = rot_f32(v.x, cs[kb][1], cs[kb][0]);
                                v.y = rot_f32(v.y, cs[kb][3], cs[kb][2]);
                                if (M3_SPAN(39, off, 8, 32768))
                                    *reinterpret_cast<uint2*>(st + (mt ? ST_C : ST_B) + off) = v;
                            }
                        }
                }
            }
            // w X for the chunk-local state into its buffer, once the previous
            // tile's S_loc MMA has read it (thread = tile row r)
            if (k > 0) bwait(&m->sl, (k - 1) & 1, m, status, 31);
            bwait(&m->full_x[s], (k >> 1) & 1, m, status, 32);
            {
                const float a2_r = __shfl_sync(kFull, pick<NT>(a2v, rsl), rln);
                const float cf_r = __shfl_sync(kFull, pick<NT>(cfv, rsl), rln);
                const float wt = exp2f(a2_last - a2_r) * cf_r;
                const uint8_t* xs = smem + s * ST_BYTES + ST_X;
                uint4 xv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    xv[c] = M3_SPAN(40, sw128(xr, xc0 + c), 16, 16384) ? *reinterpret_cast<const uint4*>(xs + sw128(xr, xc0 + c))
                                                                      : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (M3_SPAN(41, sw128(xr, xc0 + c), 16, 16384))
                        *reinterpret_cast<uint4*>(smem + OFF_WX + sw128(xr, xc0 + c)) = scale_chunk_f32(xv[c], wt);
            }
            fence_async_smem();
            mbar_arrive(&m->rot[s]);
            cu.next(wa, q);
        }
    }

    // ---- teardown: every role has left its loop
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace wsk

// 5-D map over [b][t][grp][r][inner] with a box of (64 inner, R, 1, T, 1)
bool make_tile_map(CUtensorMap* map, const void* base, int inner, int R, int grp, int L, int batch, int T);

int ws_smem_bytes() { return wsk::SMEM_BYTES; }

template <int R>
static cudaError_t launch_ws_R(const ScanParams& q, const WsPlanArgs& pa, int* status, cudaStream_t st) {
    using namespace wsk;
    constexpr int T = kRows / R;
    CUtensorMap mB, mC, mX;
    if (!make_tile_map(&mB, q.B, kN, R, q.ngroups, q.seqlen, q.batch, T) ||
        !make_tile_map(&mC, q.C, kN, R, q.ngroups, q.seqlen, q.batch, T) ||
        !make_tile_map(&mX, q.x, kP, R, q.nheads, q.seqlen, q.batch, T))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(scan_ws_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    WsArgs wa;
    wa.mode = pa.mode;
    wa.nt = pa.nt;
    wa.M = pa.M;
    wa.total = pa.total;
    wa.call_id = pa.call_id;
    wa.ho_state = pa.ho_state;
    wa.ho_flag = pa.ho_flag;
    ScanParams qq = q;
    int* stp = status;
    void* args[] = {(void*)&mB, (void*)&mC, (void*)&mX, (void*)&qq, (void*)&wa, (void*)&stp};
    if (pa.mode == 0)
        return cudaLaunchCooperativeKernel((const void*)scan_ws_kernel<R>, dim3(pa.grid), dim3(kThreads), args,
                                           SMEM_BYTES, st);
    scan_ws_kernel<R><<<pa.grid, kThreads, SMEM_BYTES, st>>>(mB, mC, mX, qq, wa, stp);
    return cudaGetLastError();
}

cudaError_t launch_scan_ws(const m3_dims& d, const ScanParams& q, const WsPlanArgs& pa, int* status,
                           cudaStream_t st) {
    switch (d.rank) {
        case 1: return launch_ws_R<1>(q, pa, status, st);
        case 2: return launch_ws_R<2>(q, pa, status, st);
        case 4: return launch_ws_R<4>(q, pa, status, st);
        case 8: return launch_ws_R<8>(q, pa, status, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace m3

M3_BOUNDS_EXPORT(scan_ws)
