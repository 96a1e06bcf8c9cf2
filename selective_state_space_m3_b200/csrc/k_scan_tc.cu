// k_scan_tc.cu -- chunked prefill of the Mamba-3 SSM layer on the sm_100a
// tensor cores (tcgen05 + TMEM + TMA), bfloat16 io, N = 128, P = 64.
//
// Same chunked algebra as the SIMT path (k_scan_simt.cu, and the header of
// that file): with B and C rotated by their cumulative phase ("Mamba-3"
// summary, b-lab.team, section 2, Proposition 3) the recurrence inside a
// chunk is the two-band masked matrix of section 1, and the state is passed
// between chunks.  Here a chunk is one 128-row tile (T = 128 / R tokens x R
// ranks), the size of one UMMA M=128 operand; the result does not depend on
// the chunk length except through rounding.
//
// Per CTA: one (batch, head, segment); the CTA walks the segment's tiles.
// Threads: warp 0 -- one lane issues the TMA loads and the tcgen05.mma;
//          warps 1..8 -- 256 workers in two warpgroups; a worker warp reads
//          TMEM lanes 32*(warp%4) .. +31 (a warp can only reach its own lane
//          quarter), so each warpgroup covers all 128 rows and the two split
//          the columns of row-wise work.
// Per tile:
//   TMA     B, C (bf16, SWIZZLE_128B, K-major: rows (t,r), 2 atoms of 64 n)
//           and X (rows (t,r), 64 p) into shared memory; issued as soon as
//           the previous tile's MMAs have read those buffers (with segments,
//           the next tile is also prefetched into L2 at that point).
//   workers coefficient stage: dt/lambda -> a_t (warp scan, every warp keeps
//           all tokens in registers), gamma, c, w = e^{a_last-a}c, e^{a}, the
//           mask tables and each warp's phase increments (for R <= 2 made one
//           tile ahead, during the previous tile's MMA wait, from dt/lambda
//           that cp.async copied into shared memory a tile earlier); cumulative phase
//           per rotary pair (float, reduced to [-pi, pi] at the tile start and
//           between tiles); rotate B and C in place in bf16x2 arithmetic.  One
//           worker barrier per tile.
//   MMA 1   G = C~ B~^T (128x128, K=128)      -> TMEM cols [0,128)
//           Y_inter = C~ S_bf (128x64, K=128) -> TMEM cols [192,256)
//   workers w X -> the S_bf region (free after MMA 1); P = mask o G ->
//           bf16 over C~'s smem.
//   MMA 2   S_loc = B~^T (w X) (128x64, K=128) -> TMEM cols [128,192)
//           Y_intra = P X (128x64, K=128)      -> TMEM cols [0,64)
//   workers S = e^{a_last} S + S_loc (float32, registers, thread = state row);
//           S_bf = bf16(S) for the next tile; y = Y_intra + e^{a_t} Y_inter.
// Two CTAs share an SM (108.5 KB of shared memory for R >= 4, 111.9 KB for
// R < 4, 256 TMEM columns and at most 96 registers per thread each), so one
// CTA's loads and MMAs overlap the other's SIMT work.
//
// Every wait on an mbarrier is bounded (1 s); on expiry the kernel records
// M3_ERR_DEVICE_TIMEOUT in the workspace status word, finishes the tile with
// no further waiting and returns after freeing its TMEM.
#define M3_BOUNDS_FILE 1
#include "m3_bounds.cuh"
#include "m3_kernels.h"
#include "tc_ptx.cuh"

namespace m3 {
namespace tc {

constexpr int kRows = 128;
constexpr int kN = 128;
constexpr int kP = 64;
constexpr int kWG = 2;                 // worker warpgroups
constexpr int kWorkers = 128 * kWG;
constexpr int kThreads = 32 + kWorkers;
constexpr int kNE = kWorkers / 32;     // token groups of the phase / rotation pass (one per worker warp)
constexpr int kSC = kP / kWG;          // state / y columns per warpgroup

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int OFF_B = 0;          // 32 KB: B~ (two 16 KB atoms)
constexpr int OFF_C = 32768;      // 32 KB: C~, later P
constexpr int OFF_X = 65536;      // 16 KB: X
constexpr int OFF_S = 81920;      // 16 KB: S_bf (rows n, 64 p)
constexpr int OFF_MISC = 98304;
constexpr int MISC_BYTES = 12544;
// dynamic shared memory of a launch (+ alignment slack); R >= 4 leaves the
// second parity of the R < 4 tables out, which keeps more of the SM's L1
template <int R>
constexpr int smem_bytes() { return OFF_MISC + (R >= 4 ? 9216 : MISC_BYTES) + 1024; }

struct Misc {
    uint64_t bar[8];              // load, ops, g, bw, p, y, free, spare
    uint32_t tmem_base;
    int abort_flag;
    int drain_flag;               // abort flag of the final drain waits (never set by others)
    int pad[13];
    float2 qs[2][kNE][32];        // per token group: phase increments of pairs (2i, 2i+1), by tile parity
    union {
        float msk[32 * 36];       // R >= 4: decay mask per (token, token), rows padded
        struct {
            float cs[2][6][128];  // R < 4, by tile parity (the next tile's are made one tile
                                  // ahead): c and gamma times e^{a_ref - a}, a_ref per block; a, gamma, c
            float tk[2][2][132];  // R < 4, by tile parity: dt and lambda of the next tile's
                                  // tokens (clamped to its last) and of the token after it
        };
    } u;
};
static_assert(sizeof(Misc) <= MISC_BYTES, "misc region too small");
static_assert(offsetof(Misc, u) + sizeof(float) * 32 * 36 <= 9216, "misc region of R >= 4 too small");
// bytes of the misc region a launch of rank R uses
template <int R>
constexpr int misc_used() { return R >= 4 ? (int)(offsetof(Misc, u) + sizeof(float) * 32 * 36) : (int)sizeof(Misc); }

enum { BAR_LOAD = 0, BAR_OPS, BAR_G, BAR_BW, BAR_P, BAR_Y, BAR_DRAIN };

// per-tile scalars of a worker thread, made by the coefficient stage
struct TileCoef {
    float a2_last;      // log2 decay over the tile
    float a2_tr;        // log2 decay up to the token of the thread's tile row
    float cf_tr;        // pending weight c of that token (main pass); for
                        // short tiles both hold the lane's own token's
    float dsl;          // dt of token 32 gsl + lane (the warp's phase-pass source)
    float wsl;          // summary pass: state weight e^{a_last - a} c of that token
};

// ------------------------------------------------------------ PTX wrappers --
using namespace ptx;

__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, Misc* m, int* status, int where) {
    return mbar_wait_flag(b, parity, &m->abort_flag, status, where);
}

// 4-byte global -> shared copies of the long tiles' dt / lambda staging
__device__ __forceinline__ void cp_async4(float* dst, const float* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(su32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void workers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kWorkers) : "memory"); }
// all workers get the OR of `cond` (named barrier 1 with a reduction), so
// they take the same branch
__device__ __forceinline__ int workers_any(int cond) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(cond), "n"(kWorkers)
        : "memory");
    return r;
}

// ------------------------------------------------------------------ kernel --
// Worker w (0..255) belongs to warpgroup wg = w / 128 and warp-in-group
// wq = warp % 4, which is the TMEM lane quarter the warp may read.  "Row"
// work (one tile row or state row per thread) is split between the two
// warpgroups by columns; the phase / rotation pass is split by token group
// (one per worker warp) and rotary pair (two per lane).
template <int R, bool SUMMARY>
__global__ void __launch_bounds__(kThreads, 2)
    scan_tc_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmX, ScanParams q, int* status) {
    constexpr int T = kRows / R;       // tokens per tile
    constexpr float kLog2e = 1.4426950408889634f;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base for the SWIZZLE_128B tiles, derived by an offset
    // from the shared array so that every access stays a 32-bit shared access
    uint8_t* smem = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
    Misc* m = reinterpret_cast<Misc*>(smem + OFF_MISC);
    const uint32_t sbase = su32(smem);
    // the whole shared-memory map (tiles and misc region) inside the launch's
    // dynamic shared memory (uniform over the CTA, before any barrier)
    if (!M3_SPAN(1, smem - smem_raw, OFF_MISC + misc_used<R>(), dyn_smem_bytes())) return;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int L = q.seqlen, H = q.nheads, G = q.ngroups;
    const int g = h / (H / G);
    const int tok0 = seg * q.cps * T;
    const int tok1 = min(L, (seg + 1) * q.cps * T);
    const int ntiles = (tok1 - tok0 + T - 1) / T;
    const size_t bh = (size_t)b * H + h;
    const size_t bhs = bh * q.nseg + seg;
    const float Ah = M3_IN(2, h, H) ? q.A[h] : 0.f;
    const long long ext_ws = (long long)q.batch * H * q.nseg;   // segment summaries (debug checks)
    (void)ext_ws;

    // ---- setup
    if (tid == 0) {
        mbar_init(&m->bar[BAR_LOAD], 1);
        mbar_init(&m->bar[BAR_OPS], kWorkers);
        mbar_init(&m->bar[BAR_G], 1);
        mbar_init(&m->bar[BAR_BW], kWorkers);
        mbar_init(&m->bar[BAR_P], kWorkers);
        mbar_init(&m->bar[BAR_Y], 1);
        mbar_init(&m->bar[BAR_DRAIN], 1);
        m->abort_flag = 0;
        m->drain_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, 256);
        tmem_relinquish();
    }

    const int wk = tid - 32;                  // worker index 0..255
    const int wg = wk >> 7;                   // warpgroup: column half of row work
    const int wq = warp & 3;                  // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;           // tile row / state row owned in TMEM
    const int c0 = wg * kSC;                  // this warpgroup's state / y columns
    float S[kSC];                             // state row `row`, columns c0 .. c0+kSC-1
    if (warp > 0) {
        const int n = row;
        if (SUMMARY) {
#pragma unroll
            for (int p = 0; p < kSC; ++p) S[p] = 0.f;
        } else if (q.nseg > 1) {
            const float4* src = reinterpret_cast<const float4*>(q.ws_sin + (bhs * kN + n) * kP + c0);
            const bool ok = M3_SPAN(3, (bhs * kN + n) * kP + c0, kSC, ext_ws * kN * kP);
#pragma unroll
            for (int c = 0; c < kSC / 4; ++c) {
                const float4 v = ok ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
                S[4 * c] = v.x; S[4 * c + 1] = v.y; S[4 * c + 2] = v.z; S[4 * c + 3] = v.w;
            }
        } else {
            const bool ok = !q.init_h || M3_SPAN(4, (bh * kN + n) * kP + c0, kSC, ext_h(q));
#pragma unroll
            for (int p = 0; p < kSC; ++p) S[p] = (q.init_h && ok) ? q.init_h[(bh * kN + n) * kP + c0 + p] : 0.f;
            if (q.init_pB && q.init_pX) {
                const bool ok0 = M3_IN(5, (size_t)b * L * H + h, ext_tok(q));
                const float w0 = ok0 ? (1.f - q.lam[(size_t)b * L * H + h]) * q.dt[(size_t)b * L * H + h] : 0.f;
                const __nv_bfloat16* pB = static_cast<const __nv_bfloat16*>(q.init_pB) + bh * R * kN;
                const __nv_bfloat16* pX = static_cast<const __nv_bfloat16*>(q.init_pX) + bh * R * kP;
                for (int r = 0; r < R; ++r) {
                    if (!M3_IN(6, bh * R * kN + r * kN + n, ext_pB(q)) ||
                        !M3_SPAN(7, bh * R * kP + r * kP + c0, kSC, ext_pX(q)))
                        continue;
                    const float bv = w0 * __bfloat162float(pB[r * kN + n]);
#pragma unroll
                    for (int p = 0; p < kSC; ++p) S[p] = fmaf(bv, __bfloat162float(pX[r * kP + c0 + p]), S[p]);
                }
            }
        }
        if (!SUMMARY) {
#pragma unroll
            for (int c = 0; c < kSC / 8; ++c) {
                uint4 v;
                v.x = pack_bf16x2(S[8 * c + 0], S[8 * c + 1]);
                v.y = pack_bf16x2(S[8 * c + 2], S[8 * c + 3]);
                v.z = pack_bf16x2(S[8 * c + 4], S[8 * c + 5]);
                v.w = pack_bf16x2(S[8 * c + 6], S[8 * c + 7]);
                if (M3_SPAN(8, sw128(n, c0 / 8 + c), 16, 16384))
                    *reinterpret_cast<uint4*>(smem + OFF_S + sw128(n, c0 / 8 + c)) = v;
            }
            fence_async_smem();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;
    const uint32_t tlane = tmem + ((uint32_t)(wq * 32) << 16);   // this warp's lane quarter

    __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(q.y);

    // ---- token work of the workers
    // Every worker warp keeps the whole tile's per-token coefficients in
    // registers (lane l holds tokens l + 32 j, j < NT) and reads another
    // token's value with a shuffle, so the coefficient step needs no shared
    // memory and no barrier.  The phase / rotation pass gives worker warp qe
    // the tokens [qe*TE, (qe+1)*TE) of the tile and lane l the rotary pairs
    // 2l and 2l+1 (one 8-byte word of a B / C row).
    constexpr int NT = (T + 31) / 32;
    constexpr int TE = T / kNE;
    constexpr bool kAhead = (R <= 2);        // coefficient stage one tile ahead
    static_assert(kAhead || NT == 1, "short tiles fit one 32-token slice");
    constexpr bool kThReg = (TE <= 4);        // theta of the group held in registers for the tile
    constexpr int kBatchTE = kThReg ? TE : 8;  // theta loads of the rotation pass issued together
    constexpr unsigned kFull = 0xffffffffu;
    constexpr float kLn2 = 0.69314718055994531f;
    const float A2 = Ah * kLog2e;             // decay per unit dt, log2 units
    const int qe = warp - 1;                  // token group (warp-uniform)
    const int g0 = qe * TE;                   // its first token
    const int gsl = g0 >> 5, gln = g0 & 31;   // slice and lane holding that token
    const int tr = row / R;                   // token of this thread's tile row
    const int rsl = tr >> 5, rln = tr & 31;   // (rsl is warp-uniform for every R)

    // Input loads read clamped (always valid) addresses and keep the raw
    // values; tokens past the tile's end are masked where the values are
    // used, so no instruction waits on a load right after issuing it.
    float dt_n[NT], lam_n[NT], dx_n = 0.f, lx_n = 1.f;
    auto load_tok = [&](int kn) {             // dt, lambda of tile kn and of the token after it
        const int t0n = tok0 + kn * T;
        const int qcn = min(T, tok1 - t0n);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int t = min(lane + 32 * j, qcn - 1);
            const size_t o = ((size_t)b * L + t0n + t) * H + h;
            const bool ok = M3_IN(9, o, ext_tok(q));
            dt_n[j] = ok ? __ldg(q.dt + o) : 0.f;
            lam_n[j] = ok ? __ldg(q.lam + o) : 1.f;
        }
        const int tn = min(t0n + qcn, L - 1);
        const size_t o = ((size_t)b * L + tn) * H + h;
        const bool ok = M3_IN(10, o, ext_tok(q));
        dx_n = ok ? __ldg(q.dt + o) : 0.f;
        lx_n = ok ? __ldg(q.lam + o) : 1.f;
    };
    auto theta_ld = [&](int t0n, int qcn, int kk) -> float2 {   // theta of pairs (2 lane, 2 lane + 1), raw
        const int t = min(g0 + kk, qcn - 1);
        return M3_SPAN(11, (((size_t)b * L + t0n + t) * G + g) * (kN / 2) + 2 * lane, 2, ext_theta(q))
                   ? __ldg(reinterpret_cast<const float2*>(q.theta + (((size_t)b * L + t0n + t) * G + g) * (kN / 2)) + lane)
                   : make_float2(0.f, 0.f);
    };
    // long tiles: tile kn's dt / lambda copied into shared memory (parity kn & 1)
    // by cp.async, a tile ahead of their use: slot s < T holds token
    // min(s, last of the tile), slot T the token after the tile (or the last
    // token); the copies land before the worker barrier of the tile that
    // issues them and are read after it, so no register waits on them
    auto stage_tok = [&](int kn) {
        const int t0n = tok0 + kn * T;
        const int qcn = min(T, tok1 - t0n);
        if (wk <= T) {
            const int t = wk < T ? t0n + min(wk, qcn - 1) : min(t0n + qcn, L - 1);
            const size_t o = ((size_t)b * L + t) * H + h;
            if (M3_IN(12, o, ext_tok(q))) {
                cp_async4(&m->u.tk[kn & 1][0][wk], q.dt + o);
                cp_async4(&m->u.tk[kn & 1][1][wk], q.lam + o);
            }
        }
        cp_async_commit();
    };
    auto take_tok = [&](int kn) {             // the staged values of tile kn into the load registers
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            dt_n[j] = m->u.tk[kn & 1][0][lane + 32 * j];
            lam_n[j] = m->u.tk[kn & 1][1][lane + 32 * j];
        }
        dx_n = m->u.tk[kn & 1][0][T];
        lx_n = m->u.tk[kn & 1][1][T];
    };
    auto prefetch_theta = [&](int kn) {       // L2 prefetch of a tile's theta rows (256 B per token)
        const int t0n = tok0 + kn * T;
        const int qn = min(T, tok1 - t0n);
        for (int j = wk; j < 2 * T; j += kWorkers) {
            const int t = j >> 1;
            if (t < qn && M3_IN(13, (((size_t)b * L + t0n + t) * G + g) * (kN / 2) + (j & 1) * 32, ext_theta(q)))
                prefetch_l2(q.theta + (((size_t)b * L + t0n + t) * G + g) * (kN / 2) + (j & 1) * 32);
        }
    };
    // y = Y_intra + e^{a_t} Y_inter of a finished tile (thread = tile row (t, r),
    // this warpgroup's columns); run while the next tile's load lands
    auto emit_y = [&](int t0y, int qcy, float eay) {
        const float2 ea2 = make_float2(eay, eay);
#pragma unroll 1
        for (int hh = 0; hh < kSC / 16; ++hh) {
            float yi[16], yx[16];
            tmem_ld16(tlane + c0 + 16 * hh, yi);
            tmem_ld16(tlane + 192 + c0 + 16 * hh, yx);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                const float2 o2 = __ffma2_rn(ea2, make_float2(yx[j], yx[j + 1]), make_float2(yi[j], yi[j + 1]));
                yi[j] = o2.x;
                yi[j + 1] = o2.y;
            }
            if (tr < qcy &&
                M3_SPAN(14, ((((size_t)b * L + t0y + tr) * H + h) * R + (row % R)) * kP + c0 + 16 * hh, 16, ext_x(q))) {
                uint4* dst = reinterpret_cast<uint4*>(
                    yg + ((((size_t)b * L + t0y + tr) * H + h) * R + (row % R)) * kP + c0 + 16 * hh);
                dst[0] = pack_chunk(yi);
                dst[1] = pack_chunk(yi + 8);
            }
        }
    };
    int y_tile = -1;                          // tile whose y is waiting to be emitted (-1: none)
    float y_ea = 0.f;                         // e^{a_t} of this thread's row in that tile
    float2 carry = make_float2(0.f, 0.f);     // cumulative phase of pairs 2 lane, 2 lane + 1 (reduced)
    float seg_a = 0.f;                        // log decay of the segment so far
    // ---- coefficient stage of tile kn (run one tile ahead, while the
    // previous tile's MMAs are in flight): per-token coefficients from the
    // raw dt / lambda loads of tile kn, the mask tables of parity kn & 1, and
    // the scalars the tile's own passes need later
    auto coef_stage = [&](int kn) -> TileCoef {
        const int t0n = tok0 + kn * T;
        const int qcn = min(T, tok1 - t0n);
        const int pb = kn & 1;
        // this tile's inputs; tokens past the end count as dt = 0, lambda = 1
        float dtv[NT], lmv[NT];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const bool in = lane + 32 * j < qcn;
            dtv[j] = in ? dt_n[j] : 0.f;
            lmv[j] = in ? lam_n[j] : 1.f;
        }
        const bool nx_in = t0n + qcn < L;
        const float dx = nx_in ? dx_n : 0.f, lx = nx_in ? lx_n : 1.f;
        // coefficients of every token (log2 units): a2 = inclusive scan of
        // dt A, gamma = lambda dt, c = gamma + (1 - lambda') dt' with ' the
        // next token (past the tile: the token after it, zero past the end)
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
        if (!SUMMARY && R >= 4) {
            // decay mask per (token t, token u) of the tile, shared by the R x R
            // rank block: e^{a_t - a_u} (gamma_u if u == t, c_u if u < t), 0 above
            constexpr int LD = T + 4;
#pragma unroll
            for (int e = wk; e < T * T; e += kWorkers) {
                const int t = e / T, u = e % T;
                const float at = __shfl_sync(kFull, a2v[0], t), au = __shfl_sync(kFull, a2v[0], u);
                const float gu = __shfl_sync(kFull, gmv[0], u), cu = __shfl_sync(kFull, cfv[0], u);
                if (M3_IN(15, t * LD + u, 32 * 36))
                    m->u.msk[t * LD + u] = (u <= t) ? exp2f(at - au) * (u == t ? gu : cu) : 0.f;
            }
        }
        if (!SUMMARY && R < 4 && qe == 0) {
            // long tiles: the mask of a 16-column block (GT tokens) factors as
            // e^{a_t - a_ref} x e^{a_ref - a_u} (gamma_u or c_u), a_ref = a at the
            // block's first token, whenever the block's own decay is small
            // enough that the second factor cannot overflow; such blocks get
            // a_ref, the others +inf (element-wise path)
            constexpr int GT = 16 / R;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const int t = lane + 32 * j;
                const float aref = __shfl_sync(kFull, a2v[j], lane & ~(GT - 1));
                const float aend = __shfl_sync(kFull, a2v[j], lane | (GT - 1));
                const bool ok = aref - aend <= 60.f;
                const float colf = exp2f(aref - a2v[j]);
                if (!M3_IN(16, t, 128)) continue;
                m->u.cs[pb][0][t] = ok ? cfv[j] * colf : 0.f;
                m->u.cs[pb][1][t] = ok ? gmv[j] * colf : 0.f;
                if ((lane & (GT - 1)) == 0) m->u.cs[pb][2][t / GT] = ok ? aref : __int_as_float(0x7f800000);
                m->u.cs[pb][3][t] = a2v[j];
                m->u.cs[pb][4][t] = gmv[j];
                m->u.cs[pb][5][t] = cfv[j];
            }
        }
        TileCoef c;
        c.a2_last = a2_last;
        // (short tiles, one slice: the lane's own a and c; the row's are
        // fetched where they are used)
        c.a2_tr = kAhead ? __shfl_sync(kFull, pick<NT>(a2v, rsl), rln) : a2v[0];
        c.cf_tr = SUMMARY ? 0.f : (kAhead ? __shfl_sync(kFull, pick<NT>(cfv, rsl), rln) : cfv[0]);
        c.dsl = pick<NT>(dtv, gsl);
        c.wsl = SUMMARY ? exp2f(a2_last - pick<NT>(a2v, gsl)) * pick<NT>(cfv, gsl) : 0.f;
        return c;
    };
    // ---- phase pass 1 of tile kn: this group's increments of pairs
    // (2 lane, 2 lane + 1), published in qs[kn & 1]; thf(kk) gives the theta
    // of token g0 + kk (theta past the tile's end meets dt = 0)
    auto pass1_stage = [&](int kn, float dsl, auto&& thf) {
        // theta loads issued in batches of up to 8 tokens before their use
        // (long tiles, one tile ahead: all 16 at once)
        constexpr int KB = kAhead ? TE : (TE < 8 ? TE : 8);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int k0 = 0; k0 < TE; k0 += KB) {
            float2 thv[KB];
#pragma unroll
            for (int kk = 0; kk < KB; ++kk) thv[kk] = thf(k0 + kk);
#pragma unroll
            for (int kk = 0; kk < KB; ++kk) {
                const float d = __shfl_sync(kFull, dsl, gln + k0 + kk);
                acc.x = fmaf(d, thv[kk].x, acc.x);
                acc.y = fmaf(d, thv[kk].y, acc.y);
            }
        }
        if (M3_IN(17, qe, kNE)) m->qs[kn & 1][qe][lane] = acc;
    };
    auto pass1_ahead = [&](int kn, float dsl) {   // theta straight from memory (L2)
        const int t0n = tok0 + kn * T;
        const int qcn = min(T, tok1 - t0n);
        pass1_stage(kn, dsl, [&](int kk) { return theta_ld(t0n, qcn, kk); });
    };
    TileCoef cur = {0.f, 0.f, 0.f, 0.f, 0.f};
    if (warp > 0 && ntiles > 0) {
        load_tok(0);
        prefetch_theta(0);
        if (ntiles > 1) prefetch_theta(1);
        if (kAhead) {
            cur = coef_stage(0);
            pass1_ahead(0, cur.dsl);
        }
    }

    uint32_t pending_load = 0;   // control lane: a TMA load is in flight
    uint32_t load_par = 0;       // its mbarrier phase

    for (int k = 0; k < ntiles; ++k) {
        const int t0 = tok0 + k * T;
        const int qc = min(T, tok1 - t0);
        const uint32_t par = k & 1;

        if (warp == 0) {
            // the whole warp takes the same exit (lanes 1..31 meet lane 0 at __syncwarp)
            if (__any_sync(0xffffffffu, *(volatile int*)&m->abort_flag)) break;
            if (lane == 0) {
                // ---------------- producer + MMA issuer
                // The previous tile's MMAs are the last readers of B, C, X: once
                // they complete, the next tile's loads can land while the
                // workers still run that tile's epilogue.
                if (k > 0) mbar_wait(&m->bar[BAR_Y], (k - 1) & 1, m, status, 1);
                const uint32_t bytes = SUMMARY ? (32768u + 16384u) : (65536u + 16384u);
                // tensor coordinates (the copy engine bounds them itself: only noted)
                M3_NOTE(18, t0, L);
                M3_NOTE(19, g, G);
                M3_NOTE(20, b, q.batch);
                mbar_expect_tx(&m->bar[BAR_LOAD], bytes);
                tma_load_5d(sbase + OFF_B, &tmB, &m->bar[BAR_LOAD], 0, 0, g, t0, b);
                tma_load_5d(sbase + OFF_B + 16384, &tmB, &m->bar[BAR_LOAD], 64, 0, g, t0, b);
                if (!SUMMARY) {
                    tma_load_5d(sbase + OFF_C, &tmC, &m->bar[BAR_LOAD], 0, 0, g, t0, b);
                    tma_load_5d(sbase + OFF_C + 16384, &tmC, &m->bar[BAR_LOAD], 64, 0, g, t0, b);
                }
                tma_load_5d(sbase + OFF_X, &tmX, &m->bar[BAR_LOAD], 0, 0, h, t0, b);
                pending_load = 1;
                load_par = par;
                // the next tile into L2: its load, issued once this tile's MMAs
                // are done, then waits for L2 instead of DRAM.  Only for cut
                // sequences: there the grid holds few CTAs and each tile's load
                // latency sits on the critical path; with one segment per
                // sequence the SMs hold enough CTAs to hide it.
                if (q.nseg > 1 && k + 1 < ntiles) {
                    const int tn = t0 + T;
                    tma_prefetch_5d(&tmB, 0, 0, g, tn, b);
                    tma_prefetch_5d(&tmB, 64, 0, g, tn, b);
                    if (!SUMMARY) {
                        tma_prefetch_5d(&tmC, 0, 0, g, tn, b);
                        tma_prefetch_5d(&tmC, 64, 0, g, tn, b);
                    }
                    tma_prefetch_5d(&tmX, 0, 0, h, tn, b);
                }
                // every worker saw the load complete before arriving here
                if (mbar_wait(&m->bar[BAR_OPS], par, m, status, 2)) pending_load = 0;
                tc_fence_after();
                const uint32_t d_g = tmem, d_sl = tmem + 128, d_yx = tmem + 192;
                if (!SUMMARY) {
                    // G = C~ B~^T : both K-major, K = n in two 64-wide atoms
                    constexpr uint32_t idG = idesc_bf16(128, 128, 0, 0);
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        umma(d_g, sdesc(sbase + OFF_C + off, 16, 1024), sdesc(sbase + OFF_B + off, 16, 1024), idG,
                             kk > 0);
                    }
                    // Y_inter = C~ S_bf : A K-major (K = n), B MN-major (K = n rows, N = p)
                    constexpr uint32_t idY = idesc_bf16(128, 64, 0, 1);
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t offa = (kk >> 2) * 16384 + (kk & 3) * 32;
                        umma(d_yx, sdesc(sbase + OFF_C + offa, 16, 1024),
                             sdesc(sbase + OFF_S + kk * 2048, 8192, 1024), idY, kk > 0);
                    }
                    umma_commit(&m->bar[BAR_G]);
                    mbar_wait(&m->bar[BAR_BW], par, m, status, 3);
                    tc_fence_after();
                }
                // S_loc = B~^T (w X) : A MN-major (M = n, two 64-wide blocks 16 KB apart),
                // B MN-major (N = p); K = tile rows, 16 rows (2 KB) per instruction.
                // The summary pass has w folded into B~ and reads X; the main
                // pass reads w X from the S_bf region.
                constexpr uint32_t idS = idesc_bf16(128, 64, 1, 1);
                const uint32_t off_wx = SUMMARY ? OFF_X : OFF_S;
                for (int kk = 0; kk < 8; ++kk)
                    umma(d_sl, sdesc(sbase + OFF_B + kk * 2048, 16384, 1024),
                         sdesc(sbase + off_wx + kk * 2048, 8192, 1024), idS, kk > 0);
                if (!SUMMARY) {
                    mbar_wait(&m->bar[BAR_P], par, m, status, 4);
                    tc_fence_after();
                    // Y_intra = P X : A K-major (K = tile cols in two atoms), B MN-major
                    constexpr uint32_t idI = idesc_bf16(128, 64, 0, 1);
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t offa = (kk >> 2) * 16384 + (kk & 3) * 32;
                        umma(d_g, sdesc(sbase + OFF_C + offa, 16, 1024),
                             sdesc(sbase + OFF_X + kk * 2048, 8192, 1024), idI, kk > 0);
                    }
                }
                umma_commit(&m->bar[BAR_Y]);
            }
            __syncwarp();
            continue;
        }

        // ---------------------------------------------------------- workers
        // Long tiles (R <= 2): tile k's coefficients (cur), mask tables and
        // phase increments were made one tile ahead, in the previous tile's
        // MMA wait; the next tile's dt / lambda are copied into shared memory
        // now and read once this tile's MMAs are issued.  Short tiles (R >= 4)
        // make them here: their MMA waits are too short to hide the stage
        // (measured).
        if (kAhead && k + 1 < ntiles) stage_tok(k + 1);
        // theta of tokens g0 + kk (zero past the end): short groups load it
        // here, ahead of its first use (L2 hits, prefetched two tiles ahead);
        // long groups reload it where it is used
        float2 th[kThReg ? TE : 1];
        if (kThReg) {
#pragma unroll
            for (int kk = 0; kk < TE; ++kk) th[kThReg ? kk : 0] = theta_ld(t0, qc, kk);
        }
        if (k + 2 < ntiles) prefetch_theta(k + 2);
        auto th_at = [&](int kk) -> float2 {
            const float2 v = kThReg ? th[kThReg ? kk : 0] : theta_ld(t0, qc, kk);
            return (g0 + kk < qc) ? v : make_float2(0.f, 0.f);
        };
        if (!kAhead) {
            cur = coef_stage(k);
            pass1_stage(k, cur.dsl, th_at);
        }
        // the previous tile's output, while this tile's TMA load lands
        if (!SUMMARY && y_tile >= 0) {
            emit_y(tok0 + y_tile * T, T, y_ea);     // a tile before the last is full
            y_tile = -1;
        }
        mbar_wait(&m->bar[BAR_LOAD], par, m, status, 10);
        if (kAhead) cp_async_wait_all();          // this thread's staged dt / lambda have landed
        // one barrier per tile: publishes qs, msk and the staged dt / lambda;
        // all workers agree to stop
        if (workers_any(*(volatile int*)&m->abort_flag)) break;
        // the shared base as an opaque value produced after the barrier: the
        // rotation's loads take their addresses from it, so they cannot be
        // moved above the tile's arrival, while they may be hoisted above the
        // pass's own stores (which never touch the same bytes)
        uint32_t sb_ld = sbase;
        asm volatile("" : "+r"(sb_ld));
        float2 ph = carry;
        {
            float2 tot = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < kNE; ++j) {
                const float2 v = m->qs[par][j][lane];
                if (j < qe) { ph.x += v.x; ph.y += v.y; }
                tot.x += v.x;
                tot.y += v.y;
            }
            carry = make_float2(wrap_pi_f(carry.x + tot.x), wrap_pi_f(carry.y + tot.y));
        }
        // phase pass 2: rotate rows (t, r) of B (and C) at pairs (2 lane,
        // 2 lane + 1) in place, bf16x2.  The running phase starts reduced to
        // [-pi, pi] and grows by at most TE increments (|dt theta| each), a few
        // tens of radians at most; at such arguments the fast sine / cosine
        // err by ~1e-5 rad, far below the bf16 rounding of the rotated rows.
        {
            const uint32_t atom = (uint32_t)(lane >> 4) * 16384u;
            const int chunk = (lane & 15) >> 1;
            const uint32_t inb = (uint32_t)(lane & 1) * 8u;
            ph = make_float2(wrap_pi_f(ph.x), wrap_pi_f(ph.y));
            const float dsl = cur.dsl, wsl = cur.wsl;
#pragma unroll 1
            for (int kb = 0; kb < TE; kb += kBatchTE) {
                float2 tb[kBatchTE];
#pragma unroll
                for (int kx = 0; kx < kBatchTE; ++kx) tb[kx] = th_at(kb + kx);
#pragma unroll
                for (int kx = 0; kx < kBatchTE; ++kx) {
                    const int kk = kb + kx;
                    const int t = g0 + kk;
                    const float d = __shfl_sync(kFull, dsl, gln + kk);
                    const float2 tk = tb[kx];
                    ph.x = fmaf(d, tk.x, ph.x);
                    ph.y = fmaf(d, tk.y, ph.y);
                    float s0, k0, s1, k1;
                    __sincosf(ph.x, &s0, &k0);
                    __sincosf(ph.y, &s1, &k1);
                    if (SUMMARY) {
                        // the summary pass needs only w_t B~_t: fold w into the rotation
                        const float wt = __shfl_sync(kFull, wsl, gln + kk);
                        s0 *= wt; k0 *= wt; s1 *= wt; k1 *= wt;
                    }
                    const uint32_t cc0 = pack_bf16x2(k0, k0), sn0 = pack_bf16x2(s0, -s0);
                    const uint32_t cc1 = pack_bf16x2(k1, k1), sn1 = pack_bf16x2(s1, -s1);
                    // all loads of the token's rows first, then the stores (the
                    // loads are free to move ahead of earlier tokens' stores)
                    constexpr int NM = SUMMARY ? 1 : 2;      // B, and C in the main pass
                    uint2 vv[NM][R];
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint32_t off = atom + sw128(t * R + r, chunk) + inb;
#pragma unroll
                        for (int mt = 0; mt < NM; ++mt)
                            vv[mt][r] = M3_SPAN(21, off, 8, 32768) ? lds64_free(sb_ld + (mt ? OFF_C : OFF_B) + off)
                                                                  : make_uint2(0u, 0u);
                    }
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint32_t off = atom + sw128(t * R + r, chunk) + inb;
#pragma unroll
                        for (int mt = 0; mt < NM; ++mt) {
                            uint2 v = vv[mt][r];
                            v.x = rot_bf(v.x, cc0, sn0);
                            v.y = rot_bf(v.y, cc1, sn1);
                            if (M3_SPAN(22, off, 8, 32768))
                                *reinterpret_cast<uint2*>(smem + (mt ? OFF_C : OFF_B) + off) = v;
                        }
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();       // the deferred y's TMEM reads precede the next MMAs
        mbar_arrive(&m->bar[BAR_OPS]);
        // the next tile's coefficients, mask tables and phase increments,
        // while this tile's MMAs run
        TileCoef nxt = cur;
        if (k + 1 < ntiles) {
            // short tiles: consumed at the next tile's top; long tiles: staged
            if (kAhead) take_tok(k + 1);
            else load_tok(k + 1);
            if (kAhead) {
                nxt = coef_stage(k + 1);
                pass1_ahead(k + 1, nxt.dsl);
            }
        }
        // this thread's tile row: its token's log2 decay and pending weight
        const float a2_tr = kAhead ? cur.a2_tr : __shfl_sync(kFull, cur.a2_tr, rln);
        const float a2_last = cur.a2_last;
        if (!SUMMARY) {
            const float cf_tr = kAhead ? cur.cf_tr : __shfl_sync(kFull, cur.cf_tr, rln);
            mbar_wait(&m->bar[BAR_G], par, m, status, 11);
            tc_fence_after();
            // w_t X_t for the chunk-local state, into the S_bf region (free once
            // G and Y_inter are done): this warpgroup's half of X row `row`
            {
                const float wt = exp2f(a2_last - a2_tr) * cf_tr;
                const uint32_t w2 = pack_bf16x2(wt, wt);
                uint4 xv[8 / kWG];
#pragma unroll
                for (int c = 0; c < 8 / kWG; ++c)      // 16-byte chunks of the 128-byte row
                    xv[c] = M3_SPAN(23, sw128(row, wg * (8 / kWG) + c), 16, 16384)
                                ? *reinterpret_cast<const uint4*>(smem + OFF_X + sw128(row, wg * (8 / kWG) + c))
                                : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int c = 0; c < 8 / kWG; ++c)
                    if (M3_SPAN(24, sw128(row, wg * (8 / kWG) + c), 16, 16384))
                        *reinterpret_cast<uint4*>(smem + OFF_S + sw128(row, wg * (8 / kWG) + c)) = scale_chunk(xv[c], w2);
            }
            fence_async_smem();
            mbar_arrive(&m->bar[BAR_BW]);
            // P = (two-band decay mask) o G on this warpgroup's 64 columns,
            // bf16, K-major over C~'s smem
#pragma unroll 1
            for (int cg = 0; cg < 128 / kWG / 16; ++cg) {
                const int col0 = wg * (128 / kWG) + cg * 16;
                float v[16];
                tmem_ld16(tlane + col0, v);
                if (R >= 4) {
                    // mask from the per-tile table, one value per R columns
                    constexpr int LD = T + 4;
                    const float* mrow = m->u.msk + tr * LD + col0 / R;
                    float mk[16 / R];
                    if (!M3_SPAN(25, tr * LD + col0 / R, 16 / R, 32 * 36)) {
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
                        const float2 g2 = __fmul2_rn(make_float2(mk[j / R], mk[(j + 1) / R]),
                                                     make_float2(v[j], v[j + 1]));
                        v[j] = g2.x;
                        v[j + 1] = g2.y;
                    }
                } else {
                    constexpr int GT = 16 / R;            // tokens per 16-column block
                    const int u0 = col0 / R;              // the block's first token (warp-uniform)
                    // (u0 + 16 / R <= T <= 128 keeps the cs rows below inside their 128 floats)
                    const bool okc = M3_SPAN(26, u0, GT, 128);
                    const float aref = okc ? m->u.cs[par][2][u0 / GT] : 0.f;
                    if (u0 > tr || !okc) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = 0.f;
                    } else if (aref != __int_as_float(0x7f800000)) {
                        const float rowf = exp2f(a2_tr - aref);
#pragma unroll
                        for (int i4 = 0; i4 < GT / 4; ++i4) {
                            const float4 fc = reinterpret_cast<const float4*>(m->u.cs[par][0] + u0)[i4];
                            const float4 fg = reinterpret_cast<const float4*>(m->u.cs[par][1] + u0)[i4];
                            const float mc[4] = {fc.x, fc.y, fc.z, fc.w}, mg[4] = {fg.x, fg.y, fg.z, fg.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int u = u0 + 4 * i4 + e;
                                const float mkv = rowf * ((u < tr) ? mc[e] : (u == tr ? mg[e] : 0.f));
#pragma unroll
                                for (int rr = 0; rr < R; ++rr) v[(4 * i4 + e) * R + rr] *= mkv;
                            }
                        }
                    } else {
                        // strong decay inside the block: element-wise
#pragma unroll
                        for (int j = 0; j < 16; j += R) {
                            const int uu = u0 + j / R;
                            const float au = m->u.cs[par][3][uu], gu = m->u.cs[par][4][uu], cu = m->u.cs[par][5][uu];
                            const float mkv = (uu <= tr) ? exp2f(a2_tr - au) * (uu == tr ? gu : cu) : 0.f;
#pragma unroll
                            for (int rr = 0; rr < R; ++rr) v[j + rr] *= mkv;
                        }
                    }
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int cc = (col0 >> 3) + c;      // 16-byte chunk over 128 columns
                    if (M3_SPAN(27, (cc >> 3) * 16384 + sw128(row, cc & 7), 16, 32768))
                        *reinterpret_cast<uint4*>(smem + OFF_C + (cc >> 3) * 16384 + sw128(row, cc & 7)) =
                            pack_chunk(v + 8 * c);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&m->bar[BAR_P]);
        }

        mbar_wait(&m->bar[BAR_Y], par, m, status, 12);
        tc_fence_after();
        // state: S = e^{a_last} S + S_loc  (thread = state row, this half's columns)
        {
            const float dec = exp2f(a2_last);
            const float2 dec2 = make_float2(dec, dec);
#pragma unroll
            for (int h16 = 0; h16 < kSC / 16; ++h16) {
                float v[16];
                tmem_ld16(tlane + 128 + c0 + 16 * h16, v);
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const int jj = 16 * h16 + j;
                    const float2 s2 = __ffma2_rn(dec2, make_float2(S[jj], S[jj + 1]), make_float2(v[j], v[j + 1]));
                    S[jj] = s2.x;
                    S[jj + 1] = s2.y;
                }
            }
            if (!SUMMARY) {
#pragma unroll
                for (int c = 0; c < kSC / 8; ++c)
                    if (M3_SPAN(28, sw128(row, c0 / 8 + c), 16, 16384))
                        *reinterpret_cast<uint4*>(smem + OFF_S + sw128(row, c0 / 8 + c)) = pack_chunk(S + 8 * c);
            }
        }
        seg_a += a2_last * kLn2;
        if (!SUMMARY) {
            y_tile = k;
            y_ea = exp2f(a2_tr);
        }
        cur = nxt;
        // (the S_bf stores and S_loc reads above are ordered before the next
        // tile's MMAs by the fences ahead of that tile's OPS arrival)
    }

    // ---- epilogue of the segment
    if (warp == 0 && lane == 0) {
        // an aborted tile may still have a TMA load in flight: let it land
        if (pending_load) mbar_wait_flag(&m->bar[BAR_LOAD], load_par, &m->drain_flag, nullptr, 0);
        // all MMAs this thread issued are complete before TMEM is freed
        umma_commit(&m->bar[BAR_DRAIN]);
        mbar_wait_flag(&m->bar[BAR_DRAIN], 0, &m->drain_flag, nullptr, 0);
    }
    if (warp > 0 && !SUMMARY && y_tile >= 0) {
        const int t0y = tok0 + y_tile * T;
        emit_y(t0y, min(T, tok1 - t0y), y_ea);
    }
    if (warp > 0) {
        const int n = row;
        if (SUMMARY) {
            float4* dst = reinterpret_cast<float4*>(q.ws_sloc + (bhs * kN + n) * kP + c0);
            if (M3_SPAN(29, (bhs * kN + n) * kP + c0, kSC, ext_ws * kN * kP)) {
#pragma unroll
                for (int c = 0; c < kSC / 4; ++c) dst[c] = make_float4(S[4 * c], S[4 * c + 1], S[4 * c + 2], S[4 * c + 3]);
            }
            if (qe == 0 && M3_SPAN(30, bhs * (kN / 2) + 2 * lane, 2, ext_ws * (kN / 2))) {
                q.ws_phase[bhs * (kN / 2) + 2 * lane] = carry.x;
                q.ws_phase[bhs * (kN / 2) + 2 * lane + 1] = carry.y;
            }
            if (wk == 0 && M3_IN(31, bhs, ext_ws)) q.ws_decay[bhs] = seg_a;
        } else if (seg == q.nseg - 1) {
            if (q.fin_h) {
                // phase of pair n/2 is held by lane n/4 of every worker warp
                const float2 cv2 = make_float2(__shfl_sync(kFull, carry.x, n >> 2), __shfl_sync(kFull, carry.y, n >> 2));
                const float phn = ((n >> 1) & 1) ? cv2.y : cv2.x;
                float sv, cv;
                sincosf(phn, &sv, &cv);
                float* dst = q.fin_h + (bh * kN + n) * kP + c0;
                const bool ok = M3_SPAN(32, (bh * kN + n) * kP + c0, kSC, ext_h(q));
#pragma unroll
                for (int p = 0; p < kSC; ++p) {
                    const float other = __shfl_xor_sync(kFull, S[p], 1);
                    if (ok) dst[p] = (n & 1) ? (sv * other + cv * S[p]) : (cv * S[p] - sv * other);
                }
            }
            if (q.fin_pB && L > 0) {
                const size_t os = (((size_t)b * L + L - 1) * G + g) * R * kN, oo = bh * R * kN;
                const __nv_bfloat16* s = static_cast<const __nv_bfloat16*>(q.B) + os;
                __nv_bfloat16* o = static_cast<__nv_bfloat16*>(q.fin_pB) + oo;
                for (int e = wk; e < R * kN; e += kWorkers)
                    if (M3_IN(33, os + e, ext_bc(q)) && M3_IN(34, oo + e, ext_pB(q))) o[e] = s[e];
            }
            if (q.fin_pX && L > 0) {
                const size_t os = (((size_t)b * L + L - 1) * H + h) * R * kP, oo = bh * R * kP;
                const __nv_bfloat16* s = static_cast<const __nv_bfloat16*>(q.x) + os;
                __nv_bfloat16* o = static_cast<__nv_bfloat16*>(q.fin_pX) + oo;
                for (int e = wk; e < R * kP; e += kWorkers)
                    if (M3_IN(35, os + e, ext_x(q)) && M3_IN(36, oo + e, ext_pX(q))) o[e] = s[e];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------- host --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

}  // namespace tc

// 5-D map over [b][t][grp][r][inner] with a box of (64 inner, R, 1, T, 1)
bool make_tile_map(CUtensorMap* map, const void* base, int inner, int R, int grp, int L, int batch, int T) {
    using namespace tc;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[5] = {(cuuint64_t)inner, (cuuint64_t)R, (cuuint64_t)grp, (cuuint64_t)L, (cuuint64_t)batch};
    const cuuint64_t e = 2;   // bf16
    const cuuint64_t strides[4] = {inner * e, (cuuint64_t)R * inner * e, (cuuint64_t)grp * R * inner * e,
                                   (cuuint64_t)L * grp * R * inner * e};
    const cuuint32_t box[5] = {64, (cuuint32_t)R, 1, (cuuint32_t)T, 1};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Diagnostic: one CTA waits, through the same bounded-wait helper the scan
// uses, on an mbarrier that no thread arrives at.  The wait gives up after
// its limit, records M3_ERR_DEVICE_TIMEOUT (and where = 99) in `status` and
// the kernel returns normally: the timeout path, exercised without a fault.
__global__ void wait_selftest_kernel(int* status) {
    __shared__ uint64_t bar;
    __shared__ tc::Misc m;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        m.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) tc::mbar_wait(&bar, 0, &m, status, 99);
    __syncthreads();
}

cudaError_t launch_wait_selftest(int* status, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(status);
    return cudaGetLastError();
}

bool tc_eligible(const m3_dims& d) {
    return d.io_dtype == M3_BF16 && d.dstate == tc::kN && d.headdim == tc::kP &&
           (d.rank == 1 || d.rank == 2 || d.rank == 4 || d.rank == 8);
}

int tc_tile_tokens(int rank) { return tc::kRows / rank; }

template <int R>
static cudaError_t launch_tc_R(const ScanParams& q, int* status, cudaStream_t st) {
    using namespace tc;
    constexpr int T = kRows / R;
    CUtensorMap mB, mC, mX;
    if (!make_tile_map(&mB, q.B, kN, R, q.ngroups, q.seqlen, q.batch, T) ||
        !make_tile_map(&mC, q.C, kN, R, q.ngroups, q.seqlen, q.batch, T) ||
        !make_tile_map(&mX, q.x, kP, R, q.nheads, q.seqlen, q.batch, T))
        return cudaErrorInvalidValue;
    cudaFuncSetAttribute(scan_tc_kernel<R, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<R>());
    cudaFuncSetAttribute(scan_tc_kernel<R, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<R>());
    // two CTAs per SM need the largest shared-memory carveout
    cudaFuncSetAttribute(scan_tc_kernel<R, false>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    cudaFuncSetAttribute(scan_tc_kernel<R, true>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (q.nseg > 1) {
        scan_tc_kernel<R, true><<<dim3(q.nseg - 1, q.nheads, q.batch), kThreads, smem_bytes<R>(), st>>>(mB, mC, mX, q, status);
        cudaError_t e = launch_scan_combine(q, st);
        if (e != cudaSuccess) return e;
    }
    scan_tc_kernel<R, false><<<dim3(q.nseg, q.nheads, q.batch), kThreads, smem_bytes<R>(), st>>>(mB, mC, mX, q, status);
    return cudaGetLastError();
}

template <int R>
static cudaError_t launch_tc_summary_R(const ScanParams& q, int* status, cudaStream_t st) {
    using namespace tc;
    constexpr int T = kRows / R;
    CUtensorMap mB, mC, mX;
    if (!make_tile_map(&mB, q.B, kN, R, q.ngroups, q.seqlen, q.batch, T) ||
        !make_tile_map(&mC, q.C, kN, R, q.ngroups, q.seqlen, q.batch, T) ||
        !make_tile_map(&mX, q.x, kP, R, q.nheads, q.seqlen, q.batch, T))
        return cudaErrorInvalidValue;
    cudaFuncSetAttribute(scan_tc_kernel<R, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<R>());
    cudaFuncSetAttribute(scan_tc_kernel<R, true>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    scan_tc_kernel<R, true><<<dim3(q.nseg - 1, q.nheads, q.batch), kThreads, smem_bytes<R>(), st>>>(mB, mC, mX, q, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_scan_combine(q, st);
}

cudaError_t launch_scan_tc_summary(const m3_dims& d, const ScanParams& q, int* status, cudaStream_t st) {
    switch (d.rank) {
        case 1: return launch_tc_summary_R<1>(q, status, st);
        case 2: return launch_tc_summary_R<2>(q, status, st);
        case 4: return launch_tc_summary_R<4>(q, status, st);
        case 8: return launch_tc_summary_R<8>(q, status, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_scan_tc(const m3_dims& d, const ScanParams& q, int* status, cudaStream_t st) {
    switch (d.rank) {
        case 1: return launch_tc_R<1>(q, status, st);
        case 2: return launch_tc_R<2>(q, status, st);
        case 4: return launch_tc_R<4>(q, status, st);
        case 8: return launch_tc_R<8>(q, status, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace m3

M3_BOUNDS_EXPORT(scan_tc)
