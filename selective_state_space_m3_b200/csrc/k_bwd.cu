// k_bwd.cu -- backward pass of the Mamba-3 layer scan (sm_100a, SIMT, fp32).
//
// Reverse mode of the recurrence of "Mamba-3" summary (b-lab.team), section 1
// (h_t = alpha h_{t-1} + beta B_{t-1} x_{t-1} + gamma B_t x_t) with the
// rotation of section 2 (Proposition 2: R_t multiplies the t-1 -> t
// transition) and the MIMO shapes of section 3.  With g_t = dJ/dh_t and
// v_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}^T (the state before R_t):
//   g_t = C_t dy_t + alpha_{t+1} R_{t+1}^T g_{t+1},   dC_t = h_t dy_t^T,
//   D_t = gamma_t g_t + beta_{t+1} R_{t+1}^T g_{t+1},  dB_t = D_t x_t,  dx_t = D_t^T B_t,
//   dgamma = <g_t, B_t x_t^T>,  dalpha = <R_t^T g_t, h_{t-1}>,  dbeta = <R_t^T g_t, B_{t-1} x_{t-1}^T>,
//   dphi_i = sum_p g_t[pair i]^T R'(phi_i) v_t[pair i],
// then the chain to dt, lambda, A and theta through alpha = e^{dt A},
// beta = (1 - lambda) dt alpha, gamma = lambda dt, phi_i = dt theta_i.
//
// The states h_t are needed in reverse order.  A first kernel runs the
// recurrence forward and stores the state before every block of K tokens
// (a checkpoint); the backward kernel, for each block from the last, runs
// the block forward again from its checkpoint into a per-(b, h) scratch of
// K states, then walks the block in reverse.  Each block's token inputs
// (and the token before it) are first staged in shared memory, so the
// per-token steps read nothing from global memory but the states.  One CTA per (b, h); thread j
// owns rotary pair i = j / (P/16) (rows 2i, 2i+1) and 16 columns of the
// state, so rotations stay in the thread; reductions over columns use lane
// shuffles, reductions over rows shared memory.  Gradients of B, C and theta
// (shared by the heads of a group) and of A are accumulated with atomics
// into zeroed float32 buffers.
#define M3_BOUNDS_FILE 6
#include "m3_bounds.cuh"
#include "m3_common.cuh"
#include "m3_kernels.h"

namespace m3 {
namespace bwd {

// element counts of the workspace parts (index checks of the debug build)
__device__ __forceinline__ long long ext_ckpt(const BwdParams& q) {
    return (long long)q.batch * q.nheads * ((q.seqlen + q.K - 1) / q.K) * q.dstate * q.headdim;
}
__device__ __forceinline__ long long ext_scr(const BwdParams& q) {
    return (long long)q.batch * q.nheads * q.K * q.dstate * q.headdim;
}
// the rows (2i, 2i+1) x columns [p0, p0 + 16) of an N x P state block at
// element offset `off` of a buffer: from row 2i, column p0 to row 2i+1,
// column p0 + 15
#define M3_STATE_SPAN(site, off, P, i, p0, ext) M3_SPAN(site, (off) + (size_t)(2 * (i)) * (P) + (p0), (P) + kPW, ext)

constexpr int kPW = 16;            // state columns per thread
constexpr int kMaxThreads = 256;

template <typename T> __device__ __forceinline__ void ld16(const T* p, float* f);
template <> __device__ __forceinline__ void ld16<float>(const float* p, float* f) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 v = q[i];
        f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
    }
}
template <> __device__ __forceinline__ void ld16<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 v = q[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            f[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
        }
    }
}
template <typename T> __device__ __forceinline__ float2 ld2(const T* p);
template <> __device__ __forceinline__ float2 ld2<float>(const float* p) { return *reinterpret_cast<const float2*>(p); }
template <> __device__ __forceinline__ float2 ld2<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Per-thread view of one token's inputs.
template <int R>
struct Tok {
    float x[R][kPW];      // x_t[r][p] on the thread's columns
    float2 b[R];          // (B_t[r][2i], B_t[r][2i+1])
    float d, lam, th;     // dt, lambda, theta_t[i]
};

// The carry-in (B_{-1}, x_{-1}) in the same per-thread view (zeros if absent).
template <typename T, int R>
__device__ __forceinline__ void load_init_prev(const BwdParams& q, int b, int h, int i, int p0, Tok<R>& k) {
    const int H = q.nheads, N = q.dstate, P = q.headdim;
    const size_t bh = (size_t)b * H + h;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (q.init_pX && M3_SPAN(1, (bh * R + r) * P + p0, kPW, ext_pX(q)))
            ld16<T>(static_cast<const T*>(q.init_pX) + (bh * R + r) * P + p0, k.x[r]);
        else for (int c = 0; c < kPW; ++c) k.x[r][c] = 0.f;
        k.b[r] = (q.init_pB && M3_SPAN(2, (bh * R + r) * N + 2 * i, 2, ext_pB(q)))
                     ? ld2<T>(static_cast<const T*>(q.init_pB) + (bh * R + r) * N + 2 * i) : make_float2(0.f, 0.f);
    }
}

__device__ __forceinline__ void st_state(float* dst, int P, int i, int p0, const float (&h0)[kPW], const float (&h1)[kPW]) {
    float4* r0 = reinterpret_cast<float4*>(dst + (size_t)(2 * i) * P + p0);
    float4* r1 = reinterpret_cast<float4*>(dst + (size_t)(2 * i + 1) * P + p0);
#pragma unroll
    for (int c = 0; c < kPW / 4; ++c) {
        r0[c] = make_float4(h0[4 * c], h0[4 * c + 1], h0[4 * c + 2], h0[4 * c + 3]);
        r1[c] = make_float4(h1[4 * c], h1[4 * c + 1], h1[4 * c + 2], h1[4 * c + 3]);
    }
}
__device__ __forceinline__ void ld_state(const float* src, int P, int i, int p0, float (&h0)[kPW], float (&h1)[kPW]) {
    const float4* r0 = reinterpret_cast<const float4*>(src + (size_t)(2 * i) * P + p0);
    const float4* r1 = reinterpret_cast<const float4*>(src + (size_t)(2 * i + 1) * P + p0);
#pragma unroll
    for (int c = 0; c < kPW / 4; ++c) {
        const float4 a = r0[c], e = r1[c];
        h0[4 * c] = a.x; h0[4 * c + 1] = a.y; h0[4 * c + 2] = a.z; h0[4 * c + 3] = a.w;
        h1[4 * c] = e.x; h1[4 * c + 1] = e.y; h1[4 * c + 2] = e.z; h1[4 * c + 3] = e.w;
    }
}

// Shared-memory staging of a block's token inputs.  Slot 0 holds the token
// before the block (the carry-in for the first block), slot 1 + k token t0 + k.
// Per slot: x [R][P], B [R][N], C [R][N], dy [R][P] (io dtype), theta [N/2],
// then dt and lambda; every part starts on a 16-byte boundary.
struct StageLayout {
    int ox, ob, oc, oy, oth, osc, bytes;     // byte offsets inside a slot, slot size
};
__host__ __device__ inline StageLayout stage_layout(int R, int N, int P, int sz) {
    StageLayout l;
    l.ox = 0;
    l.ob = l.ox + R * P * sz;
    l.oc = l.ob + R * N * sz;
    l.oy = l.oc + R * N * sz;
    l.oth = l.oy + R * P * sz;
    l.osc = l.oth + ((N / 2) * 4 + 15) / 16 * 16;
    l.bytes = l.osc + 16;
    return l;
}

// Copy tokens t0-1 .. t1-1 (x, B, theta, dt, lambda, and with `full` also C
// and dy) into the stage; the carry-in fills slot 0 when t0 == 0.
template <typename T, int R>
__device__ void stage_block(const BwdParams& q, int b, int h, int g, int t0, int t1, uint8_t* stg,
                            const StageLayout& sl, bool full) {
    const int L = q.seqlen, H = q.nheads, G = q.ngroups, N = q.dstate, P = q.headdim;
    const int nslot = t1 - t0 + 1;
    const int ux = R * P * (int)sizeof(T) / 16, ub = R * N * (int)sizeof(T) / 16;
    const int per = full ? 2 * ux + 2 * ub : ux + ub;          // 16-byte units per slot
    for (int e = threadIdx.x; e < nslot * per; e += blockDim.x) {
        const int sidx = e / per;
        int u = e % per;
        const int t = t0 - 1 + sidx;
        uint8_t* slot = stg + (size_t)sidx * sl.bytes;
        const size_t bt = (size_t)b * L + (t >= 0 ? t : 0);
        const uint4* src;
        uint4* dst;
        long long soff = 0, sext = 0;      // source element offset and buffer extent (debug checks)
        int doff;                          // destination byte offset in the slot
        (void)soff; (void)sext;
        if (u < ux) {
            src = reinterpret_cast<const uint4*>(t >= 0 ? static_cast<const T*>(q.x) + ((bt * H + h) * R) * P
                  : (q.init_pX ? static_cast<const T*>(q.init_pX) + (((size_t)b * H + h) * R) * P : nullptr));
            dst = reinterpret_cast<uint4*>(slot + sl.ox);
            doff = sl.ox;
            if (M3_DEBUG_BOUNDS) {
                soff = t >= 0 ? (long long)((bt * H + h) * R) * P : (long long)(((size_t)b * H + h) * R) * P;
                sext = t >= 0 ? ext_x(q) : ext_pX(q);
            }
        } else if ((u -= ux) < ub) {
            src = reinterpret_cast<const uint4*>(t >= 0 ? static_cast<const T*>(q.B) + ((bt * G + g) * R) * N
                  : (q.init_pB ? static_cast<const T*>(q.init_pB) + (((size_t)b * H + h) * R) * N : nullptr));
            dst = reinterpret_cast<uint4*>(slot + sl.ob);
            doff = sl.ob;
            if (M3_DEBUG_BOUNDS) {
                soff = t >= 0 ? (long long)((bt * G + g) * R) * N : (long long)(((size_t)b * H + h) * R) * N;
                sext = t >= 0 ? ext_bc(q) : ext_pB(q);
            }
        } else if ((u -= ub) < ub) {
            src = t >= 0 ? reinterpret_cast<const uint4*>(static_cast<const T*>(q.C) + ((bt * G + g) * R) * N) : nullptr;
            dst = reinterpret_cast<uint4*>(slot + sl.oc);
            doff = sl.oc;
            if (M3_DEBUG_BOUNDS) {
                soff = (long long)((bt * G + g) * R) * N;
                sext = ext_bc(q);
            }
        } else {
            u -= ub;
            src = t >= 0 ? reinterpret_cast<const uint4*>(static_cast<const T*>(q.dy) + ((bt * H + h) * R) * P) : nullptr;
            dst = reinterpret_cast<uint4*>(slot + sl.oy);
            doff = sl.oy;
            if (M3_DEBUG_BOUNDS) {
                soff = (long long)((bt * H + h) * R) * P;
                sext = ext_x(q);
            }
        }
        (void)doff;
        if (!M3_SPAN(3, (slot - stg) + doff + 16 * u, 16, dyn_smem_bytes())) continue;
        if (src && !M3_SPAN(4, soff * (long long)sizeof(T) + 16 * u, 16, sext * (long long)sizeof(T))) src = nullptr;
        dst[u] = src ? src[u] : make_uint4(0u, 0u, 0u, 0u);
    }
    {
        for (int e = threadIdx.x; e < nslot * (N / 2 + 2); e += blockDim.x) {
            const int sidx = e / (N / 2 + 2), u = e % (N / 2 + 2);
            const int t = t0 - 1 + sidx;
            uint8_t* slot = stg + (size_t)sidx * sl.bytes;
            float v = 0.f;
            if (t >= 0) {
                const size_t bt = (size_t)b * L + t;
                if (u < N / 2 ? M3_IN(5, (bt * G + g) * (N / 2) + u, ext_theta(q)) : M3_IN(6, bt * H + h, ext_tok(q)))
                    v = u < N / 2 ? q.theta[(bt * G + g) * (N / 2) + u] : (u == N / 2 ? q.dt[bt * H + h] : q.lam[bt * H + h]);
            }
            if (!M3_SPAN(7, (slot - stg) + (u < N / 2 ? sl.oth + 4 * u : sl.osc + 4 * (u - N / 2)), 4, dyn_smem_bytes()))
                continue;
            if (u < N / 2) reinterpret_cast<float*>(slot + sl.oth)[u] = v;
            else reinterpret_cast<float*>(slot + sl.osc)[u - N / 2] = v;
        }
    }
}

// One forward token from stage slots (token t and token t - 1), streaming one
// rank's rows at a time: h = R_t (alpha h + beta B_{t-1} x_{t-1}^T) + gamma B_t x_t^T.
template <typename T, int R>
__device__ __forceinline__ void fwd_token_stage(float (&h0)[kPW], float (&h1)[kPW], const uint8_t* pslot,
                                                const uint8_t* slot, const StageLayout& sl, int N, int P, int i,
                                                int p0, float A) {
    const float* sc = reinterpret_cast<const float*>(slot + sl.osc);
    const float d = sc[0], lm = sc[1], th = reinterpret_cast<const float*>(slot + sl.oth)[i];
    const float al = __expf(d * A), be = (1.f - lm) * d * al, ga = lm * d;
    float s, c;
    sincosf(d * th, &s, &c);
#pragma unroll
    for (int e = 0; e < kPW; ++e) { h0[e] *= al; h1[e] *= al; }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float px[kPW];
        ld16<T>(reinterpret_cast<const T*>(pslot + sl.ox) + (size_t)r * P + p0, px);
        const float2 pb = ld2<T>(reinterpret_cast<const T*>(pslot + sl.ob) + (size_t)r * N + 2 * i);
        const float b0 = be * pb.x, b1 = be * pb.y;
#pragma unroll
        for (int e = 0; e < kPW; ++e) { h0[e] = fmaf(b0, px[e], h0[e]); h1[e] = fmaf(b1, px[e], h1[e]); }
    }
#pragma unroll
    for (int e = 0; e < kPW; ++e) {
        const float v0 = h0[e], v1 = h1[e];
        h0[e] = c * v0 - s * v1;
        h1[e] = s * v0 + c * v1;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float xr[kPW];
        ld16<T>(reinterpret_cast<const T*>(slot + sl.ox) + (size_t)r * P + p0, xr);
        const float2 bb = ld2<T>(reinterpret_cast<const T*>(slot + sl.ob) + (size_t)r * N + 2 * i);
        const float b0 = ga * bb.x, b1 = ga * bb.y;
#pragma unroll
        for (int e = 0; e < kPW; ++e) { h0[e] = fmaf(b0, xr[e], h0[e]); h1[e] = fmaf(b1, xr[e], h1[e]); }
    }
}

// Forward over the sequence, storing the state before every block of K tokens.
template <typename T, int R>
__global__ void __launch_bounds__(kMaxThreads) ckpt_kernel(BwdParams q) {
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int N = q.dstate, P = q.headdim, NPB = P / kPW, L = q.seqlen, K = q.K;
    const int nck = (L + K - 1) / K;
    const bool act = tid < (N / 2) * NPB;
    const int i = act ? tid / NPB : 0, p0 = act ? (tid % NPB) * kPW : 0;
    const int g = h / (q.nheads / q.ngroups);
    const size_t bh = (size_t)b * q.nheads + h;
    const float A = M3_IN(10, h, q.nheads) ? q.A[h] : 0.f;
    float h0[kPW], h1[kPW];
    if (q.init_h && M3_STATE_SPAN(11, bh * N * P, P, i, p0, ext_h(q))) ld_state(q.init_h + bh * N * P, P, i, p0, h0, h1);
    else for (int c = 0; c < kPW; ++c) { h0[c] = 0.f; h1[c] = 0.f; }
    extern __shared__ __align__(16) uint8_t stg[];
    const StageLayout sl = stage_layout(R, N, P, (int)sizeof(T));
    for (int c = 0; c < nck; ++c) {
        const int t0 = c * K, t1 = min(L, t0 + K);
        if (act && M3_STATE_SPAN(12, (bh * nck + c) * N * P, P, i, p0, ext_ckpt(q)))
            st_state(q.ws_ckpt + (bh * nck + c) * N * P, P, i, p0, h0, h1);
        stage_block<T, R>(q, b, h, g, t0, t1, stg, sl, false);
        __syncthreads();
        if (act)
            for (int t = t0; t < t1; ++t)
                fwd_token_stage<T, R>(h0, h1, stg + (size_t)(t - t0) * sl.bytes, stg + (size_t)(t - t0 + 1) * sl.bytes,
                                      sl, N, P, i, p0, A);
        __syncthreads();
    }
}

// Reverse pass, one CTA per (b, h).
template <typename T, int R>
__global__ void __launch_bounds__(kMaxThreads, 2) bwd_kernel(BwdParams q) {
    __shared__ float sDx[2][4][kMaxThreads / 32 * 64];   // [parity][r][warp x column block x column]
    __shared__ float sRed[2][8][4];             // [parity][warp][4 scalars]
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = q.dstate, P = q.headdim, NPB = P / kPW, L = q.seqlen, K = q.K, H = q.nheads, G = q.ngroups;
    const int nck = (L + K - 1) / K;
    const int nact = (N / 2) * NPB;
    const bool act = tid < nact;
    const int i = act ? tid / NPB : 0, pb = act ? tid % NPB : 0, p0 = pb * kPW;
    const int g = h / (H / G);
    const size_t bh = (size_t)b * H + h;
    const float A = M3_IN(20, h, H) ? q.A[h] : 0.f;
    const int nwarps = (blockDim.x + 31) / 32;
    float* scr = q.ws_scratch + bh * (size_t)K * N * P;
    const size_t scr_off = bh * (size_t)K * N * P;   // (debug checks)
    (void)scr_off;

    float g0[kPW], g1[kPW], db0[kPW], db1[kPW];
    if (q.d_fin_h && act && M3_STATE_SPAN(21, bh * N * P, P, i, p0, ext_h(q)))
        ld_state(q.d_fin_h + bh * N * P, P, i, p0, g0, g1);
    else for (int c = 0; c < kPW; ++c) { g0[c] = 0.f; g1[c] = 0.f; }
    for (int c = 0; c < kPW; ++c) { db0[c] = 0.f; db1[c] = 0.f; }
    float dA_acc = 0.f;
    // gradients arriving at the final (B, x) copies: into dB_{L-1} (dx_{L-1} below)
    if (q.d_fin_pB && L > 0)
        for (int e = tid; e < R * N; e += blockDim.x)
            if (M3_IN(22, (((size_t)b * L + L - 1) * G + g) * R * N + e, ext_bc(q)) && M3_IN(23, bh * R * N + e, ext_pB(q)))
                atomicAdd(q.dB + (((size_t)b * L + L - 1) * G + g) * R * N + e, q.d_fin_pB[bh * R * N + e]);

    extern __shared__ __align__(16) uint8_t stg[];
    const StageLayout sl = stage_layout(R, N, P, (int)sizeof(T));
    int par = 0;
    for (int c = nck - 1; c >= 0; --c) {
        const int t0 = c * K, t1 = min(L, t0 + K);
        // every input of the block (and of the token before it) into shared memory
        stage_block<T, R>(q, b, h, g, t0, t1, stg, sl, true);
        __syncthreads();
        // (a) the block forward again from its checkpoint: h_{t0} .. h_{t1-1} into scratch
        {
            float h0[kPW], h1[kPW];
            if (act) {
                if (M3_STATE_SPAN(24, (bh * nck + c) * N * P, P, i, p0, ext_ckpt(q)))
                    ld_state(q.ws_ckpt + (bh * nck + c) * N * P, P, i, p0, h0, h1);
                else for (int e = 0; e < kPW; ++e) h0[e] = h1[e] = 0.f;
                for (int t = t0; t < t1; ++t) {
                    fwd_token_stage<T, R>(h0, h1, stg + (size_t)(t - t0) * sl.bytes,
                                          stg + (size_t)(t - t0 + 1) * sl.bytes, sl, N, P, i, p0, A);
                    if (M3_STATE_SPAN(25, scr_off + (size_t)(t - t0) * N * P, P, i, p0, ext_scr(q)))
                        st_state(scr + (size_t)(t - t0) * N * P, P, i, p0, h0, h1);
                }
            }
        }
        // (b) reverse over the block.  The step runs in phases that each
        // stream one rank's rows at a time, so few values are live at once.
        for (int t = t1 - 1; t >= t0; --t) {
            const size_t bt = (size_t)b * L + t;
            const uint8_t* slot = stg + (size_t)(t - t0 + 1) * sl.bytes;       // token t
            const uint8_t* pslot = stg + (size_t)(t - t0) * sl.bytes;          // token t - 1 (or the carry-in)
            const float d = reinterpret_cast<const float*>(slot + sl.osc)[0];
            const float lm = reinterpret_cast<const float*>(slot + sl.osc)[1];
            const float th = reinterpret_cast<const float*>(slot + sl.oth)[i];
            const float al = __expf(d * A), be = (1.f - lm) * d * al, ga = lm * d;
            float sn, cs_;
            sincosf(act ? d * th : 0.f, &sn, &cs_);
            const T* xs = reinterpret_cast<const T*>(slot + sl.ox) + p0;
            const T* bs = reinterpret_cast<const T*>(slot + sl.ob) + 2 * i;
            const T* ys = reinterpret_cast<const T*>(slot + sl.oy) + p0;
            const T* cs = reinterpret_cast<const T*>(slot + sl.oc) + 2 * i;

            // phase 1 -- readout: g += C_t dy_t ; dC_t = h_t dy_t^T
            {
                float ht0[kPW], ht1[kPW];
                if (act && M3_STATE_SPAN(26, scr_off + (size_t)(t - t0) * N * P, P, i, p0, ext_scr(q)))
                    ld_state(scr + (size_t)(t - t0) * N * P, P, i, p0, ht0, ht1);
                else for (int e = 0; e < kPW; ++e) ht0[e] = ht1[e] = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float dy[kPW];
                    ld16<T>(ys + (size_t)r * P, dy);
                    float2 cr = ld2<T>(cs + (size_t)r * N);
                    if (!act) cr = make_float2(0.f, 0.f);
                    float dc0 = 0.f, dc1 = 0.f;
#pragma unroll
                    for (int e = 0; e < kPW; ++e) {
                        g0[e] = fmaf(cr.x, dy[e], g0[e]);
                        g1[e] = fmaf(cr.y, dy[e], g1[e]);
                        dc0 = fmaf(ht0[e], dy[e], dc0);
                        dc1 = fmaf(ht1[e], dy[e], dc1);
                    }
                    for (int o = 1; o < NPB; o <<= 1) {
                        dc0 += __shfl_xor_sync(0xffffffffu, dc0, o);
                        dc1 += __shfl_xor_sync(0xffffffffu, dc1, o);
                    }
                    if (act && pb == 0 && M3_SPAN(27, ((bt * G + g) * R + r) * N + 2 * i, 2, ext_bc(q))) {
                        float* dCt = q.dC + ((bt * G + g) * R + r) * N + 2 * i;
                        atomicAdd(dCt, dc0);
                        atomicAdd(dCt + 1, dc1);
                    }
                }
            }
            // phase 2 -- input terms: D = gamma g + beta' R'^T g' ; dB = D x ; dx = D^T B ;
            // dgamma = <g, B x^T>
            float s_ga = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float xr[kPW];
                ld16<T>(xs + (size_t)r * P, xr);
                float2 br = ld2<T>(bs + (size_t)r * N);
                if (!act) br = make_float2(0.f, 0.f);
                float db_0 = 0.f, db_1 = 0.f, dxr[kPW];
#pragma unroll
                for (int e = 0; e < kPW; ++e) {
                    const float D0 = fmaf(ga, g0[e], db0[e]), D1 = fmaf(ga, g1[e], db1[e]);
                    db_0 = fmaf(D0, xr[e], db_0);
                    db_1 = fmaf(D1, xr[e], db_1);
                    dxr[e] = act ? fmaf(D0, br.x, D1 * br.y) : 0.f;
                    s_ga = fmaf(fmaf(g0[e], br.x, g1[e] * br.y), xr[e], s_ga);
                }
                for (int o = 1; o < NPB; o <<= 1) {
                    db_0 += __shfl_xor_sync(0xffffffffu, db_0, o);
                    db_1 += __shfl_xor_sync(0xffffffffu, db_1, o);
                }
                if (act && pb == 0 && M3_SPAN(28, ((bt * G + g) * R + r) * N + 2 * i, 2, ext_bc(q))) {
                    float* dBt = q.dB + ((bt * G + g) * R + r) * N + 2 * i;
                    atomicAdd(dBt, db_0);
                    atomicAdd(dBt + 1, db_1);
                }
                // dx: over the row pairs (lanes with the same column block, then warps)
                for (int o = NPB; o < 32; o <<= 1)
#pragma unroll
                    for (int e = 0; e < kPW; ++e) dxr[e] += __shfl_xor_sync(0xffffffffu, dxr[e], o);
                if (lane < NPB && M3_SPAN(29, (warp * NPB + lane) * kPW, kPW, kMaxThreads / 32 * 64))
#pragma unroll
                    for (int e = 0; e < kPW; ++e) sDx[par][r][(warp * NPB + lane) * kPW + e] = dxr[e];
            }
            if (!act) s_ga = 0.f;
            // phase 3 -- the transition: gv = R_t^T g ; dphi ; dalpha = <gv, h_{t-1}> ;
            // dbeta = <gv, B_{t-1} x_{t-1}^T> ; carry the adjoint
            float s_al = 0.f, s_be = 0.f, dph = 0.f;
#pragma unroll
            for (int e = 0; e < kPW; ++e) {
                const float gv0 = cs_ * g0[e] + sn * g1[e], gv1 = -sn * g0[e] + cs_ * g1[e];
                g0[e] = gv0;
                g1[e] = gv1;
            }
            {
                float hp0[kPW], hp1[kPW];
                if (act && (t > t0 ? M3_STATE_SPAN(30, scr_off + (size_t)(t - 1 - t0) * N * P, P, i, p0, ext_scr(q))
                                   : M3_STATE_SPAN(31, (bh * nck + c) * N * P, P, i, p0, ext_ckpt(q)))) {
                    if (t > t0) ld_state(scr + (size_t)(t - 1 - t0) * N * P, P, i, p0, hp0, hp1);
                    else ld_state(q.ws_ckpt + (bh * nck + c) * N * P, P, i, p0, hp0, hp1);
                } else {
                    for (int e = 0; e < kPW; ++e) hp0[e] = hp1[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < kPW; ++e) {
                    s_al = fmaf(g0[e], hp0[e], fmaf(g1[e], hp1[e], s_al));
                    dph = fmaf(g1[e], hp0[e], fmaf(-g0[e], hp1[e], dph));
                }
                dph *= al;
            }
            {
                // the previous token's (B, x): the carry-in for t = 0 (zeros if absent)
                const T* pxs = reinterpret_cast<const T*>(pslot + sl.ox) + p0;
                const T* pbs = reinterpret_cast<const T*>(pslot + sl.ob) + 2 * i;
                const size_t pstride_b = (size_t)N;
                float dph_p = 0.f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float px[kPW];
                    ld16<T>(pxs + (size_t)r * P, px);
                    float2 pbr = ld2<T>(pbs + (size_t)r * pstride_b);
                    if (!act) pbr = make_float2(0.f, 0.f);
#pragma unroll
                    for (int e = 0; e < kPW; ++e) {
                        s_be = fmaf(fmaf(g0[e], pbr.x, g1[e] * pbr.y), px[e], s_be);
                        dph_p = fmaf(fmaf(g1[e], pbr.x, -g0[e] * pbr.y), px[e], dph_p);
                    }
                }
                dph = fmaf(be, dph_p, dph);
            }
#pragma unroll
            for (int e = 0; e < kPW; ++e) {
                db0[e] = be * g0[e];
                db1[e] = be * g1[e];
                g0[e] *= al;
                g1[e] *= al;
            }
            if (!act) { dph = 0.f; s_al = s_be = 0.f; }
            for (int o = 1; o < NPB; o <<= 1) dph += __shfl_xor_sync(0xffffffffu, dph, o);
            float s_ph = 0.f;
            if (act && pb == 0) {
                if (M3_IN(32, (bt * G + g) * (N / 2) + i, ext_theta(q))) atomicAdd(q.dtheta + (bt * G + g) * (N / 2) + i, dph * d);
                s_ph = dph * th;
            }
            // scalars: reduce over the warp, then over warps in shared memory
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s_ga += __shfl_xor_sync(0xffffffffu, s_ga, o);
                s_al += __shfl_xor_sync(0xffffffffu, s_al, o);
                s_be += __shfl_xor_sync(0xffffffffu, s_be, o);
                s_ph += __shfl_xor_sync(0xffffffffu, s_ph, o);
            }
            if (lane == 0 && M3_IN(33, warp, 8)) {
                sRed[par][warp][0] = s_ga;
                sRed[par][warp][1] = s_al;
                sRed[par][warp][2] = s_be;
                sRed[par][warp][3] = s_ph;
            }
            __syncthreads();
            // dx_t[r][p]: one thread per (r, p)
            for (int e = tid; e < R * P; e += blockDim.x) {
                const int r = e / P, p = e % P, pbk = p / kPW, col = p % kPW;
                float acc = 0.f;
                for (int w = 0; w < nwarps; ++w)
                    if (w * 32 < nact && M3_IN(34, (w * NPB + pbk) * kPW + col, kMaxThreads / 32 * 64))
                        acc += sDx[par][r][(w * NPB + pbk) * kPW + col];
                if (t == L - 1 && q.d_fin_pX && M3_IN(35, bh * R * P + e, ext_pX(q))) acc += q.d_fin_pX[bh * R * P + e];
                if (M3_IN(36, ((bt * H + h) * R) * P + e, ext_x(q))) q.dx[((bt * H + h) * R) * P + e] = acc;
            }
            if (tid == 0) {
                float dga = 0.f, dal = 0.f, dbe = 0.f, dphth = 0.f;
                for (int w = 0; w < nwarps && M3_IN(37, w, 8); ++w) {
                    dga += sRed[par][w][0];
                    dal += sRed[par][w][1];
                    dbe += sRed[par][w][2];
                    dphth += sRed[par][w][3];
                }
                if (M3_IN(38, bt * H + h, ext_tok(q))) {
                    q.ddt[bt * H + h] = dal * A * al + dbe * (1.f - lm) * (al + d * A * al) + dga * lm + dphth;
                    q.dlam[bt * H + h] = -dbe * d * al + dga * d;
                }
                dA_acc += dal * d * al + dbe * (1.f - lm) * d * d * al;
            }
            par ^= 1;
        }
        __syncthreads();      // scratch is rewritten by the next block's forward
    }
    if (tid == 0 && M3_IN(39, h, H)) atomicAdd(q.dA + h, dA_acc);
    // carry-in gradients: d h_{-1} = g ; d prev_B = D_{-1} prev_x ; d prev_x = D_{-1}^T prev_B
    if (q.d_init_h && act && M3_STATE_SPAN(40, bh * N * P, P, i, p0, ext_h(q)))
        st_state(q.d_init_h + bh * N * P, P, i, p0, g0, g1);
    if (q.d_init_pB || q.d_init_pX) {
        Tok<R> pv;
        load_init_prev<T, R>(q, b, h, i, p0, pv);
        float dpb[R][2], dpx[R][kPW];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            dpb[r][0] = dpb[r][1] = 0.f;
#pragma unroll
            for (int e = 0; e < kPW; ++e) {
                dpb[r][0] = fmaf(db0[e], pv.x[r][e], dpb[r][0]);
                dpb[r][1] = fmaf(db1[e], pv.x[r][e], dpb[r][1]);
                dpx[r][e] = act ? fmaf(db0[e], pv.b[r].x, db1[e] * pv.b[r].y) : 0.f;
            }
            if (!act) dpb[r][0] = dpb[r][1] = 0.f;
        }
        for (int o = 1; o < NPB; o <<= 1)
#pragma unroll
            for (int r = 0; r < R; ++r) {
                dpb[r][0] += __shfl_xor_sync(0xffffffffu, dpb[r][0], o);
                dpb[r][1] += __shfl_xor_sync(0xffffffffu, dpb[r][1], o);
            }
        if (q.d_init_pB && act && pb == 0)
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if (!M3_SPAN(41, (bh * R + r) * N + 2 * i, 2, ext_pB(q))) continue;
                q.d_init_pB[(bh * R + r) * N + 2 * i] = dpb[r][0];
                q.d_init_pB[(bh * R + r) * N + 2 * i + 1] = dpb[r][1];
            }
        for (int o = NPB; o < 32; o <<= 1)
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int e = 0; e < kPW; ++e) dpx[r][e] += __shfl_xor_sync(0xffffffffu, dpx[r][e], o);
        if (lane < NPB && M3_SPAN(42, (warp * NPB + lane) * kPW, kPW, kMaxThreads / 32 * 64))
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int e = 0; e < kPW; ++e) sDx[0][r][(warp * NPB + lane) * kPW + e] = dpx[r][e];
        __syncthreads();
        if (q.d_init_pX)
            for (int e = tid; e < R * P; e += blockDim.x) {
                const int r = e / P, p = e % P, pbk = p / kPW, col = p % kPW;
                float acc = 0.f;
                for (int w = 0; w < nwarps; ++w)
                    if (w * 32 < nact && M3_IN(43, (w * NPB + pbk) * kPW + col, kMaxThreads / 32 * 64))
                        acc += sDx[0][r][(w * NPB + pbk) * kPW + col];
                if (M3_IN(44, (bh * R + r) * P + p, ext_pX(q))) q.d_init_pX[(bh * R + r) * P + p] = acc;
            }
    }
}

template <typename T, int R>
static cudaError_t launch_TR(const BwdParams& q, cudaStream_t st) {
    const int threads = ((q.dstate / 2) * (q.headdim / kPW) + 31) / 32 * 32;
    const dim3 grid((unsigned)q.nheads, (unsigned)q.batch);
    const size_t smem = (size_t)(q.K + 1) * stage_layout(R, q.dstate, q.headdim, (int)sizeof(T)).bytes;
    cudaFuncSetAttribute(ckpt_kernel<T, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(bwd_kernel<T, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    ckpt_kernel<T, R><<<grid, threads, smem, st>>>(q);
    bwd_kernel<T, R><<<grid, threads, smem, st>>>(q);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_T(const BwdParams& q, cudaStream_t st) {
    switch (q.rank) {
        case 1: return launch_TR<T, 1>(q, st);
        case 2: return launch_TR<T, 2>(q, st);
        case 3: return launch_TR<T, 3>(q, st);
        case 4: return launch_TR<T, 4>(q, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace bwd

bool bwd_supported(const m3_dims& d) {
    const int P = d.headdim, N = d.dstate;
    return (P == 16 || P == 32 || P == 64) && N % 8 == 0 && (N / 2) * (P / bwd::kPW) <= bwd::kMaxThreads &&
           d.rank >= 1 && d.rank <= 4;
}

// Tokens per block (the checkpoint interval and the shared-memory stage):
// 16, or fewer when a block's inputs would not fit in 160 KB.
int bwd_block_tokens(const m3_dims& d) {
    const int sz = d.io_dtype == M3_BF16 ? 2 : 4;
    const int bytes = bwd::stage_layout(d.rank, d.dstate, d.headdim, sz).bytes;
    int k = 16;
    while (k > 1 && (k + 1) * bytes > 160 * 1024) k >>= 1;
    return k;
}

cudaError_t launch_bwd(const m3_dims& d, const BwdParams& q, cudaStream_t st) {
    return d.io_dtype == M3_BF16 ? bwd::launch_T<__nv_bfloat16>(q, st) : bwd::launch_T<float>(q, st);
}

}  // namespace m3

M3_BOUNDS_EXPORT(bwd)
