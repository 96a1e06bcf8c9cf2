// k_seq.cu -- token-by-token scan kernels of the two transition variants of
// the Mamba-3 layer: the damping regimes and the low-rank reflection.
//
// Damping regimes ("Understanding Mamba-3 Through Oscillatory Dynamics",
// section 2.2 and Table 1, section 4.1, section 4.2 and appendix C.2): rotary
// pair i of token t evolves over its interval under dt (A I + theta[i] K_s),
// K_s = [[0, -1], [s, 0]]; its 2x2 block is [[c, -sn], [s sn, c]] with
// (c, sn) = (cos phi, sin phi) for s = +1 (underdamped, Mamba-3 itself),
// (1, phi) for s = 0 (critically damped), (cosh phi, sinh phi) for s = -1
// (overdamped), phi = dt theta[i].  The input rule is Mamba-3's
// exponential-trapezoidal one ("Mamba-3" summary, b-lab.team, section 1):
//   h_t = T_t (alpha_t h_{t-1} + beta_t B_{t-1} X_{t-1}^T) + gamma_t B_t X_t^T,
//   y_t = C_t^T h_t   (section 3, MIMO rank R).
// Low-rank reflection (the extension's abstract listed on the same paper's
// page; appendix C.4 for two reflections making a rotation): the diagonal
// alpha_t I of the transition becomes alpha_t (I - 2 u u^T / u^T u), the
// rotation R_t and the rest stay: h_t = R_t H_t (alpha h + beta B X^T) + ...
//
// Why token by token.  The chunked prefill moves the rotation onto B and C
// as a cumulative phase (Proposition 3), which needs the inverse of every
// prefix of transitions: for the overdamped block those grow like e^{|Phi|}
// and for the critical shear like |Phi|, and the reflection is not diagonal
// in any fixed basis, so neither has the chunked tensor-core form.  This
// kernel runs the recurrence directly in float32.
//
// Mapping.  State columns p evolve independently (the transition acts on the
// rows n).  A warp owns PCW (1, 2 or 4) columns of one (batch, head) and every
// row: lane l holds the rotary pairs i = l + 32 k (k < KP), i.e. rows 2i and
// 2i+1, so a pair block never leaves its thread.  Readout and reflection sums
// over n are warp shuffles; nothing crosses warps.  A CTA of 4 warps covers
// 4 PCW columns and stages each token's B, C (and u), theta, dt, lambda and
// its columns of x in shared memory with cp.async, a chunk of TK tokens ahead
// of use (two buffers); once a chunk has landed the CTA makes every token's
// pair blocks and alpha, beta, gamma once, into the same slots, for all its
// warps.  Few (batch, head) sequences get narrow warps (more warps in all,
// to hide the per-token latency), many get wide ones (fewer shared loads).
#define M3_BOUNDS_FILE 5
#include "m3_bounds.cuh"
#include "m3_common.cuh"
#include "m3_kernels.h"

namespace m3 {
namespace seq {

// element count of the reflection vectors u (index checks of the debug build)
__device__ __forceinline__ long long ext_u(const SeqParams& q) {
    return (long long)q.batch * q.seqlen * q.ngroups * q.dstate;
}

constexpr int kWarps = 4;
constexpr int kMaxCB = kWarps * 4;         // columns per CTA at the widest warps
constexpr int kThreads = 32 * kWarps;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Byte layout of one token's slot in shared memory (all offsets multiples of
// 16; x rows of the CTA's columns padded to 16 bytes).
struct Slot {
    int B, C, U, TH, X, XS, DL, CO, CS, bytes;
};
__host__ __device__ inline Slot slot_layout(int R, int N, int es, bool refl, int kcb) {
    Slot s;
    int o = 0;
    s.B = o;  o += R * N * es;
    s.C = o;  o += R * N * es;
    s.U = o;  o += refl ? N * es : 0;
    s.TH = o; o += (N / 2) * 4;
    s.XS = kcb * es < 16 ? 16 : kcb * es;   // bytes per rank row of x
    s.X = o;  o += R * s.XS;
    s.DL = o; o += 16;                      // dt, lambda
    s.CO = o; o += 16;                      // alpha, beta, gamma (made after arrival)
    s.CS = o; o += (N / 2) * 8;             // pair blocks (c, sn) (made after arrival)
    s.bytes = (o + 15) & ~15;
    return s;
}

template <typename T> __device__ __forceinline__ float2 ld2(const T* p);   // rows (2i, 2i+1)
template <> __device__ __forceinline__ float2 ld2<float>(const float* p) { return *reinterpret_cast<const float2*>(p); }
template <> __device__ __forceinline__ float2 ld2<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

// Sum over the warp of NV values per lane.  Afterwards lane l holds the total
// of value index l / (32 / NV) in v[0] (NV a power of two, <= 32): each
// halving step keeps one half and adds the partner lane's other half.
template <int NV>
__device__ __forceinline__ void reduce_scatter(float (&v)[NV], int lane) {
    int m = NV;
    int o = 16;
#pragma unroll
    for (int step = 0; step < 5; ++step, o >>= 1) {
        if (m > 1) {
            const int half = m >> 1;
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int j = 0; j < NV / 2; ++j) {
                if (j < half) {
                    const float send = upper ? v[j] : v[j + half];
                    const float keep = upper ? v[j + half] : v[j];
                    v[j] = keep + __shfl_xor_sync(kFull, send, o);
                }
            }
            m = half;
        } else {
            v[0] += __shfl_xor_sync(kFull, v[0], o);
        }
    }
}

// (c, sn, s) of one pair block for the regime (0 under, 1 critical, 2 over)
__device__ __forceinline__ void pair_block(int regime, float phi, float& c, float& sn, float& sg) {
    if (regime == 0) {
        sincosf(phi, &sn, &c);
        sg = 1.f;
    } else if (regime == 1) {
        c = 1.f;
        sn = phi;
        sg = 0.f;
    } else {
        c = coshf(phi);
        sn = sinhf(phi);
        sg = -1.f;
    }
}

template <typename T, int R, int KP, bool REFL, int PCW>
__global__ void __launch_bounds__(kThreads) seq_kernel(SeqParams q, int TK) {
    constexpr int kPC = PCW;                   // columns per warp
    constexpr int kCB = kWarps * kPC;          // columns per CTA
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c0 = blockIdx.x * kCB;            // first column of the CTA
    const int h = blockIdx.y, b = blockIdx.z;
    const int L = q.seqlen, H = q.nheads, G = q.ngroups, N = q.dstate, P = q.headdim;
    const int NH = N / 2;
    const int g = h / (H / G);
    const size_t bh = (size_t)b * H + h;
    const int cw = c0 + warp * kPC;             // first column of this warp
    const bool wact = cw < P;                   // warp has columns (P is a multiple of 16)
    const float Ah = M3_IN(1, h, H) ? q.A[h] : 0.f;
    const T* xg = static_cast<const T*>(q.x);
    const T* Bg = static_cast<const T*>(q.B);
    const T* Cg = static_cast<const T*>(q.C);
    const T* Ug = static_cast<const T*>(q.u);
    constexpr int es = sizeof(T);
    const Slot sl = slot_layout(R, N, es, REFL, kCB);
    const float sg = (REFL || q.regime == 0) ? 1.f : (q.regime == 1 ? 0.f : -1.f);

    // ---- staging of a chunk of tokens (cp.async, 16-byte pieces)
    auto stage = [&](int chunk, int buf) {
        const int t0 = chunk * TK;
        const int nt = min(TK, L - t0);
        uint8_t* base = smem + (size_t)buf * TK * sl.bytes;
        const int pB = R * N * es / 16, pU = REFL ? N * es / 16 : 0, pT = NH * 4 / 16;
        constexpr int xb = kCB * es;                     // x bytes per rank row
        const int pX = xb < 16 ? 1 : xb / 16;            // copies per rank row
        const int per = 2 * pB + pU + pT + R * pX;
        for (int e = tid; e < nt * per; e += kThreads) {
            const int tt = e / per;
            int k = e % per;
            const size_t bt = (size_t)b * L + t0 + tt;
            uint8_t* s = base + (size_t)tt * sl.bytes;
            // the token's slot inside the launch's dynamic shared memory
            if (!M3_SPAN(2, s - smem, sl.bytes, dyn_smem_bytes())) continue;
            if (k < pB) {
                if (M3_SPAN(3, (bt * G + g) * R * N * es + 16 * k, 16, ext_bc(q) * es))
                    cp_async16(s + sl.B + 16 * k, reinterpret_cast<const uint8_t*>(Bg + (bt * G + g) * R * N) + 16 * k);
                continue;
            }
            k -= pB;
            if (k < pB) {
                if (M3_SPAN(4, (bt * G + g) * R * N * es + 16 * k, 16, ext_bc(q) * es))
                    cp_async16(s + sl.C + 16 * k, reinterpret_cast<const uint8_t*>(Cg + (bt * G + g) * R * N) + 16 * k);
                continue;
            }
            k -= pB;
            if (k < pU) {
                if (M3_SPAN(5, (bt * G + g) * N * es + 16 * k, 16, ext_u(q) * es))
                    cp_async16(s + sl.U + 16 * k, reinterpret_cast<const uint8_t*>(Ug + (bt * G + g) * N) + 16 * k);
                continue;
            }
            k -= pU;
            if (k < pT) {
                if (M3_SPAN(6, (bt * G + g) * NH * 4 + 16 * k, 16, ext_theta(q) * 4))
                    cp_async16(s + sl.TH + 16 * k, reinterpret_cast<const uint8_t*>(q.theta + (bt * G + g) * NH) + 16 * k);
                continue;
            }
            k -= pT;
            const int r = k / pX, kk = k % pX;
            const uint8_t* src = reinterpret_cast<const uint8_t*>(xg + ((bt * H + h) * R + r) * P + c0) + 16 * kk;
            if (xb < 16) {
                if (c0 < P && M3_SPAN(7, (((bt * H + h) * R + r) * P + c0) * es, 8, ext_x(q) * es))
                    cp_async8(s + sl.X + r * sl.XS, src);
            } else if (c0 + kk * 16 / es < P && M3_SPAN(8, (((bt * H + h) * R + r) * P + c0) * es + 16 * kk, 16, ext_x(q) * es)) {
                cp_async16(s + sl.X + r * sl.XS + 16 * kk, src);
            }
        }
        for (int tt = tid; tt < nt; tt += kThreads) {
            const size_t o = ((size_t)b * L + t0 + tt) * H + h;
            uint8_t* s = base + (size_t)tt * sl.bytes + sl.DL;
            if (!M3_IN(9, o, ext_tok(q)) || !M3_SPAN(10, s - smem, 8, dyn_smem_bytes())) continue;
            cp_async4(s, q.dt + o);
            cp_async4(s + 4, q.lam + o);
        }
    };

    // ---- carry in
    float hs[KP][2][kPC];
    float pb[KP][2][R];
    float px[R][kPC];
#pragma unroll
    for (int k = 0; k < KP; ++k) {
        const int i = lane + 32 * k;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
#pragma unroll
            for (int c = 0; c < kPC; ++c)
                hs[k][e][c] = (q.init_h && i < NH && wact && M3_IN(11, (bh * N + 2 * i + e) * P + cw + c, ext_h(q)))
                                  ? q.init_h[(bh * N + 2 * i + e) * P + cw + c] : 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r)
                pb[k][e][r] = (q.init_pB && i < NH && M3_IN(12, (bh * R + r) * N + 2 * i + e, ext_pB(q)))
                                  ? ld_io(static_cast<const T*>(q.init_pB) + (bh * R + r) * N + 2 * i + e)
                                  : 0.f;
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int c = 0; c < kPC; ++c)
            px[r][c] = (q.init_pX && wact && M3_IN(13, (bh * R + r) * P + cw + c, ext_pX(q)))
                           ? ld_io(static_cast<const T*>(q.init_pX) + (bh * R + r) * P + cw + c) : 0.f;

    const int nchunks = (L + TK - 1) / TK;
    stage(0, 0);
    cp_async_commit();
    constexpr int NV = R * kPC;                 // readout values per lane
    for (int ch = 0; ch < nchunks; ++ch) {
        if (ch + 1 < nchunks) stage(ch + 1, (ch + 1) & 1);
        cp_async_commit();
        cp_async_wait_prev();
        __syncthreads();
        const int t0 = ch * TK;
        const int nt = min(TK, L - t0);
        uint8_t* base = smem + (size_t)(ch & 1) * TK * sl.bytes;
        // the chunk's slots inside the launch's dynamic shared memory (uniform)
        if (!M3_SPAN(14, base - smem, (size_t)nt * sl.bytes, dyn_smem_bytes())) break;
        // every token's pair blocks and alpha, beta, gamma, once for all warps
        for (int e = tid; e < nt * NH; e += kThreads) {
            const int tt = e / NH, i = e - tt * NH;
            uint8_t* s = base + (size_t)tt * sl.bytes;
            const float d = reinterpret_cast<const float*>(s + sl.DL)[0];
            float cc, sn, sgn;
            pair_block(REFL ? 0 : q.regime, d * reinterpret_cast<const float*>(s + sl.TH)[i], cc, sn, sgn);
            reinterpret_cast<float2*>(s + sl.CS)[i] = make_float2(cc, sn);
        }
        for (int tt = tid; tt < nt; tt += kThreads) {
            uint8_t* s = base + (size_t)tt * sl.bytes;
            const float d = reinterpret_cast<const float*>(s + sl.DL)[0];
            const float lm = reinterpret_cast<const float*>(s + sl.DL)[1];
            const float al = expf(d * Ah);
            float* co = reinterpret_cast<float*>(s + sl.CO);
            co[0] = al;
            co[1] = (1.f - lm) * d * al;
            co[2] = lm * d;
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const uint8_t* s = base + (size_t)tt * sl.bytes;
            const float al = reinterpret_cast<const float*>(s + sl.CO)[0];
            const float be = reinterpret_cast<const float*>(s + sl.CO)[1];
            const float ga = reinterpret_cast<const float*>(s + sl.CO)[2];
            // this token's x for the warp's columns (same for every lane)
            float xc[R][kPC];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < kPC; ++c)
                    xc[r][c] = ld_io(reinterpret_cast<const T*>(s + sl.X + r * sl.XS) + warp * kPC + c);
            // v = alpha h + beta B_{t-1} X_{t-1}^T
#pragma unroll
            for (int k = 0; k < KP; ++k)
#pragma unroll
                for (int e = 0; e < 2; ++e)
#pragma unroll
                    for (int c = 0; c < kPC; ++c) {
                        float pend = 0.f;
#pragma unroll
                        for (int r = 0; r < R; ++r) pend = fmaf(pb[k][e][r], px[r][c], pend);
                        hs[k][e][c] = fmaf(be, pend, al * hs[k][e][c]);
                    }
            if (REFL) {
                // v <- v - (2 / u^T u) u (u^T v), column by column (u = 0: no reflection)
                float uv[KP][2];
                float uu = 0.f;
#pragma unroll
                for (int k = 0; k < KP; ++k) {
                    const int i = lane + 32 * k;
                    const float2 u2 = i < NH ? ld2(reinterpret_cast<const T*>(s + sl.U) + 2 * i) : make_float2(0.f, 0.f);
                    uv[k][0] = u2.x;
                    uv[k][1] = u2.y;
                    uu = fmaf(u2.x, u2.x, fmaf(u2.y, u2.y, uu));
                }
                float dot[kPC + 1];
#pragma unroll
                for (int c = 0; c < kPC; ++c) {
                    float a = 0.f;
#pragma unroll
                    for (int k = 0; k < KP; ++k) a = fmaf(uv[k][0], hs[k][0][c], fmaf(uv[k][1], hs[k][1][c], a));
                    dot[c] = a;
                }
                dot[kPC] = uu;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
                    for (int c = 0; c <= kPC; ++c) dot[c] += __shfl_xor_sync(kFull, dot[c], o);
                const float f = dot[kPC] > 0.f ? 2.f / dot[kPC] : 0.f;
#pragma unroll
                for (int c = 0; c < kPC; ++c) {
                    const float fd = f * dot[c];
#pragma unroll
                    for (int k = 0; k < KP; ++k) {
                        hs[k][0][c] = fmaf(-fd, uv[k][0], hs[k][0][c]);
                        hs[k][1][c] = fmaf(-fd, uv[k][1], hs[k][1][c]);
                    }
                }
            }
            // pair blocks T_t (the rotation R_t in the reflection variant)
#pragma unroll
            for (int k = 0; k < KP; ++k) {
                const int i = lane + 32 * k;
                const float2 cs = i < NH ? reinterpret_cast<const float2*>(s + sl.CS)[i] : make_float2(1.f, 0.f);
                const float cc = cs.x, sn = cs.y;
#pragma unroll
                for (int c = 0; c < kPC; ++c) {
                    const float v0 = hs[k][0][c], v1 = hs[k][1][c];
                    hs[k][0][c] = fmaf(cc, v0, -sn * v1);
                    hs[k][1][c] = fmaf(sg * sn, v0, cc * v1);
                }
            }
            // + gamma B_t X_t^T; then y = C_t^T h (partial over this lane's rows)
            float bt_[KP][2][R], yv[NV];
#pragma unroll
            for (int j = 0; j < NV; ++j) yv[j] = 0.f;
#pragma unroll
            for (int k = 0; k < KP; ++k) {
                const int i = lane + 32 * k;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float2 b2 = i < NH ? ld2(reinterpret_cast<const T*>(s + sl.B) + r * N + 2 * i) : make_float2(0.f, 0.f);
                    bt_[k][0][r] = b2.x;
                    bt_[k][1][r] = b2.y;
                }
#pragma unroll
                for (int e = 0; e < 2; ++e)
#pragma unroll
                    for (int c = 0; c < kPC; ++c) {
                        float cur = 0.f;
#pragma unroll
                        for (int r = 0; r < R; ++r) cur = fmaf(bt_[k][e][r], xc[r][c], cur);
                        hs[k][e][c] = fmaf(ga, cur, hs[k][e][c]);
                    }
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float2 c2 = i < NH ? ld2(reinterpret_cast<const T*>(s + sl.C) + r * N + 2 * i) : make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < kPC; ++c)
                        yv[r * kPC + c] = fmaf(c2.x, hs[k][0][c], fmaf(c2.y, hs[k][1][c], yv[r * kPC + c]));
                }
            }
            reduce_scatter<NV>(yv, lane);
            constexpr int SPAN = 32 / NV;          // lanes holding one value's total
            if (wact && (lane % SPAN) == 0) {
                const int idx = lane / SPAN, r = idx / kPC, c = idx % kPC;
                if (M3_IN(15, ((((size_t)b * L + t0 + tt) * H + h) * R + r) * P + cw + c, ext_x(q)))
                    st_io(static_cast<T*>(q.y) + ((((size_t)b * L + t0 + tt) * H + h) * R + r) * P + cw + c, yv[0]);
            }
#pragma unroll
            for (int k = 0; k < KP; ++k)
#pragma unroll
                for (int e = 0; e < 2; ++e)
#pragma unroll
                    for (int r = 0; r < R; ++r) pb[k][e][r] = bt_[k][e][r];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < kPC; ++c) px[r][c] = xc[r][c];
        }
        __syncthreads();   // every warp is done with this buffer before it is staged again
    }

    // ---- carry out: the state is in the original frame
#pragma unroll
    for (int k = 0; k < KP; ++k) {
        const int i = lane + 32 * k;
        if (i >= NH) continue;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (q.fin_h && wact)
#pragma unroll
                for (int c = 0; c < kPC; ++c)
                    if (M3_IN(16, (bh * N + 2 * i + e) * P + cw + c, ext_h(q)))
                        q.fin_h[(bh * N + 2 * i + e) * P + cw + c] = hs[k][e][c];
            if (q.fin_pB && blockIdx.x == 0 && warp == 0)
#pragma unroll
                for (int r = 0; r < R; ++r)
                    if (M3_IN(17, (bh * R + r) * N + 2 * i + e, ext_pB(q)))
                        st_io(static_cast<T*>(q.fin_pB) + (bh * R + r) * N + 2 * i + e, pb[k][e][r]);
        }
    }
    if (q.fin_pX && wact && lane == 0)
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int c = 0; c < kPC; ++c)
                if (M3_IN(18, (bh * R + r) * P + cw + c, ext_pX(q)))
                    st_io(static_cast<T*>(q.fin_pX) + (bh * R + r) * P + cw + c, px[r][c]);
}

template <typename T, int R, int KP, bool REFL, int PCW>
static cudaError_t launch_t(const SeqParams& q, cudaStream_t st) {
    constexpr int kCB = kWarps * PCW;
    const Slot sl = slot_layout(R, q.dstate, sizeof(T), REFL, kCB);
    // tokens per staged chunk: up to 16, two buffers within 96 KB
    int TK = (96 * 1024) / (2 * sl.bytes);
    if (TK > 16) TK = 16;
    if (TK < 1) return cudaErrorInvalidValue;
    const size_t smem = (size_t)2 * TK * sl.bytes;
    cudaError_t e = cudaFuncSetAttribute(seq_kernel<T, R, KP, REFL, PCW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((q.headdim + kCB - 1) / kCB, q.nheads, q.batch);
    seq_kernel<T, R, KP, REFL, PCW><<<grid, kThreads, smem, st>>>(q, TK);
    return cudaGetLastError();
}

// columns per warp: 4 (2 and 1 give more warps per SM but measured slower on
// the SISO layer, 0.96 and 1.19 ms against 0.91 ms: the per-token work of a
// warp is mostly fixed; M3_SEQ_COLS=1|2 selects them for comparison)
template <typename T, int R, int KP, bool REFL>
static cudaError_t launch_w(const SeqParams& q, cudaStream_t st) {
    const char* ev = getenv("M3_SEQ_COLS");
    if (ev && ev[0] == '1' && ev[1] == 0) return launch_t<T, R, KP, REFL, 1>(q, st);
    if (ev && ev[0] == '2' && ev[1] == 0) return launch_t<T, R, KP, REFL, 2>(q, st);
    return launch_t<T, R, KP, REFL, 4>(q, st);
}

template <typename T, bool REFL>
static cudaError_t launch_rk(const SeqParams& q, cudaStream_t st) {
    const int KP = (q.dstate / 2 + 31) / 32;
    switch (q.rank * 8 + KP) {
        case 1 * 8 + 1: return launch_w<T, 1, 1, REFL>(q, st);
        case 1 * 8 + 2: return launch_w<T, 1, 2, REFL>(q, st);
        case 1 * 8 + 4: return launch_w<T, 1, 4, REFL>(q, st);
        case 2 * 8 + 1: return launch_w<T, 2, 1, REFL>(q, st);
        case 2 * 8 + 2: return launch_w<T, 2, 2, REFL>(q, st);
        case 2 * 8 + 4: return launch_w<T, 2, 4, REFL>(q, st);
        case 4 * 8 + 1: return launch_w<T, 4, 1, REFL>(q, st);
        case 4 * 8 + 2: return launch_w<T, 4, 2, REFL>(q, st);
        case 4 * 8 + 4: return launch_w<T, 4, 4, REFL>(q, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace seq

bool seq_supported(const m3_dims& d) {
    const int KP = (d.dstate / 2 + 31) / 32;
    return (d.rank == 1 || d.rank == 2 || d.rank == 4) && d.dstate % 8 == 0 && (KP == 1 || KP == 2 || KP == 4) &&
           d.headdim % seq::kMaxCB == 0;
}

cudaError_t launch_seq(const m3_dims& d, const SeqParams& q, cudaStream_t st) {
    const bool refl = q.u != nullptr;
    if (d.io_dtype == M3_BF16)
        return refl ? seq::launch_rk<__nv_bfloat16, true>(q, st) : seq::launch_rk<__nv_bfloat16, false>(q, st);
    return refl ? seq::launch_rk<float, true>(q, st) : seq::launch_rk<float, false>(q, st);
}

}  // namespace m3

M3_BOUNDS_EXPORT(seq)
