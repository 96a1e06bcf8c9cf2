// k_step.cu -- single-token recurrent decode of the Mamba-3 SSM layer (sm_100a).
//
// One token of
//   h <- R_t (alpha_t h + beta_t B_{t-1} X_{t-1}^T) + gamma_t B_t X_t^T,
//   y  = C_t^T h
// ("Mamba-3" summary, b-lab.team: section 1 recurrence, section 2 Proposition 2
// rotation blocks, section 3 MIMO shapes), for every (batch, head).
//
// The step is bound by HBM: the float32 state (N x P per head) is read and
// written once and is ~90% of the bytes, while the FLOPs per state element
// are ~(6R+4).  Design: one CTA per (b, h); each thread owns `NPT` rotary
// pairs (2 state rows each) at one float4 column group, so the state streams
// through registers with 128-bit coalesced loads/stores issued before any
// other work; the small per-token operands (B_t, C_t, x_t, the previous B and
// x, and the pair rotations) are staged in shared memory as float32.
#define M3_BOUNDS_FILE 3
#include "m3_bounds.cuh"
#include "m3_common.cuh"
#include "m3_kernels.h"

namespace m3 {

// element counts of the step's buffers, for the index checks of the debug build
__device__ __forceinline__ long long sx_h(const StepParams& q) {
    return (long long)q.batch * q.nheads * q.dstate * q.headdim;
}
__device__ __forceinline__ long long sx_bc(const StepParams& q, int R) { return (long long)q.batch * q.ngroups * R * q.dstate; }
__device__ __forceinline__ long long sx_pb(const StepParams& q, int R) { return (long long)q.batch * q.nheads * R * q.dstate; }
__device__ __forceinline__ long long sx_x(const StepParams& q, int R) { return (long long)q.batch * q.nheads * R * q.headdim; }
__device__ __forceinline__ long long sx_tok(const StepParams& q) { return (long long)q.batch * q.nheads; }
__device__ __forceinline__ long long sx_th(const StepParams& q) { return (long long)q.batch * q.ngroups * (q.dstate / 2); }

// T: io element type; R: rank; NPT: rotary pairs per thread.
template <typename T, int R, int NPT>
__global__ void __launch_bounds__(256) step_kernel(StepParams q) {
    extern __shared__ float smem[];
    const int N = q.dstate, P = q.headdim, NH = N / 2;
    const int PC = P / 4;                      // float4 column groups
    const int IG = blockDim.x / PC;            // pair groups
    const int tid = threadIdx.x;
    const int pc = tid % PC, ig = tid / PC;
    const int bh = blockIdx.x;
    const int b = bh / q.nheads, h = bh % q.nheads;
    const int g = h / (q.nheads / q.ngroups);

    // 1. stream in this thread's slice of the state first (longest latency)
    float4* hs = reinterpret_cast<float4*>(q.h + (size_t)bh * N * P);
    float4 s0[NPT], s1[NPT];
#pragma unroll
    for (int k = 0; k < NPT; ++k) {
        const int i = ig + k * IG;
        if (i < NH && M3_SPAN(1, (size_t)bh * N * P + (size_t)(2 * i + 1) * P + 4 * pc, 4, sx_h(q))) {
            s0[k] = hs[(size_t)(2 * i) * PC + pc];
            s1[k] = hs[(size_t)(2 * i + 1) * PC + pc];
        }
    }

    // 2. per-token operands -> shared memory (float32)
    float* cs = smem;                 // [NH]
    float* sn = cs + NH;              // [NH]
    float* sB = sn + NH;              // [R][N]
    float* sC = sB + R * N;           // [R][N]
    float* sPB = sC + R * N;          // [R][N]
    float* sX = sPB + R * N;          // [R][P]
    float* sPX = sX + R * P;          // [R][P]
    float* sY = sPX + R * P;          // [warps][R][P]
    if (!M3_SPAN(13, (sY - smem) * 4, (blockDim.x >> 5) * R * P * 4, dyn_smem_bytes())) return;
    const T* Bg = static_cast<const T*>(q.B) + ((size_t)b * q.ngroups + g) * R * N;
    const T* Cg = static_cast<const T*>(q.C) + ((size_t)b * q.ngroups + g) * R * N;
    T* PBh = static_cast<T*>(q.prev_B) + (size_t)bh * R * N;
    T* PXh = static_cast<T*>(q.prev_x) + (size_t)bh * R * P;
    const T* Xh = static_cast<const T*>(q.x) + (size_t)bh * R * P;
    for (int e = tid; e < R * N; e += blockDim.x) {
        if (!M3_IN(2, ((size_t)b * q.ngroups + g) * R * N + e, sx_bc(q, R)) || !M3_IN(3, (size_t)bh * R * N + e, sx_pb(q, R)))
            continue;
        sB[e] = ld_io(Bg + e);
        sC[e] = ld_io(Cg + e);
        sPB[e] = ld_io(PBh + e);
    }
    for (int e = tid; e < R * P; e += blockDim.x) {
        if (!M3_IN(4, (size_t)bh * R * P + e, sx_x(q, R))) continue;
        sX[e] = ld_io(Xh + e);
        sPX[e] = ld_io(PXh + e);
    }
    const bool okt = M3_IN(5, bh, sx_tok(q)) && M3_IN(6, h, q.nheads);
    const float d = okt ? q.dt[bh] : 0.f;
    const float lam = okt ? q.lam[bh] : 0.f;
    const float a = okt ? q.A[h] : 0.f;
    const float* th = q.theta + ((size_t)b * q.ngroups + g) * NH;
    for (int i = tid; i < NH; i += blockDim.x) {
        if (!M3_IN(7, ((size_t)b * q.ngroups + g) * NH + i, sx_th(q))) continue;
        const double phi = wrap_pi((double)d * (double)th[i]);
        float sv, cv;
        sincosf((float)phi, &sv, &cv);
        cs[i] = cv;
        sn[i] = sv;
    }
    __syncthreads();

    const float alpha = expf(d * a);
    const float beta = (1.0f - lam) * d * alpha;
    const float gamma = lam * d;

    // 3. update the state slice, accumulate the readout y = C^T h
    float yacc[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
        yacc[r][0] = yacc[r][1] = yacc[r][2] = yacc[r][3] = 0.f;
    float4 px[R], xx[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        px[r] = reinterpret_cast<const float4*>(sPX + r * P)[pc];
        xx[r] = reinterpret_cast<const float4*>(sX + r * P)[pc];
    }
#pragma unroll
    for (int k = 0; k < NPT; ++k) {
        const int i = ig + k * IG;
        if (i >= NH) continue;
        const int n0 = 2 * i, n1 = 2 * i + 1;
        const float c = cs[i], s = sn[i];
        float u0[4] = {s0[k].x, s0[k].y, s0[k].z, s0[k].w};
        float u1[4] = {s1[k].x, s1[k].y, s1[k].z, s1[k].w};
        float pb0[R], pb1[R], b0[R], b1[R], c0[R], c1[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            pb0[r] = sPB[r * N + n0]; pb1[r] = sPB[r * N + n1];
            b0[r] = sB[r * N + n0];   b1[r] = sB[r * N + n1];
            c0[r] = sC[r * N + n0];   c1[r] = sC[r * N + n1];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float bx0 = 0.f, bx1 = 0.f, cx0 = 0.f, cx1 = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float pxv = j == 0 ? px[r].x : j == 1 ? px[r].y : j == 2 ? px[r].z : px[r].w;
                const float xv = j == 0 ? xx[r].x : j == 1 ? xx[r].y : j == 2 ? xx[r].z : xx[r].w;
                bx0 = fmaf(pb0[r], pxv, bx0);
                bx1 = fmaf(pb1[r], pxv, bx1);
                cx0 = fmaf(b0[r], xv, cx0);
                cx1 = fmaf(b1[r], xv, cx1);
            }
            const float v0 = fmaf(alpha, u0[j], beta * bx0);
            const float v1 = fmaf(alpha, u1[j], beta * bx1);
            const float w0 = fmaf(gamma, cx0, c * v0 - s * v1);
            const float w1 = fmaf(gamma, cx1, s * v0 + c * v1);
            u0[j] = w0;
            u1[j] = w1;
#pragma unroll
            for (int r = 0; r < R; ++r) yacc[r][j] = fmaf(c0[r], w0, fmaf(c1[r], w1, yacc[r][j]));
        }
        if (!M3_SPAN(8, (size_t)bh * N * P + (size_t)n1 * P + 4 * pc, 4, sx_h(q))) continue;
        hs[(size_t)n0 * PC + pc] = make_float4(u0[0], u0[1], u0[2], u0[3]);
        hs[(size_t)n1 * PC + pc] = make_float4(u1[0], u1[1], u1[2], u1[3]);
    }

    // 4. reduce y over pair groups: lanes sharing pc inside a warp, then warps
    const int lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            for (int off = PC; off < 32; off <<= 1)
                yacc[r][j] += __shfl_xor_sync(0xffffffffu, yacc[r][j], off);
    if (lane < PC) {                       // lane == pc for the first pair group of the warp
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (M3_IN(9, (warp * R + r) * P + 4 * lane + j, nwarps * R * P))
                    sY[(warp * R + r) * P + 4 * lane + j] = yacc[r][j];
    }
    __syncthreads();
    T* Yh = static_cast<T*>(q.y) + (size_t)bh * R * P;
    for (int e = tid; e < R * P; e += blockDim.x) {
        const int r = e / P, p = e % P;
        float acc = 0.f;
        for (int w = 0; w < nwarps; ++w) acc += sY[(w * R + r) * P + p];
        if (M3_IN(10, (size_t)bh * R * P + e, sx_x(q, R))) st_io(Yh + e, acc);
    }

    // 5. this token's (B, x) become the carry's previous (B, x)
    for (int e = tid; e < R * N; e += blockDim.x)
        if (M3_IN(11, (size_t)bh * R * N + e, sx_pb(q, R))) st_io(PBh + e, sB[e]);
    for (int e = tid; e < R * P; e += blockDim.x)
        if (M3_IN(12, (size_t)bh * R * P + e, sx_x(q, R))) st_io(PXh + e, sX[e]);
}

// ---------------------------------------------------------------------------
// Pipelined decode: a persistent grid in which each CTA streams (b, h) units
// through a STAGES-deep shared-memory ring.  Every unit's inputs -- the
// float32 state (N x P), B_t, C_t, the previous B and x, x_t, theta, dt,
// lambda and A -- are contiguous blocks and are copied with 16-byte cp.async
// (4-byte for the three scalars), committed as one group per unit, so the
// copies of the next units are in flight while the current unit computes.
// The updated state goes straight from registers to global memory with
// coalesced float4 stores.  Same arithmetic and thread mapping as step_kernel.
// Each thread makes the rotations of its own pairs (no barrier between a
// unit's arrival and its state update); the y partials of the warps are
// summed through the consumed state block.  (Adding them into a per-stage
// accumulator with shared-memory atomics instead, which saves one more
// barrier, measured 15 % slower.)
struct PipeLayout {
    int off_h, off_B, off_C, off_PB, off_X, off_PX, off_TH, off_S, stage;
};

__host__ __device__ constexpr PipeLayout pipe_layout(int N, int P, int R, int es) {
    PipeLayout l{};
    l.off_h = 0;
    l.off_B = l.off_h + N * P * 4;
    l.off_C = l.off_B + R * N * es;
    l.off_PB = l.off_C + R * N * es;
    l.off_X = l.off_PB + R * N * es;
    l.off_PX = l.off_X + R * P * es;
    l.off_TH = l.off_PX + R * P * es;
    l.off_S = l.off_TH + (N / 2) * 4;          // dt, lambda, A
    l.stage = ((l.off_S + 16) + 127) & ~127;
    return l;
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N_>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N_) : "memory"); }

// two consecutive io elements (a rotary pair) as float2
__device__ __forceinline__ float2 ld_pair(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 ld_pair(const __nv_bfloat16* p) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

template <typename T, int R, int STAGES, int N, int P>
__global__ void __launch_bounds__(256, 2) step_pipe_kernel(StepParams q, int units) {
    extern __shared__ __align__(128) unsigned char psm[];
    constexpr int NH = N / 2;
    constexpr int PC = P / 4;              // float4 column groups
    constexpr int IG = 256 / PC;           // pair groups
    constexpr int NPT = (NH + IG - 1) / IG;
    static_assert(256 % PC == 0 && PC <= 32 && (PC & (PC - 1)) == 0, "column groups");
    const int tid = threadIdx.x;
    const int pc = tid % PC, ig = tid / PC;
    const int H = q.nheads, G = q.ngroups, HG = H / G;
    constexpr PipeLayout lay = pipe_layout(N, P, R, (int)sizeof(T));
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(psm);

    auto issue = [&](int u, int st) {
        if (u < units) {
            const int b = u / H, h = u - b * H, g = h / HG;
            const size_t bg = (size_t)b * G + g;
            const uint32_t d0 = sbase + st * lay.stage;
            const char* src_h = reinterpret_cast<const char*>(q.h + (size_t)u * N * P);
            constexpr int nh = N * P / 4, nb = R * N * (int)sizeof(T) / 16, nx = R * P * (int)sizeof(T) / 16;
#pragma unroll
            for (int c0 = 0; c0 < nh; c0 += 256)
                if (M3_SPAN(20, (size_t)u * N * P + 4 * (c0 + tid), 4, sx_h(q)) &&
                    M3_SPAN(21, st * lay.stage + lay.off_h + 16 * (c0 + tid), 16, dyn_smem_bytes()))
                    cp16(d0 + lay.off_h + 16 * (c0 + tid), src_h + 16 * (c0 + tid));
            const char* sB = reinterpret_cast<const char*>(static_cast<const T*>(q.B) + bg * R * N);
            const char* sC = reinterpret_cast<const char*>(static_cast<const T*>(q.C) + bg * R * N);
            const char* sPB = reinterpret_cast<const char*>(static_cast<const T*>(q.prev_B) + (size_t)u * R * N);
            const char* sX = reinterpret_cast<const char*>(static_cast<const T*>(q.x) + (size_t)u * R * P);
            const char* sPX = reinterpret_cast<const char*>(static_cast<const T*>(q.prev_x) + (size_t)u * R * P);
            const char* sTH = reinterpret_cast<const char*>(q.theta + bg * NH);
#pragma unroll
            for (int c0 = 0; c0 < nb; c0 += 256) {
                const int c = c0 + tid;
                if ((nb % 256 == 0 || c < nb) &&
                    M3_SPAN(22, (bg * R * N) * sizeof(T) + 16 * c, 16, sx_bc(q, R) * (long long)sizeof(T)) &&
                    M3_SPAN(23, ((size_t)u * R * N) * sizeof(T) + 16 * c, 16, sx_pb(q, R) * (long long)sizeof(T)) &&
                    M3_SPAN(24, st * lay.stage + lay.off_PB + 16 * c, 16, dyn_smem_bytes())) {
                    cp16(d0 + lay.off_B + 16 * c, sB + 16 * c);
                    cp16(d0 + lay.off_C + 16 * c, sC + 16 * c);
                    cp16(d0 + lay.off_PB + 16 * c, sPB + 16 * c);
                }
            }
#pragma unroll
            for (int c0 = 0; c0 < nx; c0 += 256) {
                const int c = c0 + tid;
                if ((nx % 256 == 0 || c < nx) &&
                    M3_SPAN(25, ((size_t)u * R * P) * sizeof(T) + 16 * c, 16, sx_x(q, R) * (long long)sizeof(T)) &&
                    M3_SPAN(26, st * lay.stage + lay.off_PX + 16 * c, 16, dyn_smem_bytes())) {
                    cp16(d0 + lay.off_X + 16 * c, sX + 16 * c);
                    cp16(d0 + lay.off_PX + 16 * c, sPX + 16 * c);
                }
            }
            if (tid < NH / 4 && M3_SPAN(27, bg * NH + 4 * tid, 4, sx_th(q)) &&
                M3_SPAN(28, st * lay.stage + lay.off_TH + 16 * tid, 16, dyn_smem_bytes()))
                cp16(d0 + lay.off_TH + 16 * tid, sTH + 16 * tid);
            if (tid == 0 && M3_IN(29, u, sx_tok(q)) && M3_IN(30, h, H) &&
                M3_SPAN(31, st * lay.stage + lay.off_S, 12, dyn_smem_bytes())) {
                cp4(d0 + lay.off_S, q.dt + u);
                cp4(d0 + lay.off_S + 4, q.lam + u);
                cp4(d0 + lay.off_S + 8, q.A + h);
            }
        }
        cp_commit();    // one group per unit (possibly empty), so wait counts stay uniform
    };

    int u = blockIdx.x;
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) issue(u + s * (int)gridDim.x, s);
    for (int i = 0; u < units; ++i, u += gridDim.x) {
        const int st = i % STAGES;
        cp_wait<STAGES - 2>();       // this thread's copies of unit u have landed
        __syncthreads();             // everyone's, and unit u-1 is finished
        issue(u + (STAGES - 1) * (int)gridDim.x, (i + STAGES - 1) % STAGES);

        const unsigned char* stg = psm + st * lay.stage;
        const float* hs = reinterpret_cast<const float*>(stg + lay.off_h);
        const T* sB = reinterpret_cast<const T*>(stg + lay.off_B);
        const T* sC = reinterpret_cast<const T*>(stg + lay.off_C);
        const T* sPB = reinterpret_cast<const T*>(stg + lay.off_PB);
        const T* sX = reinterpret_cast<const T*>(stg + lay.off_X);
        const T* sPX = reinterpret_cast<const T*>(stg + lay.off_PX);
        const float* sTH = reinterpret_cast<const float*>(stg + lay.off_TH);
        const float* sc = reinterpret_cast<const float*>(stg + lay.off_S);
        const float d = sc[0], lam = sc[1], a = sc[2];
        const float alpha = expf(d * a);
        const float beta = (1.0f - lam) * d * alpha;
        const float gamma = lam * d;
        const float2 alpha2 = make_float2(alpha, alpha), beta2 = make_float2(beta, beta);
        const float2 gamma2 = make_float2(gamma, gamma);
        // this thread's 4 columns of x and of the previous x, duplicated into pairs
        float2 px2[R][4], xx2[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float pv = ld_io(sPX + r * P + 4 * pc + j), xv = ld_io(sX + r * P + 4 * pc + j);
                px2[r][j] = make_float2(pv, pv);
                xx2[r][j] = make_float2(xv, xv);
            }
        // y partials per (rank, column), the two lanes holding the two rows of
        // each pair (summed at the end)
        float2 yacc2[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j) yacc2[r][j] = make_float2(0.f, 0.f);
        float4* hg = reinterpret_cast<float4*>(q.h + (size_t)u * N * P);
#pragma unroll
        for (int k = 0; k < NPT; ++k) {
            const int ip = ig + k * IG;
            if (ip >= NH) continue;
            const int n0 = 2 * ip, n1 = 2 * ip + 1;
            // the pair's rotation by dt theta (reduced to [-pi, pi]: the fast
            // sine and cosine then err by ~1e-6)
            float2 cs;
            __sincosf(wrap_pi_f(d * sTH[ip]), &cs.y, &cs.x);
            const float4 h0 = reinterpret_cast<const float4*>(hs)[n0 * PC + pc];
            const float4 h1 = reinterpret_cast<const float4*>(hs)[n1 * PC + pc];
            // (row n0, row n1) of the previous B, of B_t and of C_t per rank
            float2 pb[R], bb[R], cc[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                pb[r] = ld_pair(sPB + r * N + n0);
                bb[r] = ld_pair(sB + r * N + n0);
                cc[r] = ld_pair(sC + r * N + n0);
            }
            const float hv0[4] = {h0.x, h0.y, h0.z, h0.w};
            const float hv1[4] = {h1.x, h1.y, h1.z, h1.w};
            float o0[4], o1[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float2 bx = make_float2(0.f, 0.f), cx = make_float2(0.f, 0.f);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    bx = __ffma2_rn(pb[r], px2[r][j], bx);
                    cx = __ffma2_rn(bb[r], xx2[r][j], cx);
                }
                // alpha h + beta B_{t-1} x_{t-1}^T, rows (n0, n1)
                const float2 v = __ffma2_rn(alpha2, make_float2(hv0[j], hv1[j]), __fmul2_rn(beta2, bx));
                // rotation R(dt theta) of the pair, then + gamma B_t x_t^T
                const float2 rv = make_float2(cs.x * v.x - cs.y * v.y, cs.y * v.x + cs.x * v.y);
                const float2 w = __ffma2_rn(gamma2, cx, rv);
                o0[j] = w.x;
                o1[j] = w.y;
#pragma unroll
                for (int r = 0; r < R; ++r) yacc2[r][j] = __ffma2_rn(cc[r], w, yacc2[r][j]);
            }
            if (!M3_SPAN(32, (size_t)u * N * P + (size_t)n1 * P + 4 * pc, 4, sx_h(q))) continue;
            hg[(size_t)n0 * PC + pc] = make_float4(o0[0], o0[1], o0[2], o0[3]);
            hg[(size_t)n1 * PC + pc] = make_float4(o1[0], o1[1], o1[2], o1[3]);
        }
        float yacc[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j) yacc[r][j] = yacc2[r][j].x + yacc2[r][j].y;
        // y: reduce over pair groups (lanes sharing pc inside a warp, then warps)
        const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int off = PC; off < 32; off <<= 1)
                    yacc[r][j] += __shfl_xor_sync(0xffffffffu, yacc[r][j], off);
        // the stage's state block is consumed: it holds the per-warp y partials
        __syncthreads();
        float* sY = reinterpret_cast<float*>(psm + st * lay.stage + lay.off_h);   // [warps][R][P]
        if (lane < PC) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int j = 0; j < 4; ++j) sY[(warp * R + r) * P + 4 * lane + j] = yacc[r][j];
        }
        __syncthreads();
        T* Yh = static_cast<T*>(q.y) + (size_t)u * R * P;
#pragma unroll
        for (int e0 = 0; e0 < R * P; e0 += 256) {
            const int e = e0 + tid;
            if ((R * P) % 256 == 0 || e < R * P) {
                float acc = 0.f;
#pragma unroll
                for (int w = 0; w < 8; ++w) acc += sY[w * R * P + e];
                if (M3_IN(33, (size_t)u * R * P + e, sx_x(q, R))) st_io(Yh + e, acc);
            }
        }
        // this token's (B, x) become the carry's previous (B, x): 16-byte copies
        {
            constexpr int nb = R * N * (int)sizeof(T) / 16, nx = R * P * (int)sizeof(T) / 16;
            uint4* oB = reinterpret_cast<uint4*>(static_cast<T*>(q.prev_B) + (size_t)u * R * N);
            uint4* oX = reinterpret_cast<uint4*>(static_cast<T*>(q.prev_x) + (size_t)u * R * P);
            const uint4* iB = reinterpret_cast<const uint4*>(sB);
            const uint4* iX = reinterpret_cast<const uint4*>(sX);
#pragma unroll
            for (int c0 = 0; c0 < nb; c0 += 256)
                if ((nb % 256 == 0 || c0 + tid < nb) &&
                    M3_SPAN(34, ((size_t)u * R * N) * sizeof(T) + 16 * (c0 + tid), 16, sx_pb(q, R) * (long long)sizeof(T)))
                    oB[c0 + tid] = iB[c0 + tid];
#pragma unroll
            for (int c0 = 0; c0 < nx; c0 += 256)
                if ((nx % 256 == 0 || c0 + tid < nx) &&
                    M3_SPAN(35, ((size_t)u * R * P) * sizeof(T) + 16 * (c0 + tid), 16, sx_x(q, R) * (long long)sizeof(T)))
                    oX[c0 + tid] = iX[c0 + tid];
        }
    }
    cp_wait<0>();
}

template <typename T, int R>
static cudaError_t launch_R(const StepParams& q, int npt, int threads, size_t smem, cudaStream_t st) {
    const dim3 grid((unsigned)(q.batch * q.nheads));
    switch (npt) {
        case 1: step_kernel<T, R, 1><<<grid, threads, smem, st>>>(q); break;
        case 2: step_kernel<T, R, 2><<<grid, threads, smem, st>>>(q); break;
        case 4: step_kernel<T, R, 4><<<grid, threads, smem, st>>>(q); break;
        case 8: step_kernel<T, R, 8><<<grid, threads, smem, st>>>(q); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_T(const StepParams& q, int R, int npt, int threads, size_t smem,
                            cudaStream_t st) {
    switch (R) {
        case 1: return launch_R<T, 1>(q, npt, threads, smem, st);
        case 2: return launch_R<T, 2>(q, npt, threads, smem, st);
        case 4: return launch_R<T, 4>(q, npt, threads, smem, st);
        case 8: return launch_R<T, 8>(q, npt, threads, smem, st);
        default: return cudaErrorInvalidValue;
    }
}


constexpr int kPipeStages = 3;

template <typename T, int R>
static cudaError_t launch_pipe_R(const m3_dims& d, const StepParams& q, cudaStream_t st) {
    constexpr int N = 128, P = 64;
    constexpr PipeLayout lay = pipe_layout(N, P, R, (int)sizeof(T));
    const size_t smem = (size_t)kPipeStages * lay.stage;
    static_assert((size_t)8 * R * P * sizeof(float) <= (size_t)N * P * 4, "y scratch fits the state block");
    auto kern = step_pipe_kernel<T, R, kPipeStages, N, P>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return cudaErrorInvalidValue;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    const int units = d.batch * d.nheads;
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
    if (per_sm < 1) per_sm = 1;
    int grid = device_sm_count() * per_sm;
    if (grid > units) grid = units;
    kern<<<grid, 256, smem, st>>>(q, units);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_pipe_T(const m3_dims& d, const StepParams& q, cudaStream_t st) {
    switch (d.rank) {
        case 1: return launch_pipe_R<T, 1>(d, q, st);
        case 2: return launch_pipe_R<T, 2>(d, q, st);
        case 4: return launch_pipe_R<T, 4>(d, q, st);
        case 8: return launch_pipe_R<T, 8>(d, q, st);
        default: return cudaErrorInvalidValue;
    }
}

// Host launcher.  Returns M3_ERR_UNSUPPORTED for shapes this kernel does not
// take (P/4 not a power of two, P > 128, rank not in {1,2,4,8}, more than 8
// pairs per thread).
m3_status launch_step(const m3_dims& d, const StepParams& q, cudaStream_t st) {
    const int P = d.headdim, N = d.dstate, R = d.rank;
    if (P % 4 != 0 || P > 128 || ((P / 4) & (P / 4 - 1)) != 0) return M3_ERR_UNSUPPORTED;
    if (!(R == 1 || R == 2 || R == 4 || R == 8)) return M3_ERR_UNSUPPORTED;
    const int PC = P / 4;
    int IG = 256 / PC;
    if (IG > N / 2) IG = N / 2;
    int threads = IG * PC;
    // whole warps: pad pair groups so the block is a multiple of 32 threads
    while (threads % 32 != 0) { ++IG; threads = IG * PC; }
    int npt = (N / 2 + IG - 1) / IG;
    if (npt > 8) return M3_ERR_UNSUPPORTED;
    if (npt == 3) npt = 4;
    if (npt > 4 && npt < 8) npt = 8;
    const int nwarps = threads / 32;
    const size_t smem = sizeof(float) * ((size_t)N + 3 * (size_t)R * N + 2 * (size_t)R * P +
                                         (size_t)nwarps * R * P);
    if (d.batch == 0) return M3_OK;
    const int es = d.io_dtype == M3_BF16 ? 2 : 4;
    // the pipelined kernel is specialised for the N = 128, P = 64 head
    const bool pipe_ok = N == 128 && P == 64 && threads == 256 && (R * N * es) % 16 == 0;
    cudaError_t e;
    if (pipe_ok) {
        e = (d.io_dtype == M3_BF16) ? launch_pipe_T<__nv_bfloat16>(d, q, st)
                                    : launch_pipe_T<float>(d, q, st);
    } else {
        e = (d.io_dtype == M3_BF16) ? launch_T<__nv_bfloat16>(q, R, npt, threads, smem, st)
                                    : launch_T<float>(q, R, npt, threads, smem, st);
    }
    return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

}  // namespace m3

M3_BOUNDS_EXPORT(step)
