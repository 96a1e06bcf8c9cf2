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
#include "m3_common.cuh"
#include "m3_kernels.h"

namespace m3 {

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
        if (i < NH) {
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
    const T* Bg = static_cast<const T*>(q.B) + ((size_t)b * q.ngroups + g) * R * N;
    const T* Cg = static_cast<const T*>(q.C) + ((size_t)b * q.ngroups + g) * R * N;
    T* PBh = static_cast<T*>(q.prev_B) + (size_t)bh * R * N;
    T* PXh = static_cast<T*>(q.prev_x) + (size_t)bh * R * P;
    const T* Xh = static_cast<const T*>(q.x) + (size_t)bh * R * P;
    for (int e = tid; e < R * N; e += blockDim.x) {
        sB[e] = ld_io(Bg + e);
        sC[e] = ld_io(Cg + e);
        sPB[e] = ld_io(PBh + e);
    }
    for (int e = tid; e < R * P; e += blockDim.x) {
        sX[e] = ld_io(Xh + e);
        sPX[e] = ld_io(PXh + e);
    }
    const float d = q.dt[bh];
    const float lam = q.lam[bh];
    const float a = q.A[h];
    const float* th = q.theta + ((size_t)b * q.ngroups + g) * NH;
    for (int i = tid; i < NH; i += blockDim.x) {
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
            for (int j = 0; j < 4; ++j) sY[(warp * R + r) * P + 4 * lane + j] = yacc[r][j];
    }
    __syncthreads();
    T* Yh = static_cast<T*>(q.y) + (size_t)bh * R * P;
    for (int e = tid; e < R * P; e += blockDim.x) {
        const int r = e / P, p = e % P;
        float acc = 0.f;
        for (int w = 0; w < nwarps; ++w) acc += sY[(w * R + r) * P + p];
        st_io(Yh + e, acc);
    }

    // 5. this token's (B, x) become the carry's previous (B, x)
    for (int e = tid; e < R * N; e += blockDim.x) st_io(PBh + e, sB[e]);
    for (int e = tid; e < R * P; e += blockDim.x) st_io(PXh + e, sX[e]);
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
    cudaError_t e = (d.io_dtype == M3_BF16)
                        ? launch_T<__nv_bfloat16>(q, R, npt, threads, smem, st)
                        : launch_T<float>(q, R, npt, threads, smem, st);
    return e == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

}  // namespace m3
