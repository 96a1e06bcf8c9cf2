// k_scan_simt.cu -- chunked prefill of the Mamba-3 SSM layer, SIMT float32.
//
// This is the float32 path (the tensor-core path takes bfloat16 operands,
// too coarse for a float32 tolerance) and the fallback for shapes the
// tensor-core kernel does not take.
//
// Chunked form.  With B and C rotated by their cumulative phase (Proposition 3
// of the "Mamba-3" summary, b-lab.team, section 2) the state recurrence loses
// its rotation:  h~_t = alpha_t h~_{t-1} + beta_t B~_{t-1} x_{t-1}^T
//                        + gamma_t B~_t x_t^T,   y_t = C~_t^T h~_t.
// Unrolling it inside a chunk gives the two-band masked matrix of section 1
// (a decay mask times a bidiagonal matrix):
//   y_t = sum_{u<=t} e^{a_t - a_u} w_tu (C~_t . B~_u) x_u + e^{a_t} C~_t^T S_in
//   w_tu = gamma_u (u == t),  c_u = gamma_u + (1-lambda_{u+1}) dt_{u+1} (u < t)
// with a_t the chunk-local cumulative sum of dt*A, and the state passed on is
//   S_out = e^{a_last} S_in + sum_u e^{a_last - a_u} c_u B~_u x_u^T,
// an "augmented" state that already holds the pending beta term of the
// chunk's last token (c_u uses the next token's dt and lambda; the very last
// token of the sequence has none, so its c is gamma).
//
// Parallel layout.  Each (batch, head) sequence is cut into `nseg` segments
// of whole chunks.  A segment works in its own rotation frame, which starts as
// the original frame (phase 0) at the segment's first token.  When nseg > 1:
//   1. summary kernel: every segment but the last computes its local
//      augmented end state from zero, its total log-decay and total phase;
//   2. combine kernel: S_in(k) = R(Phi_{k-1}) (e^{a_{k-1}} S_in(k-1) + S_loc(k-1)),
//      S_in(0) = h_{-1} + (1 - lambda_0) dt_0 B_{-1} x_{-1}^T;
//   3. main kernel: each segment walks its chunks from S_in(k), writes y, and
//      the last segment writes the final carry.
#define M3_BOUNDS_FILE 2
#include "m3_bounds.cuh"
#include "m3_common.cuh"
#include "m3_kernels.h"

namespace m3 {

size_t simt_smem_bytes(int qs, int R, int N, int P, bool summary) {
    const size_t NH = N / 2, QR = (size_t)qs * R;
    size_t f = 2 * (size_t)(qs + 1) + 5 * (size_t)qs + 2 * (size_t)qs * NH + QR * N * (summary ? 1 : 2) +
               QR * P + (summary ? 0 : QR * QR) + (size_t)N * P + 4;
    return NH * sizeof(double) + f * sizeof(float);
}

// Initial augmented state of segment 0 from the caller's carry.
template <typename T>
__device__ __forceinline__ float carry_in(const ScanParams& q, int b, int h, int n, int p, float w0) {
    const int N = q.dstate, P = q.headdim, R = q.rank;
    const size_t bh = (size_t)b * q.nheads + h;
    float v = (q.init_h && M3_IN(1, (bh * N + n) * P + p, ext_h(q))) ? q.init_h[(bh * N + n) * P + p] : 0.f;
    if (q.init_pB && q.init_pX) {
        const T* pB = static_cast<const T*>(q.init_pB) + bh * R * N;
        const T* pX = static_cast<const T*>(q.init_pX) + bh * R * P;
        float acc = 0.f;
        for (int r = 0; r < R; ++r)
            if (M3_IN(2, bh * R * N + r * N + n, ext_pB(q)) && M3_IN(3, bh * R * P + r * P + p, ext_pX(q)))
                acc = fmaf(ld_io(pB + r * N + n), ld_io(pX + r * P + p), acc);
        v = fmaf(w0, acc, v);
    }
    return v;
}

template <typename T, bool SUMMARY>
__global__ void __launch_bounds__(256) scan_simt_kernel(ScanParams q) {
    extern __shared__ double smem_d[];
    const int seg = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int L = q.seqlen, H = q.nheads, G = q.ngroups, N = q.dstate, P = q.headdim, R = q.rank;
    const int NH = N / 2, g = h / (H / G), qs = q.qs, QRmax = qs * R;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int tok0 = seg * q.cps * qs;
    const int tok1 = min(L, (seg + 1) * q.cps * qs);
    const size_t bh = (size_t)b * H + h;
    const size_t bhs = bh * q.nseg + seg;
    const float Ah = M3_IN(4, h, H) ? q.A[h] : 0.f;
    const long long ext_ws = (long long)q.batch * H * q.nseg;   // segment summaries (debug checks)
    (void)ext_ws;

    double* sPhi = smem_d;                                   // [NH]
    float* sf = reinterpret_cast<float*>(sPhi + NH);
    float* sDt = sf;                  sf += qs + 1;
    float* sLam = sf;                 sf += qs + 1;
    float* sA = sf;                   sf += qs;
    float* sEa = sf;                  sf += qs;
    float* sGam = sf;                 sf += qs;
    float* sCf = sf;                  sf += qs;
    float* sW = sf;                   sf += qs;
    float* sCos = sf;                 sf += qs * NH;
    float* sSin = sf;                 sf += qs * NH;
    float* sB = sf;                   sf += QRmax * N;
    float* sC = sf;                   if (!SUMMARY) sf += QRmax * N;
    float* sX = sf;                   sf += QRmax * P;
    float* sG = sf;                   if (!SUMMARY) sf += QRmax * QRmax;
    float* sS = sf;                   sf += N * P;
    float* sScal = sf;                // [0] = chunk decay e^{a_last}, [1] = segment log-decay
    // the carved arrays end inside the launch's dynamic shared memory
    if (!M3_SPAN(5, reinterpret_cast<const char*>(sScal) - reinterpret_cast<const char*>(smem_d), 8,
                 dyn_smem_bytes()))
        return;

    for (int i = tid; i < NH; i += nt) sPhi[i] = 0.0;
    if (tid == 0) sScal[1] = 0.f;
    if (SUMMARY) {
        for (int e = tid; e < N * P; e += nt) sS[e] = 0.f;
    } else if (q.nseg > 1) {
        for (int e = tid; e < N * P; e += nt)
            sS[e] = M3_IN(6, bhs * N * P + e, ext_ws * N * P) ? q.ws_sin[bhs * N * P + e] : 0.f;
    } else {
        const float w0 = (L > 0 && M3_IN(7, (size_t)b * L * H + h, ext_tok(q)))
                             ? (1.f - q.lam[(size_t)b * L * H + h]) * q.dt[(size_t)b * L * H + h] : 0.f;
        for (int e = tid; e < N * P; e += nt) sS[e] = carry_in<T>(q, b, h, e / P, e % P, w0);
    }
    __syncthreads();

    const T* xg = static_cast<const T*>(q.x);
    const T* Bg = static_cast<const T*>(q.B);
    const T* Cg = static_cast<const T*>(q.C);
    T* yg = static_cast<T*>(q.y);

    for (int c0 = tok0; c0 < tok1; c0 += qs) {
        const int qc = min(qs, tok1 - c0);
        const int has_next = (c0 + qc < L) ? 1 : 0;
        const int QR = qc * R;
        for (int k = tid; k < qc + has_next; k += nt) {
            const size_t o = ((size_t)b * L + c0 + k) * H + h;
            if (!M3_IN(8, k, qs + 1) || !M3_IN(9, o, ext_tok(q))) continue;
            sDt[k] = q.dt[o];
            sLam[k] = q.lam[o];
        }
        __syncthreads();
        // discretisation coefficients of the chunk (section 1 of the summary)
        if (tid == 0) {
            float acc = 0.f;
            for (int k = 0; k < qc; ++k) {
                acc += sDt[k] * Ah;
                sA[k] = acc;
                sEa[k] = expf(acc);
                sGam[k] = sLam[k] * sDt[k];
                const float nxt = (k + 1 < qc + has_next) ? (1.f - sLam[k + 1]) * sDt[k + 1] : 0.f;
                sCf[k] = sGam[k] + nxt;
            }
            for (int k = 0; k < qc; ++k) sW[k] = expf(acc - sA[k]) * sCf[k];
            sScal[0] = expf(acc);
            sScal[1] += acc;
        }
        // cumulative phase of the chunk, one thread per rotary pair
        for (int i = tid; i < NH; i += nt) {
            double ph = sPhi[i];
            for (int k = 0; k < qc; ++k) {
                const float th = M3_IN(10, (((size_t)b * L + c0 + k) * G + g) * NH + i, ext_theta(q))
                                     ? q.theta[(((size_t)b * L + c0 + k) * G + g) * NH + i] : 0.f;
                ph = wrap_pi(ph + (double)sDt[k] * (double)th);
                float sv, cv;
                sincosf((float)ph, &sv, &cv);
                if (!M3_IN(11, k * NH + i, qs * NH)) continue;
                sCos[k * NH + i] = cv;
                sSin[k * NH + i] = sv;
            }
            sPhi[i] = ph;
        }
        __syncthreads();
        // B~ = R(Phi)^T B, C~ = R(Phi)^T C, and X, into shared memory
        for (int e = tid; e < qc * R * NH; e += nt) {
            const int i = e % NH, kr = e / NH, k = kr / R;
            const size_t src = ((((size_t)b * L + c0 + k) * G + g) * R + (kr % R)) * N + 2 * i;
            if (!M3_IN(12, k * NH + i, qs * NH) || !M3_SPAN(13, kr * N + 2 * i, 2, QRmax * N) ||
                !M3_SPAN(14, src, 2, ext_bc(q)))
                continue;
            const float c = sCos[k * NH + i], s = sSin[k * NH + i];
            const float b0 = ld_io(Bg + src), b1 = ld_io(Bg + src + 1);
            sB[kr * N + 2 * i] = c * b0 + s * b1;
            sB[kr * N + 2 * i + 1] = -s * b0 + c * b1;
            if (!SUMMARY) {
                const float c0v = ld_io(Cg + src), c1v = ld_io(Cg + src + 1);
                sC[kr * N + 2 * i] = c * c0v + s * c1v;
                sC[kr * N + 2 * i + 1] = -s * c0v + c * c1v;
            }
        }
        for (int e = tid; e < QR * P; e += nt) {
            const int p = e % P, kr = e / P, k = kr / R;
            if (!M3_IN(15, e, QRmax * P) || !M3_IN(16, ((((size_t)b * L + c0 + k) * H + h) * R + (kr % R)) * P + p, ext_x(q)))
                continue;
            sX[e] = ld_io(xg + ((((size_t)b * L + c0 + k) * H + h) * R + (kr % R)) * P + p);
        }
        __syncthreads();
        if (!SUMMARY) {
            // masked Gram: (two-band mask) o (C~ B~^T), rows/cols ordered (t, r)
            for (int e = tid; e < QR * QR; e += nt) {
                const int i = e / QR, j = e % QR, ki = i / R, kj = j / R;
                float v = 0.f;
                if (!M3_IN(17, e, QRmax * QRmax) || !M3_SPAN(18, i * N, N, QRmax * N) ||
                    !M3_SPAN(19, j * N, N, QRmax * N) || !M3_IN(20, ki, qs) || !M3_IN(21, kj, qs))
                    continue;
                if (kj <= ki) {
                    float dot = 0.f;
                    for (int n = 0; n < N; ++n) dot = fmaf(sC[i * N + n], sB[j * N + n], dot);
                    const float m = expf(sA[ki] - sA[kj]) * (ki == kj ? sGam[kj] : sCf[kj]);
                    v = dot * m;
                }
                sG[e] = v;
            }
            __syncthreads();
            // y = (M o G) X + e^{a_t} C~ S_in
            for (int e = tid; e < QR * P; e += nt) {
                const int i = e / P, p = e % P, ki = i / R;
                float acc = 0.f, acc2 = 0.f;
                const int jend = (ki + 1) * R;
                if (!M3_SPAN(22, i * QR, jend, QRmax * QRmax) || !M3_IN(23, (jend - 1) * P + p, QRmax * P) ||
                    !M3_SPAN(24, i * N, N, QRmax * N) || !M3_IN(25, ki, qs) ||
                    !M3_IN(26, ((((size_t)b * L + c0 + ki) * H + h) * R + (i % R)) * P + p, ext_x(q)))
                    continue;
                for (int j = 0; j < jend; ++j) acc = fmaf(sG[i * QR + j], sX[j * P + p], acc);
                for (int n = 0; n < N; ++n) acc2 = fmaf(sC[i * N + n], sS[n * P + p], acc2);
                st_io(yg + ((((size_t)b * L + c0 + ki) * H + h) * R + (i % R)) * P + p,
                      fmaf(sEa[ki], acc2, acc));
            }
            __syncthreads();
        }
        // S_out = e^{a_last} S_in + sum_u e^{a_last - a_u} c_u B~_u x_u^T
        const float dec = sScal[0];
        for (int e = tid; e < N * P; e += nt) {
            const int n = e / P, p = e % P;
            float acc = 0.f;
            if (!M3_IN(27, (QR - 1) * N + n, QRmax * N) || !M3_IN(28, (QR - 1) * P + p, QRmax * P) ||
                !M3_IN(29, (QR - 1) / R, qs))
                continue;
            for (int j = 0; j < QR; ++j) acc = fmaf(sB[j * N + n] * sW[j / R], sX[j * P + p], acc);
            sS[e] = fmaf(dec, sS[e], acc);
        }
        __syncthreads();
    }

    if (SUMMARY) {
        for (int e = tid; e < N * P; e += nt)
            if (M3_IN(30, bhs * N * P + e, ext_ws * N * P)) q.ws_sloc[bhs * N * P + e] = sS[e];
        for (int i = tid; i < NH; i += nt)
            if (M3_IN(31, bhs * NH + i, ext_ws * NH)) q.ws_phase[bhs * NH + i] = (float)sPhi[i];
        if (tid == 0 && M3_IN(32, bhs, ext_ws)) q.ws_decay[bhs] = sScal[1];
    } else if (seg == q.nseg - 1) {
        // final carry in the original frame: h = R(Phi) h~
        if (q.fin_h) {
            for (int e = tid; e < NH * P; e += nt) {
                const int i = e / P, p = e % P;
                float sv, cv;
                sincosf((float)sPhi[i], &sv, &cv);
                const float s0 = sS[(2 * i) * P + p], s1 = sS[(2 * i + 1) * P + p];
                if (!M3_IN(33, (bh * N + 2 * i + 1) * P + p, ext_h(q))) continue;
                q.fin_h[(bh * N + 2 * i) * P + p] = cv * s0 - sv * s1;
                q.fin_h[(bh * N + 2 * i + 1) * P + p] = sv * s0 + cv * s1;
            }
        }
        if (q.fin_pB && L > 0) {
            T* o = static_cast<T*>(q.fin_pB) + bh * R * N;
            const T* s = Bg + (((size_t)b * L + L - 1) * G + g) * R * N;
            for (int e = tid; e < R * N; e += nt)
                if (M3_IN(34, bh * R * N + e, ext_pB(q)) && M3_IN(35, (((size_t)b * L + L - 1) * G + g) * R * N + e, ext_bc(q)))
                    o[e] = s[e];
        }
        if (q.fin_pX && L > 0) {
            T* o = static_cast<T*>(q.fin_pX) + bh * R * P;
            const T* s = xg + (((size_t)b * L + L - 1) * H + h) * R * P;
            for (int e = tid; e < R * P; e += nt)
                if (M3_IN(36, bh * R * P + e, ext_pX(q)) && M3_IN(37, (((size_t)b * L + L - 1) * H + h) * R * P + e, ext_x(q)))
                    o[e] = s[e];
        }
    }
}

// S_in(k) for every segment from the segment summaries (see the header).
template <typename T>
__global__ void __launch_bounds__(256) scan_combine_kernel(ScanParams q) {
    const int h = blockIdx.y, b = blockIdx.z;
    const int N = q.dstate, P = q.headdim, NH = N / 2, L = q.seqlen, H = q.nheads;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= NH * P) return;
    const int i = e / P, p = e % P;
    const size_t bh = (size_t)b * H + h;
    const long long ext_ws = (long long)q.batch * H * q.nseg;   // segment summaries (debug checks)
    (void)ext_ws;
    const float w0 = M3_IN(40, (size_t)b * L * H + h, ext_tok(q))
                         ? (1.f - q.lam[(size_t)b * L * H + h]) * q.dt[(size_t)b * L * H + h] : 0.f;
    float s0 = carry_in<T>(q, b, h, 2 * i, p, w0);
    float s1 = carry_in<T>(q, b, h, 2 * i + 1, p, w0);
    // The summaries of a batch of segments are loaded before the chain runs
    // through them (their loads would otherwise wait behind the previous
    // segment's stores, one memory round trip per segment).
    constexpr int KB = 8;
    for (int k0 = 0; k0 < q.nseg; k0 += KB) {
        float l0[KB], l1[KB], dl[KB], ph[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const int k = min(k0 + j, q.nseg - 1);
            const size_t bhs = bh * q.nseg + k;
            const bool ok = M3_IN(41, (bhs * N + 2 * i + 1) * P + p, ext_ws * N * P) && M3_IN(42, bhs * NH + i, ext_ws * NH);
            l0[j] = ok ? __ldg(q.ws_sloc + (bhs * N + 2 * i) * P + p) : 0.f;
            l1[j] = ok ? __ldg(q.ws_sloc + (bhs * N + 2 * i + 1) * P + p) : 0.f;
            dl[j] = ok ? __ldg(q.ws_decay + bhs) : 0.f;
            ph[j] = ok ? __ldg(q.ws_phase + bhs * NH + i) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const int k = k0 + j;
            if (k >= q.nseg) break;
            const size_t bhs = bh * q.nseg + k;
            if (M3_IN(43, (bhs * N + 2 * i + 1) * P + p, ext_ws * N * P)) {
                q.ws_sin[(bhs * N + 2 * i) * P + p] = s0;
                q.ws_sin[(bhs * N + 2 * i + 1) * P + p] = s1;
            }
            if (k + 1 == q.nseg) break;
            const float dec = expf(dl[j]);
            const float v0 = fmaf(dec, s0, l0[j]);
            const float v1 = fmaf(dec, s1, l1[j]);
            float sv, cv;
            sincosf(ph[j], &sv, &cv);
            s0 = cv * v0 - sv * v1;
            s1 = sv * v0 + cv * v1;
        }
    }
}

template <typename T>
static cudaError_t launch_simt_T(const ScanParams& q, cudaStream_t st) {
    const size_t sm_main = simt_smem_bytes(q.qs, q.rank, q.dstate, q.headdim, false);
    const size_t sm_sum = simt_smem_bytes(q.qs, q.rank, q.dstate, q.headdim, true);
    cudaFuncSetAttribute(scan_simt_kernel<T, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_main);
    cudaFuncSetAttribute(scan_simt_kernel<T, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_sum);
    if (q.nseg > 1) {
        scan_simt_kernel<T, true><<<dim3(q.nseg - 1, q.nheads, q.batch), 256, sm_sum, st>>>(q);
        const int NHP = q.dstate / 2 * q.headdim;
        scan_combine_kernel<T><<<dim3((NHP + 255) / 256, q.nheads, q.batch), 256, 0, st>>>(q);
    }
    scan_simt_kernel<T, false><<<dim3(q.nseg, q.nheads, q.batch), 256, sm_main, st>>>(q);
    return cudaGetLastError();
}

// the combine step on its own (used by the tensor-core path, bf16 carry)
cudaError_t launch_scan_combine(const ScanParams& q, cudaStream_t st) {
    const int NHP = q.dstate / 2 * q.headdim;
    scan_combine_kernel<__nv_bfloat16><<<dim3((NHP + 255) / 256, q.nheads, q.batch), 256, 0, st>>>(q);
    return cudaGetLastError();
}

cudaError_t launch_scan_simt(const m3_dims& d, const ScanParams& q, cudaStream_t st) {
    return d.io_dtype == M3_BF16 ? launch_simt_T<__nv_bfloat16>(q, st) : launch_simt_T<float>(q, st);
}

}  // namespace m3

M3_BOUNDS_EXPORT(scan_simt)
