// k_rope.cu -- cumulative phase and rotated B, C ("RoPE trick"), sm_100a.
//
// "Mamba-3" summary (b-lab.team), section 2, Proposition 3: the complex SSM
// equals the real one run on B and C rotated by the cumulative phase
//   Phi_t[i] = sum_{s<=t} dt_s theta_s[i],
//   (B~_{2i}, B~_{2i+1}) = R(Phi_t[i])^T (B_{2i}, B_{2i+1}),  same for C.
// Phi is per head (dt is per head) while theta, B and C are per group, so the
// outputs are per head.
//
// One CTA per (b, h) walks the sequence in blocks of TB tokens: theta and dt
// of the block are staged in shared memory, one thread per rotary pair
// advances the running phase (double precision, reduced to [-pi, pi] every
// token) and stores cos/sin per (token, pair), then all threads rotate the
// block's B and C pairs with coalesced pair-wide loads and stores.
#define M3_BOUNDS_FILE 4
#include "m3_bounds.cuh"
#include "m3_common.cuh"
#include "m3_kernels.h"

namespace m3 {

// element counts of the per-head outputs (B~, C~; the phase), for the index
// checks of the debug build
__device__ __forceinline__ long long rx_rot(const RopeParams& q) {
    return (long long)q.batch * q.seqlen * q.nheads * q.rank * q.dstate;
}
__device__ __forceinline__ long long rx_phase(const RopeParams& q) {
    return (long long)q.batch * q.seqlen * q.nheads * (q.dstate / 2);
}

template <typename T> struct Pair;
template <> struct Pair<float> {
    using V = float2;
    static __device__ __forceinline__ float2 ld(const float* p) { return *reinterpret_cast<const float2*>(p); }
    static __device__ __forceinline__ void st(float* p, float a, float b) {
        *reinterpret_cast<float2*>(p) = make_float2(a, b);
    }
    static __device__ __forceinline__ float lo(float2 v) { return v.x; }
    static __device__ __forceinline__ float hi(float2 v) { return v.y; }
};
template <> struct Pair<__nv_bfloat16> {
    using V = __nv_bfloat162;
    static __device__ __forceinline__ __nv_bfloat162 ld(const __nv_bfloat16* p) {
        return *reinterpret_cast<const __nv_bfloat162*>(p);
    }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float a, float b) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
    }
    static __device__ __forceinline__ float lo(__nv_bfloat162 v) { return __low2float(v); }
    static __device__ __forceinline__ float hi(__nv_bfloat162 v) { return __high2float(v); }
};

constexpr int kRopeTB = 32;

template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(RopeParams q) {
    extern __shared__ float smem[];
    const int N = q.dstate, NH = N / 2, R = q.rank, L = q.seqlen;
    const int b = blockIdx.x / q.nheads, h = blockIdx.x % q.nheads;
    const int G = q.ngroups, H = q.nheads, g = h / (H / G);
    float* sTh = smem;                    // [TB][NH]
    float* sCos = sTh + kRopeTB * NH;     // [TB][NH]
    float* sSin = sCos + kRopeTB * NH;    // [TB][NH]
    float* sDt = sSin + kRopeTB * NH;     // [TB]
    const int tid = threadIdx.x;
    if (!M3_SPAN(1, (sDt - smem) * 4, kRopeTB * 4, dyn_smem_bytes())) return;

    double phi[2] = {0.0, 0.0};           // pairs tid and tid + 256 (N <= 1024)
    for (int t0 = 0; t0 < L; t0 += kRopeTB) {
        const int tb = min(kRopeTB, L - t0);
        for (int e = tid; e < tb * NH; e += blockDim.x) {
            const int k = e / NH, i = e % NH;
            sTh[e] = M3_IN(2, (((size_t)b * L + t0 + k) * G + g) * NH + i, ext_theta(q))
                         ? q.theta[(((size_t)b * L + t0 + k) * G + g) * NH + i] : 0.f;
        }
        for (int k = tid; k < tb; k += blockDim.x)
            sDt[k] = M3_IN(3, ((size_t)b * L + t0 + k) * H + h, ext_tok(q)) ? q.dt[((size_t)b * L + t0 + k) * H + h] : 0.f;
        __syncthreads();
        for (int s = 0; s < 2; ++s) {
            const int i = tid + s * blockDim.x;
            if (i >= NH) break;
            double ph = phi[s];
            for (int k = 0; k < tb; ++k) {
                ph = wrap_pi(ph + (double)sDt[k] * (double)sTh[k * NH + i]);
                float sv, cv;
                sincosf((float)ph, &sv, &cv);
                sCos[k * NH + i] = cv;
                sSin[k * NH + i] = sv;
                if (q.phase && M3_IN(4, (((size_t)b * L + t0 + k) * H + h) * NH + i, rx_phase(q)))
                    q.phase[(((size_t)b * L + t0 + k) * H + h) * NH + i] = (float)ph;
            }
            phi[s] = ph;
        }
        __syncthreads();
        const T* Bin = static_cast<const T*>(q.B);
        const T* Cin = static_cast<const T*>(q.C);
        T* Bo = static_cast<T*>(q.B_rot);
        T* Co = static_cast<T*>(q.C_rot);
        for (int e = tid; e < tb * R * NH; e += blockDim.x) {
            const int i = e % NH, kr = e / NH, r = kr % R, k = kr / R;
            const size_t t = (size_t)b * L + t0 + k;
            const size_t src = ((t * G + g) * R + r) * N + 2 * i;
            const size_t dst = ((t * H + h) * R + r) * N + 2 * i;
            if (!M3_SPAN(5, src, 2, ext_bc(q)) || !M3_SPAN(6, dst, 2, rx_rot(q))) continue;
            const float c = sCos[k * NH + i], s = sSin[k * NH + i];
            const auto bv = Pair<T>::ld(Bin + src);
            const auto cv = Pair<T>::ld(Cin + src);
            const float b0 = Pair<T>::lo(bv), b1 = Pair<T>::hi(bv);
            const float c0 = Pair<T>::lo(cv), c1 = Pair<T>::hi(cv);
            Pair<T>::st(Bo + dst, c * b0 + s * b1, -s * b0 + c * b1);
            Pair<T>::st(Co + dst, c * c0 + s * c1, -s * c0 + c * c1);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Bandwidth-oriented variant for N/2 a multiple of 16 (every layer workload):
// one CTA per (16 rotary pairs, head, batch) walks the sequence in blocks of
// 64 tokens.  The phase of a block is a parallel prefix (thread = pair x
// group of 4 tokens, double precision) from a per-pair carry kept in shared
// memory; cos/sin of every (token, pair) go to shared memory and the block's
// B and C rows are rotated with 16-byte loads and stores.  Many small CTAs
// keep enough loads in flight to stream at HBM rate.
constexpr int kRpPairs = 16;      // rotary pairs per CTA
constexpr int kRpTok = 64;        // tokens per block
constexpr int kRpGrp = 16;        // token groups (4 tokens each)

template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {       // 8 bf16 = 4 pairs
    static constexpr int kPairs = 4;
    static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 v = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&v);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct Vec16<float> {               // 4 floats = 2 pairs
    static constexpr int kPairs = 2;
    static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

// Three CTAs per SM (78 registers): a third more rows in flight per SM than
// at two, measured 1.04 -> 0.93 ms on the R=4 layer (four CTAs spill).
template <typename T>
__global__ void __launch_bounds__(256, 3) rope_block_kernel(RopeParams q) {
    constexpr int VP = Vec16<T>::kPairs;                 // pairs per 16-byte vector
    constexpr int NV = kRpPairs / VP;                    // vectors per row slice
    __shared__ float sTh[kRpTok][kRpPairs];
    __shared__ float sDt[kRpTok];
    __shared__ float2 sCS[kRpTok][kRpPairs];             // (cos, sin)
    __shared__ double sPart[kRpGrp][kRpPairs];
    __shared__ double sCarry[kRpPairs];
    const int N = q.dstate, NH = N / 2, R = q.rank, L = q.seqlen, G = q.ngroups, H = q.nheads;
    const int i0 = blockIdx.x * kRpPairs;                // first pair of this CTA
    const int h = blockIdx.y, b = blockIdx.z, g = h / (H / G);
    const int tid = threadIdx.x;
    const int p = tid % kRpPairs, qg = tid / kRpPairs;   // phase work: pair, token group
    if (tid < kRpPairs) sCarry[tid] = 0.0;
    const T* __restrict__ Bin = static_cast<const T*>(q.B);
    const T* __restrict__ Cin = static_cast<const T*>(q.C);
    T* __restrict__ Bo = static_cast<T*>(q.B_rot);
    T* __restrict__ Co = static_cast<T*>(q.C_rot);
    // theta and dt of a block: 4 theta values and (first 64 threads) one dt per
    // thread, loaded one block ahead into registers (clamped addresses, masked
    // when stored to shared memory)
    constexpr int kThPer = kRpTok * kRpPairs / 256;
    float thr[kThPer], dtr = 0.f;
    auto load_block = [&](int tn) {
        const int tbn = min(kRpTok, L - tn);
#pragma unroll
        for (int j = 0; j < kThPer; ++j) {
            const int e = tid + 256 * j, k = min(e / kRpPairs, tbn - 1), i = e % kRpPairs;
            thr[j] = M3_IN(10, (((size_t)b * L + tn + k) * G + g) * NH + i0 + i, ext_theta(q))
                         ? __ldg(q.theta + (((size_t)b * L + tn + k) * G + g) * NH + i0 + i) : 0.f;
        }
        if (tid < kRpTok)
            dtr = M3_IN(11, ((size_t)b * L + tn + min(tid, tbn - 1)) * H + h, ext_tok(q))
                      ? __ldg(q.dt + ((size_t)b * L + tn + min(tid, tbn - 1)) * H + h) : 0.f;
    };
    load_block(0);
    for (int t0 = 0; t0 < L; t0 += kRpTok) {
        const int tb = min(kRpTok, L - t0);
#pragma unroll
        for (int j = 0; j < kThPer; ++j) {
            const int e = tid + 256 * j, k = e / kRpPairs;
            sTh[k][e % kRpPairs] = k < tb ? thr[j] : 0.f;
        }
        if (tid < kRpTok) sDt[tid] = tid < tb ? dtr : 0.f;
        __syncthreads();
        if (t0 + kRpTok < L) load_block(t0 + kRpTok);
        // phase: partial sums of 4 tokens, prefix over the 16 groups, running phase
        double part = 0.0;
#pragma unroll
        for (int k = 0; k < 4; ++k) part += (double)sDt[4 * qg + k] * (double)sTh[4 * qg + k][p];
        sPart[qg][p] = part;
        __syncthreads();
        double ph = sCarry[p];
        double tot = 0.0;
#pragma unroll
        for (int j = 0; j < kRpGrp; ++j) {
            const double v = sPart[j][p];
            if (j < qg) ph += v;
            tot += v;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int kk = 4 * qg + k;
            ph = wrap_pi(ph + (double)sDt[kk] * (double)sTh[kk][p]);
            float sv, cv;
            sincosf((float)ph, &sv, &cv);
            sCS[kk][p] = make_float2(cv, sv);
            if (q.phase && kk < tb && M3_IN(12, (((size_t)b * L + t0 + kk) * H + h) * NH + i0 + p, rx_phase(q)))
                q.phase[(((size_t)b * L + t0 + kk) * H + h) * NH + i0 + p] = (float)ph;
        }
        __syncthreads();                                 // sCS ready; every thread has read sCarry
        if (qg == 0) sCarry[p] = wrap_pi(sCarry[p] + tot);
        // rotate the block's rows (t, r) of B and C on this CTA's pairs
        // four items per thread per round, all loads issued before any store
        const int items = tb * R * NV;
        for (int e0 = 0; e0 < items; e0 += 4 * 256) {
            uint4 vb[4], vc[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = min(e0 + tid + 256 * u, items - 1);
                const int v = e % NV, kr = e / NV, r = kr % R, k = kr / R;
                const size_t src = ((((size_t)b * L + t0 + k) * G + g) * R + r) * N + 2 * (i0 + v * VP);
                if (!M3_SPAN(13, src, 2 * VP, ext_bc(q))) {
                    vb[u] = vc[u] = make_uint4(0u, 0u, 0u, 0u);
                    continue;
                }
                vb[u] = *reinterpret_cast<const uint4*>(Bin + src);
                vc[u] = *reinterpret_cast<const uint4*>(Cin + src);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + tid + 256 * u;
                if (e >= items) break;
                const int v = e % NV, kr = e / NV, r = kr % R, k = kr / R;
                const size_t dst = ((((size_t)b * L + t0 + k) * H + h) * R + r) * N + 2 * (i0 + v * VP);
                float fb[2 * VP], fc[2 * VP];
                Vec16<T>::unpack(vb[u], fb);
                Vec16<T>::unpack(vc[u], fc);
#pragma unroll
                for (int j = 0; j < VP; ++j) {
                    const float2 cs = sCS[k][v * VP + j];
                    const float b0 = fb[2 * j], b1 = fb[2 * j + 1], c0 = fc[2 * j], c1 = fc[2 * j + 1];
                    fb[2 * j] = cs.x * b0 + cs.y * b1;
                    fb[2 * j + 1] = cs.x * b1 - cs.y * b0;
                    fc[2 * j] = cs.x * c0 + cs.y * c1;
                    fc[2 * j + 1] = cs.x * c1 - cs.y * c0;
                }
                if (!M3_SPAN(14, dst, 2 * VP, rx_rot(q))) continue;
                *reinterpret_cast<uint4*>(Bo + dst) = Vec16<T>::pack(fb);
                *reinterpret_cast<uint4*>(Co + dst) = Vec16<T>::pack(fc);
            }
        }
        __syncthreads();                                 // before the next block overwrites sTh / sCS
    }
}

m3_status launch_rope(const m3_dims& d, const RopeParams& q, cudaStream_t st) {
    if (d.dstate / 2 > 512) return M3_ERR_UNSUPPORTED;
    if (d.batch == 0 || d.seqlen == 0) return M3_OK;
    if ((d.dstate / 2) % kRpPairs == 0) {
        const dim3 grid((unsigned)(d.dstate / 2 / kRpPairs), (unsigned)d.nheads, (unsigned)d.batch);
        if (d.io_dtype == M3_BF16) rope_block_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(q);
        else rope_block_kernel<float><<<grid, 256, 0, st>>>(q);
        return cudaGetLastError() == cudaSuccess ? M3_OK : M3_ERR_CUDA;
    }
    const size_t smem = sizeof(float) * (3 * (size_t)kRopeTB * (d.dstate / 2) + kRopeTB);
    if (smem > 200 * 1024) return M3_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)(d.batch * d.nheads));
    if (d.io_dtype == M3_BF16) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(rope_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        rope_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(q);
    } else {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(rope_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        rope_kernel<float><<<grid, 256, smem, st>>>(q);
    }
    return cudaGetLastError() == cudaSuccess ? M3_OK : M3_ERR_CUDA;
}

}  // namespace m3

M3_BOUNDS_EXPORT(rope)
