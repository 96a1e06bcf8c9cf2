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
#include "m3_common.cuh"
#include "m3_kernels.h"

namespace m3 {

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

    double phi[2] = {0.0, 0.0};           // pairs tid and tid + 256 (N <= 1024)
    for (int t0 = 0; t0 < L; t0 += kRopeTB) {
        const int tb = min(kRopeTB, L - t0);
        for (int e = tid; e < tb * NH; e += blockDim.x) {
            const int k = e / NH, i = e % NH;
            sTh[e] = q.theta[(((size_t)b * L + t0 + k) * G + g) * NH + i];
        }
        for (int k = tid; k < tb; k += blockDim.x) sDt[k] = q.dt[((size_t)b * L + t0 + k) * H + h];
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
                if (q.phase) q.phase[(((size_t)b * L + t0 + k) * H + h) * NH + i] = (float)ph;
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

m3_status launch_rope(const m3_dims& d, const RopeParams& q, cudaStream_t st) {
    if (d.dstate / 2 > 512) return M3_ERR_UNSUPPORTED;
    if (d.batch == 0 || d.seqlen == 0) return M3_OK;
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
