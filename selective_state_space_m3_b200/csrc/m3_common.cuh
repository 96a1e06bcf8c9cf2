// m3_common.cuh -- small device helpers shared by the scan, step and rope
// kernels of the Mamba-3 layer scan (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "m3.h"

namespace m3 {

constexpr double kTwoPi = 6.283185307179586476925286766559;

// Load / store one io element as float (io dtype is float32 or bfloat16).
template <typename T> __device__ __forceinline__ float ld_io(const T* p);
template <> __device__ __forceinline__ float ld_io<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld_io<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st_io(T* p, float v);
template <> __device__ __forceinline__ void st_io<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void st_io<__nv_bfloat16>(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
}

// Reduce an angle (radians, double) to [-pi, pi].  The running cumulative
// phase is kept in double, where the product dt*theta of two float32 values
// is exact and the reduction by a double 2*pi loses nothing that matters at
// float32 output precision.
__device__ __forceinline__ double wrap_pi(double phi) {
    return phi - kTwoPi * rint(phi * (1.0 / kTwoPi));
}

// Reduce a float angle to [-pi, pi] (two-constant additive reduction:
// 2*pi split into a float head and tail so k*2pi is formed exactly enough)
__device__ __forceinline__ float wrap_pi_f(float x) {
    constexpr float kInv2Pi = 0.15915494309189535f;
    constexpr float k2PiHi = 6.28318548202514648f;      // float(2 pi)
    constexpr float k2PiLo = -1.7484555314695172e-7f;   // 2 pi - float(2 pi)
    const float k = rintf(x * kInv2Pi);
    return fmaf(-k, k2PiLo, fmaf(-k, k2PiHi, x));
}

// Status word at the start of a scan workspace.
struct WorkspaceHeader {
    int status;      // m3_status of the last device-side failure, 0 = none
    int where;       // which wait gave up (debug aid)
};
constexpr size_t kWorkspaceHeaderBytes = 256;

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

}  // namespace m3
