// k_phase.cu -- prologue kernels of the phase interventions (sm_100a).
//
// "Understanding Mamba-3 Through Oscillatory Dynamics" (paperlayer.ai
// summary), section 5.3 and appendix D.4: the learned phase increments are
// removed (set to zero), reversed, or shuffled across the rotary pairs of a
// token (the set of increments kept), and, separately, the rotation is kept
// on writing (B) only or on readout (C) only; section 4.3 compares against
// fixed (data-independent) rotations.  Every intervention here is a change
// of the scan's inputs, so the scan kernels themselves are reused:
//   * zero / reverse / shuffle / fixed rewrite theta (theta_transform_kernel);
//   * write-only / read-only run the scan on pre-rotated operands
//     (m3_rope_bc, Proposition 3 of the "Mamba-3" summary, b-lab.team,
//     section 2) with theta = 0, the unrotated side copied per head
//     (expand_heads_kernel).
#define M3_BOUNDS_FILE 7
#include "m3_bounds.cuh"
#include "m3_common.cuh"
#include "m3_kernels.h"

namespace m3 {

// out[b][t][g][i] from in[b][t][g][:] by mode; perm [N/2] and freq [G][N/2]
// are device copies of host arrays the API has validated.
__global__ void theta_transform_kernel(int mode, const float* __restrict__ in, const int* __restrict__ perm,
                                       const float* __restrict__ freq, float* __restrict__ out, size_t rows, int G,
                                       int NH) {
    const size_t n = rows * (size_t)NH;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const size_t row = e / NH;
        const int i = (int)(e % NH);
        float v = 0.f;
        switch (mode) {
            case M3_PHASE_ZERO: v = 0.f; break;
            case M3_PHASE_REVERSE: v = -in[e]; break;
            case M3_PHASE_SHUFFLE:
                // perm holds NH indices the host checked to be a permutation of [0, NH)
                if (M3_IN(1, perm[i], NH)) v = in[row * NH + perm[i]];
                break;
            case M3_PHASE_FIXED: v = freq[(row % G) * NH + i]; break;
            default: v = in[e]; break;
        }
        out[e] = v;
    }
}

// dst[b][t][h][:] = src[b][t][g(h)][:], rows of `row_bytes` (a multiple of 16).
__global__ void expand_heads_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t bt_count, int H,
                                    int G, int row_units) {
    const size_t n = bt_count * (size_t)H * row_units;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const int u = (int)(e % row_units);
        const size_t rest = e / row_units;
        const int h = (int)(rest % H);
        const size_t bt = rest / H;
        const int g = h / (H / G);
        if (M3_IN(2, (bt * G + g) * row_units + u, bt_count * (size_t)G * row_units))
            dst[e] = src[(bt * G + g) * row_units + u];
    }
}

static unsigned grid_for(size_t n) {
    size_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return (unsigned)(blocks ? blocks : 1);
}

cudaError_t launch_theta_transform(int mode, const float* in, const int* perm, const float* freq, float* out,
                                   size_t rows, int G, int NH, cudaStream_t st) {
    const size_t n = rows * (size_t)NH;
    if (n == 0) return cudaSuccess;
    theta_transform_kernel<<<grid_for(n), 256, 0, st>>>(mode, in, perm, freq, out, rows, G, NH);
    return cudaGetLastError();
}

cudaError_t launch_expand_heads(const void* src, void* dst, size_t bt_count, int H, int G, size_t row_bytes,
                                cudaStream_t st) {
    const size_t n = bt_count * (size_t)H * (row_bytes / 16);
    if (n == 0) return cudaSuccess;
    expand_heads_kernel<<<grid_for(n), 256, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                                     bt_count, H, G, (int)(row_bytes / 16));
    return cudaGetLastError();
}

}  // namespace m3

M3_BOUNDS_EXPORT(phase)
