// m3_bounds.cuh -- index checks of the debug build.
//
// Built with -DM3_DEBUG_BOUNDS=1 (libm3_debug.so), every kernel checks each
// global-memory index it computes against the element count of the buffer
// (as the call's m3_dims gives it) and each shared-memory index against the
// extent of the array or region it addresses, before the access.  A failed
// check skips the access (a load gives zero) and is recorded in the file's
// device-side record: the number of failures, and the site, index and limit
// of the first one.  Nothing traps; m3_debug_bounds_report() collects the
// records of all files.  In the release build the checks are the constant
// true and their arguments are not evaluated, so the kernels are unchanged.
//
// Every file that uses the checks defines M3_BOUNDS_FILE (its number in the
// site codes: site = file * 1000 + check) before including this header and
// ends with M3_BOUNDS_EXPORT(tag), which defines the host-side reader of the
// file's record.  Checks of copies whose addresses the hardware bounds by
// itself (TMA tensor coordinates) only record (M3_NOTE) and never skip, so
// that every expected transaction still arrives.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace m3 {

struct BoundsRecord {
    unsigned int failures;   // failed checks since the record was last cleared
    int site;                // first failure: M3_BOUNDS_FILE * 1000 + check number
    long long index;         // its index (for a span: the last element it reaches)
    long long limit;         // the extent it was checked against
};

}  // namespace m3

#ifndef M3_DEBUG_BOUNDS
#define M3_DEBUG_BOUNDS 0
#endif

#if M3_DEBUG_BOUNDS

#ifndef M3_BOUNDS_FILE
#error "define M3_BOUNDS_FILE before including m3_bounds.cuh"
#endif

namespace m3 {

static __device__ BoundsRecord g_bounds_rec;

static __device__ __noinline__ void bounds_record(int site, long long i, long long n) {
    if (atomicAdd(&g_bounds_rec.failures, 1u) == 0u) {
        g_bounds_rec.site = site;
        g_bounds_rec.index = i;
        g_bounds_rec.limit = n;
    }
}

// 0 <= i < n
__device__ __forceinline__ bool bounds_in(int site, long long i, long long n) {
    if (i >= 0 && i < n) return true;
    bounds_record(site, i, n);
    return false;
}

// elements [i, i + len) all inside [0, n)
__device__ __forceinline__ bool bounds_span(int site, long long i, long long len, long long n) {
    if (i >= 0 && len >= 0 && i + len <= n) return true;
    bounds_record(site, i < 0 ? i : i + len - 1, n);
    return false;
}

}  // namespace m3

#define M3_IN(site, i, n) \
    (::m3::bounds_in(M3_BOUNDS_FILE * 1000 + (site), (long long)(i), (long long)(n)))
#define M3_SPAN(site, i, len, n) \
    (::m3::bounds_span(M3_BOUNDS_FILE * 1000 + (site), (long long)(i), (long long)(len), (long long)(n)))
#define M3_NOTE(site, i, n) ((void)M3_IN(site, i, n))

#define M3_BOUNDS_EXPORT(tag)                                                              \
    namespace m3 {                                                                         \
    cudaError_t bounds_take_##tag(BoundsRecord* out, bool clear) {                          \
        cudaError_t e = cudaMemcpyFromSymbol(out, g_bounds_rec, sizeof(BoundsRecord));       \
        if (e == cudaSuccess && clear) {                                                    \
            const BoundsRecord z = {0u, 0, 0, 0};                                           \
            e = cudaMemcpyToSymbol(g_bounds_rec, &z, sizeof(BoundsRecord));                 \
        }                                                                                  \
        return e;                                                                          \
    }                                                                                      \
    }

#else

#define M3_IN(site, i, n) (true)
#define M3_SPAN(site, i, len, n) (true)
#define M3_NOTE(site, i, n) ((void)0)
#define M3_BOUNDS_EXPORT(tag)

#endif

namespace m3 {

// dynamic shared memory of the running launch, in bytes
__device__ __forceinline__ uint32_t dyn_smem_bytes() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
    return r;
}

// Element counts of a call's buffers (the layouts of include/m3.h), for the
// checks above; Q is any parameter block with the m3_dims fields.
template <class Q> __device__ __forceinline__ long long ext_x(const Q& q) {          // x, y, dy, dx
    return (long long)q.batch * q.seqlen * q.nheads * q.rank * q.headdim;
}
template <class Q> __device__ __forceinline__ long long ext_bc(const Q& q) {         // B, C (and dB, dC)
    return (long long)q.batch * q.seqlen * q.ngroups * q.rank * q.dstate;
}
template <class Q> __device__ __forceinline__ long long ext_tok(const Q& q) {        // dt, lambda
    return (long long)q.batch * q.seqlen * q.nheads;
}
template <class Q> __device__ __forceinline__ long long ext_theta(const Q& q) {      // theta
    return (long long)q.batch * q.seqlen * q.ngroups * (q.dstate / 2);
}
template <class Q> __device__ __forceinline__ long long ext_h(const Q& q) {          // carry h
    return (long long)q.batch * q.nheads * q.dstate * q.headdim;
}
template <class Q> __device__ __forceinline__ long long ext_pB(const Q& q) {         // carry prev_B
    return (long long)q.batch * q.nheads * q.rank * q.dstate;
}
template <class Q> __device__ __forceinline__ long long ext_pX(const Q& q) {         // carry prev_x
    return (long long)q.batch * q.nheads * q.rank * q.headdim;
}

}  // namespace m3
