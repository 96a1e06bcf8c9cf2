// m3_static.cu -- a prefill entry point that allocates nothing.
//
// Some callers cannot allocate device memory when they run the scan: a
// plugin hosted by an engine that owns every byte of the device and gives
// its plugins no allocator, or a latency-critical loop that is not allowed
// to call into the CUDA allocator once it has started.  m3_scan_fwd needs a
// caller-provided workspace for the segment hand-off of long sequences;
// this variant instead uses one fixed scratch array that lives in the
// library's own device image (a file-scope __device__ array, so it exists on
// every GPU that loads the library, for as long as the process runs).
//
// The array's host-side name is only a stand-in for the device object: its
// device address is looked up once per device with cudaGetSymbolAddress
// while that device is current, cached, and passed to the kernels.  The
// lookup happens on the first call made on each device.
#include <mutex>

#include "m3_common.cuh"
#include "m3_kernels.h"
#include "m3_nvtx.h"

namespace {

// Largest workspace the static variant can serve: the public limit itself.
constexpr size_t kScratchBytes = M3_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_m3_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {nullptr};

// Device address of g_m3_scratch on the current device (looked up once).
m3_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return M3_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_m3_scratch) != cudaSuccess || !p) return M3_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return M3_OK;
}

}  // namespace

extern "C" m3_status m3_static_forget_device(void) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return M3_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    g_addr[dev] = nullptr;
    return M3_OK;
}

extern "C" m3_status m3_scan_fwd_static(const m3_dims* dims, const void* x, const void* B, const void* C,
                                        const float* dt, const float* A, const float* lambda,
                                        const float* theta, const m3_carry* init, void* y,
                                        m3_carry* final_state, void* stream) {
    const m3::NvtxRange range("m3_scan_fwd_static");
    size_t need = 0;
    m3_status s = m3_scan_workspace_size(dims, &need);
    if (s != M3_OK) return s;
    if (need > kScratchBytes) return M3_ERR_WORKSPACE;   // larger than the fixed scratch
    void* ws = nullptr;
    s = scratch_address(&ws);
    if (s != M3_OK) return s;
    // The array keeps whatever the previous call left in it.  Only the status
    // word must start at zero; the segment hand-off area is fully written
    // before it is read within each call.
    if (cudaMemsetAsync(ws, 0, m3::kWorkspaceHeaderBytes, (cudaStream_t)stream) != cudaSuccess)
        return M3_ERR_CUDA;
    return m3_scan_fwd(dims, x, B, C, dt, A, lambda, theta, init, y, final_state, ws, kScratchBytes, stream);
}
