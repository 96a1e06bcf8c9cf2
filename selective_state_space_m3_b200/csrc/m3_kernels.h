// m3_kernels.h -- launch parameters and host launchers of the scan, step
// and rope kernels (internal to the library; the public ABI is include/m3.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "m3.h"

namespace m3 {

struct StepParams {
    int batch, nheads, ngroups, headdim, dstate;
    float* h;            // [b][h][n][p] fp32, in/out
    void* prev_B;        // [b][h][r][n] io, in/out
    void* prev_x;        // [b][h][r][p] io, in/out
    const void* x;       // [b][h][r][p] io
    const void* B;       // [b][g][r][n] io
    const void* C;       // [b][g][r][n] io
    const float* dt;     // [b][h]
    const float* A;      // [h]
    const float* lam;    // [b][h]
    const float* theta;  // [b][g][n/2]
    void* y;             // [b][h][r][p] io
};

struct RopeParams {
    int batch, seqlen, nheads, ngroups, dstate, rank;
    const void* B;        // [b][t][g][r][n]
    const void* C;
    const float* dt;      // [b][t][h]
    const float* theta;   // [b][t][g][n/2]
    void* B_rot;          // [b][t][h][r][n]
    void* C_rot;
    float* phase;         // [b][t][h][n/2] or null
};

struct ScanParams {
    int batch, seqlen, nheads, ngroups, headdim, dstate, rank;
    int qs;      // chunk length the kernel uses (tokens)
    int nseg;    // segments per (b, h)
    int cps;     // chunks per segment
    const void* x;
    const void* B;
    const void* C;
    const float* dt;
    const float* A;
    const float* lam;
    const float* theta;
    const float* init_h;
    const void* init_pB;
    const void* init_pX;
    void* y;
    float* fin_h;
    void* fin_pB;
    void* fin_pX;
    float* ws_sloc;    // [b][h][seg][N][P]
    float* ws_decay;   // [b][h][seg]
    float* ws_phase;   // [b][h][seg][N/2]
    float* ws_sin;     // [b][h][seg][N][P]
};

// token-by-token scan of the transition variants (k_seq.cu): damping regimes
// (u == nullptr, regime 0/1/2) and the low-rank reflection (u != nullptr)
struct SeqParams {
    int batch, seqlen, nheads, ngroups, headdim, dstate, rank;
    int regime;          // 0 under, 1 critical, 2 over (ignored with u)
    const void* x;
    const void* B;
    const void* C;
    const void* u;       // [b][t][g][n] io, or null
    const float* dt;
    const float* A;
    const float* lam;
    const float* theta;
    const float* init_h;
    const void* init_pB;
    const void* init_pX;
    void* y;
    float* fin_h;
    void* fin_pB;
    void* fin_pX;
};
bool seq_supported(const m3_dims& d);
cudaError_t launch_seq(const m3_dims& d, const SeqParams& q, cudaStream_t st);

// backward pass (k_bwd.cu); gradients are float32, dB / dC / dtheta / dA
// accumulated with atomics into buffers zeroed by the caller
struct BwdParams {
    int batch, seqlen, nheads, ngroups, headdim, dstate, rank;
    int K;                     // checkpoint interval (tokens)
    const void* x;
    const void* B;
    const void* C;
    const float* dt;
    const float* A;
    const float* lam;
    const float* theta;
    const float* init_h;       // nullable
    const void* init_pB;       // nullable
    const void* init_pX;       // nullable
    const void* dy;            // [b][t][h][r][p] io dtype
    const float* d_fin_h;      // nullable [b][h][n][p]
    const float* d_fin_pB;     // nullable [b][h][r][n]
    const float* d_fin_pX;     // nullable [b][h][r][p]
    float* dx;                 // [b][t][h][r][p]
    float* dB;                 // [b][t][g][r][n]
    float* dC;                 // [b][t][g][r][n]
    float* ddt;                // [b][t][h]
    float* dA;                 // [h]
    float* dlam;               // [b][t][h]
    float* dtheta;             // [b][t][g][n/2]
    float* d_init_h;           // nullable
    float* d_init_pB;          // nullable
    float* d_init_pX;          // nullable
    float* ws_ckpt;            // [b][h][ceil(L/K)][n][p]
    float* ws_scratch;         // [b][h][K][n][p]
};
bool bwd_supported(const m3_dims& d);
int bwd_block_tokens(const m3_dims& d);
cudaError_t launch_bwd(const m3_dims& d, const BwdParams& q, cudaStream_t st);

// phase interventions (k_phase.cu)
cudaError_t launch_theta_transform(int mode, const float* in, const int* perm, const float* freq, float* out,
                                   size_t rows, int G, int NH, cudaStream_t st);
cudaError_t launch_expand_heads(const void* src, void* dst, size_t bt_count, int H, int G, size_t row_bytes,
                                cudaStream_t st);

// SM count of the current device, cached per device (148 if it cannot be queried)
int device_sm_count();

m3_status launch_step(const m3_dims& d, const StepParams& q, cudaStream_t st);
m3_status launch_rope(const m3_dims& d, const RopeParams& q, cudaStream_t st);
size_t simt_smem_bytes(int qs, int R, int N, int P, bool summary);
cudaError_t launch_scan_simt(const m3_dims& d, const ScanParams& q, cudaStream_t st);
cudaError_t launch_scan_combine(const ScanParams& q, cudaStream_t st);
// tensor-core path (bf16, N = 128, P = 64, rank 1/2/4/8); `status` is the
// workspace status word its bounded waits report to
bool tc_eligible(const m3_dims& d);
int tc_tile_tokens(int rank);
cudaError_t launch_scan_tc(const m3_dims& d, const ScanParams& q, int* status, cudaStream_t st);
cudaError_t launch_wait_selftest(int* status, cudaStream_t st);
// the summary pass of the tile kernel only (segments), then the combine
cudaError_t launch_scan_tc_summary(const m3_dims& d, const ScanParams& q, int* status, cudaStream_t st);

// persistent warp-specialised prefill (k_scan_ws.cu): mode 0 cuts the
// concatenated chains of tiles into one range per CTA and hands states from
// a chain's head to its tail (cooperative launch); mode 1 runs one segment
// per CTA with its incoming state from the summary pass
struct WsPlanArgs {
    int mode, nt, M, total, grid, call_id;
    float* ho_state;   // [grid][N][P]
    int* ho_flag;      // [grid]
};
int ws_smem_bytes();
cudaError_t launch_scan_ws(const m3_dims& d, const ScanParams& q, const WsPlanArgs& pa, int* status,
                           cudaStream_t st);

}  // namespace m3
