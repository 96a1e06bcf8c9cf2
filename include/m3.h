/*
 * m3.h -- C ABI of the B200 (sm_100a) Mamba-3 SSM layer scan.
 *
 * The operation.  Per batch b and head h (group g = h / (nheads/ngroups)), a
 * state h_t in R^{N x P} follows the exponential-trapezoidal recurrence with
 * data-dependent rotations and MIMO rank-R inputs:
 *
 *   alpha_t = exp(dt_t A_h),  beta_t = (1 - lambda_t) dt_t exp(dt_t A_h),
 *   gamma_t = lambda_t dt_t
 *       ("Mamba-3" summary, b-lab.team, section 1 "Exponential-Trapezoidal
 *        Discretization", the recurrence and the definitions below it)
 *   R_t = blockdiag_i R(dt_t theta_t[i]),  R(phi) = [[cos phi, -sin phi],
 *                                                    [sin phi,  cos phi]]
 *       (same page, section 2 "Complex-Valued State Space Model",
 *        Proposition 2)
 *   h_t = R_t (alpha_t h_{t-1} + beta_t B_{t-1} X_{t-1}^T) + gamma_t B_t X_t^T
 *   y_t = C_t^T h_t                         (R x P per head; section 3 "MIMO")
 *
 * The rotation applied to the beta term is this library's reading of the
 * pages (they print the trapezoid and the rotation separately); it is the
 * reading under which Proposition 3 -- the rotation moved onto B and C as a
 * cumulative phase -- holds, and the prefill kernels rely on it.
 *
 * Layouts (C order, innermost index last; every tensor densely packed):
 *   x, y    [batch][seqlen][nheads][rank][headdim]     io dtype
 *   B, C    [batch][seqlen][ngroups][rank][dstate]     io dtype
 *   dt, lambda [batch][seqlen][nheads]                 float32
 *   A       [nheads]                                   float32
 *   theta   [batch][seqlen][ngroups][dstate/2]         float32
 *   carry:  h      [batch][nheads][dstate][headdim]    float32
 *           prev_B [batch][nheads][rank][dstate]       io dtype
 *           prev_x [batch][nheads][rank][headdim]      io dtype
 * Rotary pair i is state rows (2i, 2i+1) (interleaved).  Heads of one group
 * share B, C and theta; dt, lambda and A are per head.  The io dtype is
 * float32 or bfloat16; arithmetic is float32 (tensor-core products take
 * bfloat16 operands with float32 accumulation on the bfloat16 path).
 *
 * Ownership and threading.  Every pointer is a device pointer owned by the
 * caller (except the size outputs of the *_workspace_size calls, the
 * dims/carry structs and m3_scan_fwd_phase's perm / freq arrays, which are
 * host memory read during the call).  The library allocates no
 * device memory, keeps no state between calls apart from cached device
 * attributes, and never synchronises the stream except in m3_device_status
 * and in m3_scan_fwd_phase's copy of its host arrays (SHUFFLE / FIXED modes:
 * a copy from pageable host memory may wait for the stream).
 * Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 * stream).  Calls on different streams are independent if they share no
 * buffers.  Device pointers must be 16-byte aligned.
 *
 * Errors.  Argument, shape and alignment checks run on the host before any
 * launch and return M3_ERR_INVALID_ARG / M3_ERR_UNSUPPORTED / M3_ERR_WORKSPACE
 * with nothing enqueued.  A failed launch returns M3_ERR_CUDA.  Kernels that
 * wait on on-chip barriers bound every wait; on expiry they record
 * M3_ERR_DEVICE_TIMEOUT in the workspace's status word and return early,
 * which m3_device_status reports.  No C++ exception crosses this boundary.
 * Environment (testing and tuning only; unset in normal use).  Three
 * variables change the prefill's launch plan and are read on every plan, so
 * a workspace-size query and the call it serves must see the same values:
 * M3_SCAN_PATH=simt sends the prefill (m3_scan_fwd and the calls built on it)
 * to the float32 SIMT kernels even where the tensor-core path applies;
 * M3_SCAN_NSEG=n (n >= 1) cuts each sequence into n segments (at most one per
 * chunk) instead of the planner's choice; M3_TC_KERNEL=persistent runs the
 * tensor-core prefill on the persistent warp-specialised kernel (one CTA per
 * SM, tiles pipelined across roles) instead of the default tile kernel.
 * M3_SEQ_COLS=1|2 runs the transition variants with 1 or 2 state columns per
 * warp instead of 4 (for comparison; measured slower).
 * Buffer extents cannot be checked through plain pointers: every buffer must
 * hold at least the elements its layout gives for `dims` (nothing is read
 * from a buffer whose extent for `dims` is zero); a smaller buffer is read or
 * written out of bounds.
 */
#ifndef M3_H_
#define M3_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum m3_status {
    M3_OK = 0,
    M3_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misaligned pointer */
    M3_ERR_UNSUPPORTED = 2,     /* valid but outside what the kernels handle  */
    M3_ERR_WORKSPACE = 3,       /* workspace missing or smaller than required */
    M3_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed       */
    M3_ERR_DEVICE_TIMEOUT = 5   /* a kernel's bounded on-chip wait expired    */
} m3_status;

typedef enum m3_dtype { M3_F32 = 0, M3_BF16 = 1 } m3_dtype;

typedef struct m3_dims {
    int batch;      /* >= 0 (0 = nothing to do)                               */
    int seqlen;     /* L >= 0 for m3_scan_fwd / m3_rope_bc; ignored by m3_step */
    int nheads;     /* H >= 1                                                  */
    int ngroups;    /* G >= 1, H % G == 0                                      */
    int headdim;    /* P >= 1                                                  */
    int dstate;     /* N >= 2, even (N/2 rotary pairs)                         */
    int rank;       /* R >= 1 (1 = SISO)                                       */
    int chunk;      /* Q >= 1: chunk length of the chunked prefill on the
                     * float32 SIMT path (shortened to fit shared memory);
                     * the tcgen05 path ignores it and uses chunks of 128/R
                     * tokens (one 128-row tile).  The result is the same
                     * recurrence either way; m3_scan_plan reports the
                     * chunk actually used.                                   */
    int io_dtype;   /* m3_dtype of x, B, C, y, prev_B, prev_x                  */
} m3_dims;

/* The recurrent carry between calls: the state and the previous token's
 * (B, x), which the next token's beta term needs.  In m3_scan_fwd's `init`
 * any member may be NULL (read as zeros); in its `final_state` any member may
 * be NULL (not written).  m3_step needs all three. */
typedef struct m3_carry {
    float* h;
    void* prev_B;
    void* prev_x;
} m3_carry;

/* Bytes of device workspace m3_scan_fwd needs for `dims` (0 is never
 * returned: the first 256 bytes hold the status word).  Host-only. */
m3_status m3_scan_workspace_size(const m3_dims* dims, size_t* bytes);

/* Chunked prefill over a whole sequence.
 * Computes y_t for t = 0..L-1 from the recurrence above, starting from
 * `init` (h_{-1}, B_{-1}, x_{-1}; NULL = zeros), and writes the carry after
 * the last token into `final_state` (h_{L-1}, B_{L-1}, x_{L-1}) if given.
 * The chunked form follows the pages' state-space-duality view: inside a
 * chunk the output is the product of the two-band masked matrix with X
 * ("Mamba-3" summary, section 1, last paragraph: a decay mask times a
 * two-band matrix), across chunks the state is passed on; with B and C
 * rotated by their cumulative phase (section 2, Proposition 3) the rotation
 * leaves the state recurrence.  `final_state` may alias `init`.
 * `workspace` is device memory of at least m3_scan_workspace_size bytes,
 * owned by the caller and zero-filled once before its first use (its first
 * 256 bytes hold the status word that m3_device_status reads and clears);
 * calls that share a workspace must not overlap on the device. */
m3_status m3_scan_fwd(const m3_dims* dims,
                      const void* x, const void* B, const void* C,
                      const float* dt, const float* A, const float* lambda,
                      const float* theta,
                      const m3_carry* init,
                      void* y, m3_carry* final_state,
                      void* workspace, size_t workspace_bytes,
                      void* stream);

/* One decode token with carried state (the recurrence above for a single t).
 * Per-token layouts drop the seqlen axis: x, y [batch][nheads][rank][headdim];
 * B, C [batch][ngroups][rank][dstate]; dt, lambda [batch][nheads];
 * theta [batch][ngroups][dstate/2].  `state` is read and updated in place
 * (h, prev_B, prev_x all required).  dims->seqlen and dims->chunk are
 * ignored.  No workspace: this kernel has no on-chip waits. */
m3_status m3_step(const m3_dims* dims, m3_carry* state,
                  const void* x, const void* B, const void* C,
                  const float* dt, const float* A, const float* lambda,
                  const float* theta, void* y, void* stream);

/* Cumulative phase and rotated B, C ("Mamba-3" summary, section 2,
 * Proposition 3, the "RoPE trick"):
 *   Phi_t[i] = sum_{s <= t} dt_s theta_s[i]   (per head: dt is per head)
 *   (B~_{2i}, B~_{2i+1}) = R(Phi_t[i])^T (B_{2i}, B_{2i+1}), same for C.
 * Outputs B_rot, C_rot [batch][seqlen][nheads][rank][dstate] in the io dtype;
 * `phase` [batch][seqlen][nheads][dstate/2] float32, reduced to [-pi, pi]
 * (may be NULL).  dims->headdim and dims->chunk are ignored. */
m3_status m3_rope_bc(const m3_dims* dims,
                     const void* B, const void* C,
                     const float* dt, const float* theta,
                     void* B_rot, void* C_rot, float* phase,
                     void* stream);

/* Gradients arriving at, or leaving through, a carry (m3_scan_bwd).  All
 * float32: h [b][h][n][p], prev_B [b][h][r][n], prev_x [b][h][r][p]; any
 * member may be NULL (absent). */
typedef struct m3_grad_carry {
    float* h;
    float* prev_B;
    float* prev_x;
} m3_grad_carry;

/* Bytes of device workspace m3_scan_bwd needs for `dims` (host-only): a
 * 256-byte header, the state checkpoints (one N x P float32 state per block
 * of up to 16 tokens per (b, h)) and a per-(b, h) scratch of one block's
 * states. */
m3_status m3_scan_bwd_workspace_size(const m3_dims* dims, size_t* bytes);

/* Backward pass of m3_scan_fwd: the gradient of
 *   J = sum_t <dy_t, y_t> + <d_final.h, h_{L-1}> + <d_final.prev_B, B_{L-1}>
 *       + <d_final.prev_x, x_{L-1}>
 * with respect to every input, by reverse mode of the same recurrence
 * ("Mamba-3" summary, b-lab.team, sections 1-3; the chain rule written out
 * in k_bwd.cu).  Inputs as in m3_scan_fwd (same layouts, same `init`), plus
 * dy ([b][t][h][r][p], io dtype) and d_final (nullable; members nullable).
 * Outputs, all float32 and all overwritten: dx [b][t][h][r][p]; dB, dC
 * [b][t][g][r][n] (summed over the heads of each group); ddt, dlambda
 * [b][t][h]; dA [h] (summed over batch and tokens); dtheta [b][t][g][N/2]
 * (summed over the heads of each group); d_init (nullable; members
 * nullable): the gradient of the carry-in.
 * Supported shapes: headdim 16, 32 or 64; rank 1..4; (N/2) * (P/16) <= 256.
 * Others return M3_ERR_UNSUPPORTED.  Pointers 16-byte aligned.  The library
 * zeroes the accumulated outputs on `stream` itself; all work is
 * asynchronous on `stream`. */
m3_status m3_scan_bwd(const m3_dims* dims,
                      const void* x, const void* B, const void* C,
                      const float* dt, const float* A, const float* lambda,
                      const float* theta, const m3_carry* init,
                      const void* dy, const m3_grad_carry* d_final,
                      float* dx, float* dB, float* dC, float* ddt, float* dA,
                      float* dlambda, float* dtheta, m3_grad_carry* d_init,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Phase interventions ("Understanding Mamba-3 Through Oscillatory Dynamics",
 * section 5.3 and appendix D.4; fixed rotations, section 4.3).  The first
 * five rewrite theta before the scan; the last two keep the rotation on one
 * side of the state only, in the form of Proposition 3 ("Mamba-3" summary,
 * b-lab.team, section 2):  y_t = C'_t^T h'_t with h' the theta = 0 recurrence
 * driven by B', where B' = B~ (rotated by the cumulative phase) or B, and
 * C' = C~ or C. */
typedef enum m3_phase_mode {
    M3_PHASE_NATIVE = 0,      /* theta as given                                   */
    M3_PHASE_ZERO = 1,        /* theta := 0 (no rotation)                         */
    M3_PHASE_REVERSE = 2,     /* theta := -theta                                  */
    M3_PHASE_SHUFFLE = 3,     /* theta_t[i] := theta_t[perm[i]], every token      */
    M3_PHASE_FIXED = 4,       /* theta_t[i] := freq[g][i], the same every token   */
    M3_PHASE_WRITE_ONLY = 5,  /* rotation on writing (B~), none on readout (C)    */
    M3_PHASE_READ_ONLY = 6    /* rotation on readout (C~), none on writing (B)    */
} m3_phase_mode;

/* Bytes of device workspace m3_scan_fwd_phase needs (host-only). */
m3_status m3_scan_phase_workspace_size(const m3_dims* dims, int mode, size_t* bytes);

/* m3_scan_fwd under a phase intervention.  Arguments as m3_scan_fwd, plus:
 *   mode  an m3_phase_mode;
 *   perm  (SHUFFLE) HOST array of N/2 int32, a permutation of 0..N/2-1
 *         (checked; M3_ERR_INVALID_ARG otherwise); NULL for other modes;
 *   freq  (FIXED) HOST array [G][N/2] of float32 phase increments per unit
 *         dt; NULL for other modes.
 * Both are copied into the workspace on `stream`.  For ZERO, REVERSE,
 * SHUFFLE and FIXED the carry (init / final_state) means what it means for
 * m3_scan_fwd.  For WRITE_ONLY and READ_ONLY the state is that of the
 * theta = 0 recurrence on (B', C'), i.e. the rotated frame of Proposition 3
 * without the final rotation back, and `init` is read in that frame.  The
 * device status word is the workspace's first 256 bytes, as for m3_scan_fwd. */
m3_status m3_scan_fwd_phase(const m3_dims* dims, int mode, const int* perm, const float* freq,
                            const void* x, const void* B, const void* C,
                            const float* dt, const float* A, const float* lambda,
                            const float* theta, const m3_carry* init, void* y,
                            m3_carry* final_state, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Damping-regime variants ("Understanding Mamba-3 Through Oscillatory
 * Dynamics", section 2.2 and Table 1, section 4.1, section 4.2, appendix
 * C.2).  Rotary pair i of token t evolves over its interval under the
 * generator dt_t (A_h I + theta_t[i] K_s), K_s = [[0, -1], [s, 0]], so the
 * eigenvalue pair is centred on A_h in every regime:
 *   M3_DAMP_UNDER     s = +1: block R(phi) (Mamba-3 itself),
 *   M3_DAMP_CRITICAL  s =  0: block [[1, -phi], [0, 1]] (a shear),
 *   M3_DAMP_OVER      s = -1: block [[cosh phi, -sinh phi], [-sinh phi, cosh phi]],
 * phi = dt_t theta_t[i]; the exponential-trapezoidal input rule and the
 * readout are unchanged:
 *   h_t = T_t (alpha_t h_{t-1} + beta_t B_{t-1} X_{t-1}^T) + gamma_t B_t X_t^T,
 *   y_t = C_t^T h_t.
 * (This library's reading: the pages name the regimes and fix the shared
 * centre, the state structure and the input rule, not the block itself.) */
typedef enum m3_damping {
    M3_DAMP_UNDER = 0,
    M3_DAMP_CRITICAL = 1,
    M3_DAMP_OVER = 2
} m3_damping;

/* The scan under a damping regime.  Arguments, layouts, carry and results as
 * m3_scan_fwd (the carry's h is in the original frame), plus `regime` (an
 * m3_damping); no workspace.  The recurrence runs token by token in float32
 * (the chunked form of m3_scan_fwd needs the inverse of every prefix of
 * transitions, which grows like e^{|Phi|} or |Phi| outside the underdamped
 * regime).  Overdamped pairs grow like e^{dt (A + |theta|)}: inputs with
 * |theta| > |A| leave the regime and make the state grow.  Supported shapes:
 * rank 1, 2 or 4; dstate a multiple of 8 and at most 256; headdim a multiple
 * of 16; others return M3_ERR_UNSUPPORTED.  dims->chunk is ignored. */
m3_status m3_scan_fwd_damped(const m3_dims* dims, int regime,
                             const void* x, const void* B, const void* C,
                             const float* dt, const float* A, const float* lambda,
                             const float* theta, const m3_carry* init,
                             void* y, m3_carry* final_state, void* stream);

/* Low-rank reflection extension (the extension's abstract listed on
 * "Understanding Mamba-3 Through Oscillatory Dynamics": an input-dependent
 * rank-one reflection added to Mamba-3's diagonal transition, keeping the
 * exponential-trapezoidal rule, RoPE and the readout; appendix C.4 of that
 * paper: two reflections compose to a rotation).  Reading:
 *   h_t = R_t H_t (alpha_t h_{t-1} + beta_t B_{t-1} X_{t-1}^T) + gamma_t B_t X_t^T,
 *   H_t = I - 2 u_t u_t^T / (u_t^T u_t),   H_t = I where u_t = 0,
 * with u_t [batch][seqlen][ngroups][dstate] in the io dtype (per token and
 * group, like B; only its direction matters; required, like the other
 * inputs, whenever there are tokens).  Everything else as
 * m3_scan_fwd_damped (token by token, float32, no workspace, same shapes). */
m3_status m3_scan_fwd_reflect(const m3_dims* dims, const void* u,
                              const void* x, const void* B, const void* C,
                              const float* dt, const float* A, const float* lambda,
                              const float* theta, const m3_carry* init,
                              void* y, m3_carry* final_state, void* stream);

/* How m3_scan_fwd will run `dims` (host-only, nothing launched): the number
 * of kernel launches one call makes, the segments each (batch, head)
 * sequence is cut into, the chunk length the kernels use, and the path
 * (0 = SIMT float32, 1 = tcgen05 tensor cores).  Any output may be NULL. */
m3_status m3_scan_plan(const m3_dims* dims, int* launches, int* segments,
                       int* chunk_used, int* path);

/* Waits for `stream`, then reads and clears the status word at the start of
 * a workspace used by m3_scan_fwd: M3_OK, or M3_ERR_DEVICE_TIMEOUT if a
 * bounded on-chip wait expired (that call's outputs are then invalid). */
m3_status m3_device_status(void* workspace, void* stream);

/* Diagnostic for the failure path: launches one small kernel whose single
 * on-chip wait (the same bounded wait the prefill kernels use) is never
 * satisfied, so it gives up after its limit (about 1 s) and records
 * M3_ERR_DEVICE_TIMEOUT in the workspace status word, which
 * m3_device_status then returns.  Nothing faults and the context stays
 * usable.  `workspace` needs at least 256 bytes. */
m3_status m3_selftest_bounded_wait(void* workspace, size_t workspace_bytes, void* stream);

/* Index checks of the debug build.  The library compiled with
 * -DM3_DEBUG_BOUNDS=1 (libm3_debug.so beside libm3.so) checks, in every
 * kernel, each global-memory index against the element count that `dims`
 * gives the buffer and each shared-memory index against the array or
 * region it addresses, before the access.  A failed check skips the access
 * (a load reads zero) and is counted in a device-side record; nothing traps
 * and the context stays usable.  The release build (libm3.so) has no checks
 * and its kernels are unchanged by them.
 *
 * m3_debug_bounds_report synchronises the device, then fills `out`:
 * enabled = 1 in the debug build (0 otherwise, with everything else zero),
 * failures = failed checks since the last clear, and site / index / limit of
 * the first failure recorded by the lowest-numbered source file that has one
 * (site = file * 1000 + check: 1 tile prefill, 2 SIMT prefill and segment
 * combine, 3 decode step, 4 rope, 5 transition variants, 6 backward,
 * 7 phase prologues, 8 persistent prefill, 9 this self-test; for a span the
 * index is its last element).  `clear` != 0 resets the records after reading.
 * M3_ERR_INVALID_ARG for a NULL `out`, M3_ERR_CUDA if the device cannot be
 * read.  Host call; the release build touches no device. */
typedef struct m3_bounds_report {
    int enabled;
    unsigned int failures;
    int site;
    long long index;
    long long limit;
} m3_bounds_report;
m3_status m3_debug_bounds_report(m3_bounds_report* out, int clear);

/* Diagnostic for the checks themselves (debug build only; the release build
 * returns M3_ERR_UNSUPPORTED and launches nothing): one thread writes 1.0f to
 * buffer[index] if the check index < limit passes.  The host requires
 * 0 <= index < capacity and 0 <= limit <= capacity (M3_ERR_INVALID_ARG
 * otherwise), so with index >= limit the check fails, the store is skipped
 * and the failure is recorded as site 9001 -- and even a store that were not
 * skipped would stay inside the caller's `capacity` floats.  `buffer` is a
 * device pointer to `capacity` floats; enqueued on `stream`. */
m3_status m3_selftest_bounds_check(float* buffer, long long capacity, long long index, long long limit,
                                   void* stream);

/* Prefill that allocates nothing and takes no workspace.
 * The paper has no counterpart to this call: it exists for callers that
 * cannot allocate device memory while they run -- for example a plugin
 * hosted by an engine that owns all device memory and gives its plugins no
 * allocator, or a latency-critical loop that must not enter the CUDA
 * allocator after start-up -- and so cannot provide m3_scan_fwd's workspace.
 * Same arguments and results as m3_scan_fwd minus the workspace.  The
 * scratch it needs lives in one fixed array of M3_STATIC_SCRATCH_BYTES
 * inside the library's device image; every GPU that loads the library holds
 * that array until the process exits.  Sizes whose workspace
 * (m3_scan_workspace_size) exceeds it return M3_ERR_WORKSPACE before any
 * launch.  The call itself allocates nothing (no cudaMalloc, no cudaFree).
 * The first call on each device looks up the array's device address with
 * that device current and caches it; make that first call before any stream
 * capture.  The cached address belongs to the device's primary context:
 * after cudaDeviceReset it is stale, so call m3_static_forget_device with
 * that device current before the next m3_scan_fwd_static on it.  All calls share the one array and it keeps the last call's
 * contents (each call clears the status word it needs zeroed), so calls that
 * overlap on the GPU -- on different streams, or on different host threads --
 * race and must be serialised by the caller.  On-chip wait timeouts are
 * recorded in the array's status word but not reported through this call;
 * callers that need that report use m3_scan_fwd. */
#define M3_STATIC_SCRATCH_BYTES (32u << 20)
m3_status m3_scan_fwd_static(const m3_dims* dims,
                             const void* x, const void* B, const void* C,
                             const float* dt, const float* A, const float* lambda,
                             const float* theta,
                             const m3_carry* init,
                             void* y, m3_carry* final_state,
                             void* stream);

/* Drops the cached device address of the static scratch array for the
 * current device (needed only after cudaDeviceReset: the next
 * m3_scan_fwd_static looks it up again).  Must not overlap a running
 * m3_scan_fwd_static on that device.  Host-only; M3_ERR_CUDA if no device
 * is current. */
m3_status m3_static_forget_device(void);

/* Static, never NULL. */
const char* m3_status_string(m3_status status);

#ifdef __cplusplus
}
#endif

#endif /* M3_H_ */
