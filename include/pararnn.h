/*
 * pararnn.h - C ABI of the B200 (sm_100a) ParaRNN Newton-solve library
 * (libpararnn.so).
 *
 * The library solves a whole nonlinear diagonal RNN recurrence in parallel
 * over the sequence axis, the method of the page
 *   "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
 *    pra 7B parâmetros" (cafecomtech.com, 2026-04-23):
 *   - section "O compromisso que SSMs fizeram": the classic RNN applies
 *     h_l = sigma(h_{l-1}, x_l) one step at a time; a linear SSM
 *     h_l = A_l h_{l-1} + B_l x_l can instead be combined as a parallel
 *     (associative) scan;
 *   - section "A sacada: método de Newton": the whole sequence is one system
 *     of equations whose unknowns are all hidden states; Newton linearises it
 *     with the Jacobians, which take the place of A_l, so each iteration is a
 *     linear SSM solved by a parallel scan;
 *   - section "Engenharia pra escalar": with diagonal matrices in the cell
 *     the Jacobian is diagonal (ParaGRU) or 2x2 block-diagonal per channel
 *     over (c, h) (ParaLSTM), and Newton iterations, system assembly and
 *     the parallel reduction run fused in one kernel.
 *
 * Cells (per channel d; s = logistic; the pages state only that the cell's
 * matrices are diagonal, these are the diagonal GRU / LSTM):
 *   GRU : z = s(u_z + a_z h), r = s(u_r + a_r h), c = tanh(u_c + a_c r h),
 *         h' = (1 - z) h + z c                       gates u = (z, r, c)
 *   LSTM: i = s(u_i + a_i h), f = s(u_f + a_f h), o = s(u_o + a_o h),
 *         g = tanh(u_g + a_g h), c' = f c + i g, h' = o tanh(c')
 *                                                    gates u = (i, f, o, g)
 *
 * Newton solve (reading of the pages, which leave these open):
 *   unknowns H = (h_1..h_L) (and c_1..c_L), F_l(H) = state_l - cell(state_{l-1}, u_l);
 *   initial guess H^0 = 0; r_k = max |F(H^k)| over all b, l, d and both LSTM
 *   components; stop at the first k with r_k <= tol, or at k = max_iters;
 *   iters = number of Newton updates in the returned states, residual = r of
 *   the returned states.  Newton update: delta_l = J_l delta_{l-1} - F_l,
 *   delta_0 = 0, H^{k+1} = H^k + delta, with J_l = d cell / d state_{l-1}
 *   at H^k.
 *
 * Conventions for every entry point:
 *   - Layouts are row-major with D fastest: u [B][L][G][D] (G = 3 or 4),
 *     a [G][D], h0/c0 [B][D], states and gradients [B][L][D].
 *   - All array pointers are DEVICE pointers, 16-byte aligned, owned by the
 *     caller.  The library never allocates device memory; scratch space is
 *     the caller's `workspace` (size from the *_workspace_size query,
 *     256-byte aligned).  Inputs are never modified; outputs are fully
 *     overwritten.
 *   - B, L, D >= 1; D must be a multiple of 8 (else PARARNN_ERR_UNSUPPORTED);
 *     B*L*D*4 bytes must fit in 2^40.  Violations return an error before any
 *     work is queued.  Errors never abort the process; details are in
 *     pararnn_last_error() (thread-local).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream) of the
 *     current device.  Work is queued on it.
 *   - Every wait inside the kernels is bounded (about 2 s); a wait that runs
 *     out makes the call report PARARNN_ERR_TIMEOUT instead of hanging.
 */
#ifndef PARARNN_H
#define PARARNN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PARARNN_API __attribute__((visibility("default")))
#else
#define PARARNN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PARARNN_OK = 0,
    PARARNN_NOT_CONVERGED = 1,     /* warning: outputs valid, residual > tol  */
    PARARNN_ERR_INVALID_ARG = -1,  /* bad pointer, size, tolerance, ...      */
    PARARNN_ERR_WORKSPACE = -2,    /* workspace missing or too small         */
    PARARNN_ERR_CUDA = -3,         /* a CUDA runtime call failed             */
    PARARNN_ERR_TIMEOUT = -4,      /* a bounded device-side wait ran out     */
    PARARNN_ERR_NONFINITE = -5,    /* residual is NaN or inf                 */
    PARARNN_ERR_UNSUPPORTED = -6   /* e.g. D not a multiple of 8             */
} pararnn_status;

typedef enum { PARARNN_F32 = 0, PARARNN_BF16 = 1 } pararnn_dtype;

/* ABI-identical to cudaStream_t. */
typedef struct CUstream_st* pararnn_stream_t;

/* Outcome of the last solve / adjoint run on a workspace (see
 * pararnn_read_result). */
typedef struct {
    int32_t status;    /* pararnn_status                                    */
    int32_t iters;     /* Newton updates applied to the returned states     */
    float residual;    /* max |F| of the returned states                    */
    float residual0;   /* max |F| of the initial guess H^0 = 0              */
} pararnn_result;

/* ----------------------------------------------------------- workspaces */

/* Bytes of device workspace needed by the solves and adjoints for a given
 * shape.  0 means the shape is invalid. */
PARARNN_API size_t pararnn_gru_workspace_size(int64_t B, int64_t L, int64_t D);
PARARNN_API size_t pararnn_lstm_workspace_size(int64_t B, int64_t L, int64_t D);
PARARNN_API size_t pararnn_gru_adjoint_workspace_size(int64_t B, int64_t L, int64_t D);
PARARNN_API size_t pararnn_lstm_adjoint_workspace_size(int64_t B, int64_t L, int64_t D);

/* ---------------------------------------------------------------- solves */

/* ParaGRU Newton solve ("A sacada: método de Newton"; diagonal Jacobian,
 * "Engenharia pra escalar").  One cooperative kernel runs every Newton
 * iteration: per iteration it evaluates the cell, its Jacobian and the
 * residual at every (b, l, d), scans the affine maps (A_l, -F_l) over l,
 * updates the states in place, and re-evaluates the residual of the new
 * states to decide convergence on the device.
 *   u        [B][L][3][D] gate pre-activations (z, r, c), dtype u_dtype
 *   a        [3][D] fp32 diagonal recurrence weights (a_z, a_r, a_c)
 *   h0       [B][D] fp32 initial state, or NULL for zeros
 *   h        [B][L][D] fp32 output h_1..h_L
 *   tol      >= 0, finite; max_iters >= 0
 *   iters_out, residual_out: host pointers (may be NULL)
 * Synchronous: returns after the stream has finished the solve.  Returns
 * PARARNN_OK, PARARNN_NOT_CONVERGED (last iterate and its residual are
 * returned), PARARNN_ERR_NONFINITE, or an error. */
PARARNN_API pararnn_status pararnn_gru_solve(const void* u, pararnn_dtype u_dtype, const float* a,
                                 const float* h0, float* h, int64_t B, int64_t L, int64_t D,
                                 float tol, int max_iters, void* workspace,
                                 size_t workspace_bytes, pararnn_stream_t stream,
                                 int* iters_out, float* residual_out);

/* Same as pararnn_gru_solve but only queues the work on `stream`; the outcome
 * stays in the workspace until pararnn_read_result. */
PARARNN_API pararnn_status pararnn_gru_solve_async(const void* u, pararnn_dtype u_dtype, const float* a,
                                       const float* h0, float* h, int64_t B, int64_t L,
                                       int64_t D, float tol, int max_iters, void* workspace,
                                       size_t workspace_bytes, pararnn_stream_t stream);

/* ParaLSTM Newton solve over the per-channel state (c, h) with the 2x2
 * block-diagonal Jacobian ("Engenharia pra escalar").
 *   u [B][L][4][D] gates (i, f, o, g); a [4][D]; c0, h0 [B][D] or NULL;
 *   c, h [B][L][D] outputs.  Otherwise as pararnn_gru_solve. */
PARARNN_API pararnn_status pararnn_lstm_solve(const void* u, pararnn_dtype u_dtype, const float* a,
                                  const float* c0, const float* h0, float* c, float* h,
                                  int64_t B, int64_t L, int64_t D, float tol, int max_iters,
                                  void* workspace, size_t workspace_bytes,
                                  pararnn_stream_t stream, int* iters_out, float* residual_out);

PARARNN_API pararnn_status pararnn_lstm_solve_async(const void* u, pararnn_dtype u_dtype, const float* a,
                                        const float* c0, const float* h0, float* c, float* h,
                                        int64_t B, int64_t L, int64_t D, float tol,
                                        int max_iters, void* workspace, size_t workspace_bytes,
                                        pararnn_stream_t stream);

/* Queues on `stream` a copy of the last solve's (or segment pass's) residual
 * into out[0] and 1.0f into out[1] if a device-side error was raised (else
 * 0.0f); out is two device floats.  Asynchronous: for host loops that reduce
 * the outcome across GPUs before reading it. */
PARARNN_API pararnn_status pararnn_result_to_device(const void* workspace, float* out,
                                                    pararnn_stream_t stream);

/* Synchronises `stream` and reads the outcome of the last solve or adjoint
 * queued on `workspace`.  Returns result->status (or an error if the read
 * itself fails).  `result` is a host pointer. */
PARARNN_API pararnn_status pararnn_read_result(const void* workspace, pararnn_stream_t stream,
                                   pararnn_result* result);

/* ------------------------------- input projection fused with Newton pass 0 */

/* ParaGRU solve from the layer input: the gate pre-activations are the input
 * projection u = x W^T + bias ("O compromisso que SSMs fizeram": the input
 * enters the recurrence through a projection, B_l x_l), computed on the
 * tensor cores in a kernel whose epilogue also runs Newton pass 0 ("A
 * sacada: método de Newton": at the initial guess H^0 = 0 the step maps
 * depend on the gates alone), so the first pass neither waits for u nor
 * reads it back.  The solve then continues from H^1 exactly as
 * pararnn_gru_solve (same stopping rule, status, iteration count).
 *   x     [B][L][Din] bf16, device (Din a multiple of 8)
 *   w     [3][D][Din] bf16, device: the projection's rows for gates z, r, c
 *         (row g*D + d produces u[..][g][d]; the layout of a linear layer's
 *         weight with 3*D outputs)
 *   bias  [3][D] fp32 or NULL (zeros)
 *   a, h0 as pararnn_gru_solve
 *   u     [B][L][3][D] bf16, device, out: u = bf16(x W^T + bias) with an
 *         fp32 accumulator, rounded to nearest even; the solve runs on these
 *         rounded values, so pararnn_gru_solve on u gives the same states
 *   h     [B][L][D] fp32 out
 * Workspace: pararnn_gru_project_workspace_size(B, L, D, Din) bytes (0 for
 * invalid shapes).  Errors as pararnn_gru_solve; Din not a positive multiple
 * of 8 gives UNSUPPORTED.  The _async form queues the work on `stream`; read
 * the outcome with pararnn_read_result. */
PARARNN_API size_t pararnn_gru_project_workspace_size(int64_t B, int64_t L, int64_t D, int64_t Din);
PARARNN_API pararnn_status pararnn_gru_project_solve(const void* x, const void* w, const float* bias,
                                                     const float* a, const float* h0, void* u,
                                                     float* h, int64_t B, int64_t L, int64_t Din,
                                                     int64_t D, float tol, int max_iters,
                                                     void* workspace, size_t workspace_bytes,
                                                     pararnn_stream_t stream, int* iters_out,
                                                     float* residual_out);
PARARNN_API pararnn_status pararnn_gru_project_solve_async(const void* x, const void* w,
                                                           const float* bias, const float* a,
                                                           const float* h0, void* u, float* h,
                                                           int64_t B, int64_t L, int64_t Din,
                                                           int64_t D, float tol, int max_iters,
                                                           void* workspace, size_t workspace_bytes,
                                                           pararnn_stream_t stream);

/* ------------------------------------------------- fixed-scratch solve */

/* ParaGRU Newton solve without a caller workspace.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory at the point of the call -- a plain C host program or a
 * plugin that owns no device allocator, or a latency-critical loop that must
 * not call cudaMalloc (which can synchronise the device) -- and so cannot
 * provide the workspace pararnn_gru_solve needs.
 *
 * Its scratch is one fixed array of pararnn_gru_solve_noalloc_max_scratch()
 * bytes (16 MiB) per device, part of the library's module image; the call
 * allocates nothing (no cudaMalloc, no cudaFree, no other allocator).  The
 * array is held on every device where the library's module is loaded, until
 * the process exits, whether or not this entry point is ever called.
 * Shapes whose pararnn_gru_workspace_size exceeds that return
 * PARARNN_ERR_WORKSPACE, and invalid arguments their usual status, before
 * any device call, with the reason in pararnn_last_error().  The first call
 * on a device looks up the scratch's device address (cudaGetSymbolAddress,
 * with that device current) and caches it per device ordinal for the life of
 * the process: make that first call before capturing `stream` into a graph,
 * and do not call this entry point on a device after the host program has
 * reset it (cudaDeviceReset), since the cached address then is stale.  The
 * scratch is shared by every call on the device, so calls that overlap in
 * time (other threads, or other streams not yet finished) race and must be
 * serialised by the caller.  Arguments, outputs and return values are those
 * of pararnn_gru_solve; synchronous. */
PARARNN_API pararnn_status pararnn_gru_solve_noalloc(const void* u, pararnn_dtype u_dtype, const float* a,
                                         const float* h0, float* h, int64_t B, int64_t L, int64_t D,
                                         float tol, int max_iters, pararnn_stream_t stream,
                                         int* iters_out, float* residual_out);

/* Bytes of the fixed scratch behind pararnn_gru_solve_noalloc. */
PARARNN_API size_t pararnn_gru_solve_noalloc_max_scratch(void);

/* -------------------------------------------------------------- adjoints */

/* Gradients of a loss through the converged ParaGRU states.  The pages do
 * not describe training gradients; the reading here: at the solution
 * F(H) = 0, dLoss/du = (dF/du)^T lambda with lambda solving the transposed
 * Newton system, i.e. the reverse-time linear recurrence
 *   lambda_l = dh_l + A_{l+1} lambda_{l+1},   lambda_L = dh_L,
 * which is again a linear SSM, scanned in reverse with A_l^T (= A_l here).
 *   h        [B][L][D] converged forward states (from pararnn_gru_solve)
 *   dh       [B][L][D] fp32 upstream gradient dLoss/dh_l
 *   du       [B][L][3][D] fp32 output dLoss/du
 *   da       [3][D] fp32 output dLoss/da, summed over b and l (overwritten,
 *            deterministic: fixed summation order)
 *   dh0      [B][D] fp32 output dLoss/dh0, or NULL
 * Asynchronous on `stream`; a device-side failure is reported by
 * pararnn_read_result on the same workspace. */
PARARNN_API pararnn_status pararnn_gru_adjoint(const void* u, pararnn_dtype u_dtype, const float* a,
                                   const float* h0, const float* h, const float* dh, float* du,
                                   float* da, float* dh0, int64_t B, int64_t L, int64_t D,
                                   void* workspace, size_t workspace_bytes,
                                   pararnn_stream_t stream);

/* ParaLSTM adjoint: reverse-time scan of the 2x2 transposed Jacobians
 *   lambda_l = (dc_l, dh_l) + J_{l+1}^T lambda_{l+1}.
 *   c, h     [B][L][D] converged forward states
 *   dh       [B][L][D] upstream dLoss/dh; dc [B][L][D] dLoss/dc or NULL (= 0)
 *   du       [B][L][4][D], da [4][D], dc0 / dh0 [B][D] or NULL.            */
PARARNN_API pararnn_status pararnn_lstm_adjoint(const void* u, pararnn_dtype u_dtype, const float* a,
                                    const float* c0, const float* h0, const float* c,
                                    const float* h, const float* dh, const float* dc, float* du,
                                    float* da, float* dc0, float* dh0, int64_t B, int64_t L,
                                    int64_t D, void* workspace, size_t workspace_bytes,
                                    pararnn_stream_t stream);

/* ---------------------------------------------------- user-written cells */

/* The fused solve for a cell the caller writes ("Como usar": the user writes
 * only the recurrence step; Newton, the Jacobians and the parallel reduction
 * are the library's).  `source` is CUDA C++ defining
 *
 *   template <class T, class U>
 *   __device__ void recurrence_step(const T* s, const U* u, const U* a,
 *                                   T* out);
 *
 * for one (b, d) channel: s = its n_state components at step l-1, u = its
 * n_gates gate pre-activations at step l, a = its n_gates recurrence
 * weights, out = its n_state components at step l.  The body uses +, -, *,
 * / and exp, log, tanh, sigmoid, sqrt, sin, cos (value_of(x) gives a plain
 * float for branches).  It runs with T = U = float for values, with T a
 * forward-mode dual number (U = float) for the Jacobian block d out / d s,
 * and with T = U a dual number for the adjoint's derivatives; the Jacobian
 * is diagonal (n_state = 1) or one 2x2 block per channel (n_state = 2).  pararnn_cell_create compiles it with NVRTC into the same
 * warp-specialised kernel as the built-in cells (dual-number Jacobians; the
 * CUDA math library's expf/tanhf/..., or with PARARNN_CELL_FAST_MATH the
 * hardware approximations), for sm_100a, and loads it on the current
 * device.
 *
 * Returns PARARNN_ERR_INVALID_ARG if the source does not compile (the start
 * of the compiler log is in pararnn_last_error(), all of it in
 * pararnn_cell_compile_log()), PARARNN_ERR_UNSUPPORTED for n_gates outside
 * 1..4, n_state outside 1..2 or when NVRTC cannot be loaded, and
 * PARARNN_ERR_CUDA when the module cannot be loaded (no device, not sm_100).
 * The handle belongs to the caller (pararnn_cell_destroy); it is bound to
 * the device that was current at creation. */
typedef struct pararnn_cell_st* pararnn_cell;

/* flags of pararnn_cell_create */
#define PARARNN_CELL_FAST_MATH 1u /* exp, log, tanh, sigmoid, sin, cos and the duals' divisions
                                     from the hardware approximations (__expf, __fdividef, ...)
                                     instead of the CUDA math library's accurate functions */

PARARNN_API pararnn_status pararnn_cell_create(const char* source, int n_gates, int n_state,
                                               unsigned flags, pararnn_cell* out);
/* Compute warps per CTA (two steps each) of the kernel chosen for a gate
 * dtype: the widest tile whose kernel spills at most 256 bytes a thread;
 * 0 for a NULL cell. */
PARARNN_API int pararnn_cell_compute_warps(pararnn_cell cell, pararnn_dtype u_dtype);
PARARNN_API void pararnn_cell_destroy(pararnn_cell cell);
/* Compiler log of the calling thread's last pararnn_cell_create ("" if none). */
PARARNN_API const char* pararnn_cell_compile_log(void);
/* Workspace bytes for one solve (0 = invalid shape); depends on u's dtype,
 * which sets the tile. */
PARARNN_API size_t pararnn_cell_workspace_size(pararnn_cell cell, pararnn_dtype u_dtype, int64_t B,
                                               int64_t L, int64_t D);

/* Newton solve of the cell's recurrence, with the stopping rule, outputs and
 * errors of pararnn_gru_solve.
 *   u   [B][L][n_gates][D] bf16 or fp32;  a [n_gates][D] fp32
 *   s0  [n_state][B][D] fp32 initial state (NULL = zeros)
 *   s   [n_state][B][L][D] fp32 out, components one after another
 * Device pointers, 16-byte aligned; D a multiple of 8.  Synchronous like
 * pararnn_gru_solve; the _async form returns after the launch and the
 * outcome is read with pararnn_read_result. */
PARARNN_API pararnn_status pararnn_cell_solve(pararnn_cell cell, const void* u, pararnn_dtype u_dtype,
                                              const float* a, const float* s0, float* s, int64_t B,
                                              int64_t L, int64_t D, float tol, int max_iters,
                                              void* workspace, size_t workspace_bytes,
                                              pararnn_stream_t stream, int* iters_out,
                                              float* residual_out);
/* Training gradients through a user cell: the reverse-time adjoint of
 * pararnn_gru_adjoint for the cell's own equations, at converged forward
 * states s (from pararnn_cell_solve).  The derivatives of the step with
 * respect to its state, gates and weights come from one forward-mode
 * dual-number evaluation per step.
 *   ds   [n_state][B][L][D] upstream gradient dLoss/ds, fp32, every component
 *   du   [B][L][n_gates][D] fp32 out;  da [n_gates][D] fp32 out (overwritten)
 *   ds0  [n_state][B][D] fp32 out, dLoss/ds0 (NULL = not wanted)
 * Other arguments as for pararnn_cell_solve; the workspace comes from
 * pararnn_cell_adjoint_workspace_size.  Asynchronous on `stream`; the
 * status reports argument and launch errors. */
PARARNN_API size_t pararnn_cell_adjoint_workspace_size(pararnn_cell cell, int64_t B, int64_t L,
                                                       int64_t D);
PARARNN_API pararnn_status pararnn_cell_adjoint(pararnn_cell cell, const void* u,
                                                pararnn_dtype u_dtype, const float* a,
                                                const float* s0, const float* s, const float* ds,
                                                float* du, float* da, float* ds0, int64_t B,
                                                int64_t L, int64_t D, void* workspace,
                                                size_t workspace_bytes, pararnn_stream_t stream);
PARARNN_API pararnn_status pararnn_cell_solve_async(pararnn_cell cell, const void* u,
                                                    pararnn_dtype u_dtype, const float* a,
                                                    const float* s0, float* s, int64_t B, int64_t L,
                                                    int64_t D, float tol, int max_iters,
                                                    void* workspace, size_t workspace_bytes,
                                                    pararnn_stream_t stream);

/* Duration of each Newton pass of the last solve run on `workspace` (the
 * built-in and user-cell solves), from device timestamps the kernel takes
 * when every CTA has finished a pass: pass_us[i] = microseconds of pass i,
 * pass 0 from the kernel's start; *n_passes = passes recorded (at most 15).
 * Synchronises `stream`.  The durations include the grid barrier that ends
 * each pass; they sum to the kernel's time less its prologue and epilogue.
 * The per-iteration roofline is (bytes a pass moves) / pass_us[i]. */
PARARNN_API pararnn_status pararnn_read_pass_times(const void* workspace, pararnn_stream_t stream,
                                                   double* pass_us, int max_passes, int* n_passes);

/* ------------------------------------------------- segments of a sequence */

/* The Newton solve with the sequence split into segments, one per GPU ("A
 * sacada: método de Newton": every iteration solves a linear recurrence
 * whose step maps s -> J_l s + o_l depend only on the iterate H^k, so over a
 * segment they compose into one affine map of the state entering it).  One
 * iteration k on each segment:
 *   1. pararnn_*_segment_fold: the segment's record from H^k -- its step
 *      maps folded (steps 2..Ls), the iterate's first and last states, the
 *      first step's gates, the residual over steps 2..Ls;
 *   2. gather every segment's record, in segment order (the one data
 *      exchange between GPUs: pararnn_segment_record_floats each);
 *   3. pararnn_*_segment_combine: the records composed in order -> the new
 *      state entering this segment (carry), the iterate's state before it
 *      (lin), and max |F(H^k)| over all segments, the same on every GPU;
 *      stop here if it is <= tol (or k = max_iters);
 *   4. pararnn_*_segment_pass(s_in = H^k, s_lin = lin, s_carry = carry,
 *      s_out = H^k in place) -> H^{k+1} on the segment; its residual (read
 *      with pararnn_read_result) maxed over the segments is that of H^{k+1},
 *      which takes the next decision without another fold.
 * Components are stacked one after another: [NS][B][Ls][D] for states over
 * the segment, [NS][B][D] for one step (LSTM: c, then h).  Device pointers,
 * 16-byte aligned, D a multiple of 8; all calls asynchronous on `stream`.
 *
 * segment_pass: one pass over the segment (gates u [B][Ls][G][D] of its
 * steps) from the iterate s_in (NULL = the zero guess H^0), linearising the
 * first step at s_lin (the iterate's state before the segment; NULL = 0),
 * with s_carry (NULL = 0) as the new state before it.  Writes s_out (s_in
 * itself, or a buffer that does not overlap it) and, if s_end is not NULL,
 * the last step's states.  The workspace is the solve's
 * (pararnn_*_workspace_size(B, Ls, D)); its result (pararnn_read_result)
 * holds the residual of s_out with s_carry as the state before it. */
PARARNN_API pararnn_status pararnn_gru_segment_pass(const void* u, pararnn_dtype u_dtype,
                                                    const float* a, const float* h_in,
                                                    const float* h_lin, const float* h_carry,
                                                    float* h_out, float* h_end, int64_t B,
                                                    int64_t L, int64_t D, void* workspace,
                                                    size_t workspace_bytes,
                                                    pararnn_stream_t stream);
PARARNN_API pararnn_status pararnn_lstm_segment_pass(const void* u, pararnn_dtype u_dtype,
                                                     const float* a, const float* s_in,
                                                     const float* s_lin, const float* s_carry,
                                                     float* s_out, float* s_end, int64_t B,
                                                     int64_t L, int64_t D, void* workspace,
                                                     size_t workspace_bytes,
                                                     pararnn_stream_t stream);
/* Floats of one segment's record (n_state = 1: ParaGRU, 2: ParaLSTM) for B x
 * D channels: F = NC + 2 NS + G fields of B*D floats (NC = 2 or 6 map
 * entries, NS = 1 or 2, G = 3 or 4), then 4 floats (the first is the
 * residual over the segment's steps 2..Ls).  0 for invalid arguments. */
PARARNN_API size_t pararnn_segment_record_floats(int n_state, int64_t B, int64_t D);
/* Workspace bytes of segment_fold (its partial folds, one per part of 64 or
 * more steps). */
PARARNN_API size_t pararnn_segment_fold_workspace_size(int n_state, int64_t B, int64_t L, int64_t D);
/* segment_fold: the segment's record (overwritten in full) from the iterate
 * s_in [NS][B][Ls][D] (NULL = the zero guess) and the gates u [B][Ls][G][D]
 * (bf16 or fp32). */
PARARNN_API pararnn_status pararnn_gru_segment_fold(const void* u, pararnn_dtype u_dtype,
                                                    const float* a, const float* h_in,
                                                    float* record, int64_t B, int64_t L,
                                                    int64_t D, void* workspace,
                                                    size_t workspace_bytes,
                                                    pararnn_stream_t stream);
PARARNN_API pararnn_status pararnn_lstm_segment_fold(const void* u, pararnn_dtype u_dtype,
                                                     const float* a, const float* s_in,
                                                     float* record, int64_t B, int64_t L,
                                                     int64_t D, void* workspace,
                                                     size_t workspace_bytes,
                                                     pararnn_stream_t stream);
/* segment_combine: records [n_segments][record_floats] in segment order and
 * the initial state s0 [NS][B][D] (NULL = 0) -> for segment `index`: carry
 * (the state entering it at iterate k+1) and lin (the iterate's state before
 * it), [NS][B][D]; *residual (a device float, overwritten) = max |F(H^k)|
 * over every segment's steps, NaN kept. */
PARARNN_API pararnn_status pararnn_gru_segment_combine(const float* records, int n_segments,
                                                       int index, const float* a,
                                                       const float* h0, float* h_carry,
                                                       float* h_lin, float* residual, int64_t B,
                                                       int64_t D, pararnn_stream_t stream);
PARARNN_API pararnn_status pararnn_lstm_segment_combine(const float* records, int n_segments,
                                                        int index, const float* a,
                                                        const float* s0, float* s_carry,
                                                        float* s_lin, float* residual, int64_t B,
                                                        int64_t D, pararnn_stream_t stream);

/* ----------------------------------------------------------- decode step */

/* One recurrence step for B sequences at once, the token-by-token generation
 * that "Por que RNN ainda importa" credits RNNs with (cost per token fixed,
 * whatever the context length): s_next = f(s_prev, u) with the cells of the
 * solves above.
 *   u       [B][G][D] gate pre-activations of this step (G = 3: z, r, c for
 *           the GRU; G = 4: i, f, o, g for the LSTM), bf16 or fp32
 *   a       [G][D] diagonal recurrence weights, fp32
 *   *_prev  [B][D] current state, fp32; NULL = zeros
 *   *_next  [B][D] next state, fp32, written in full
 * All device pointers, 16-byte aligned; D a multiple of 8.  An output may be
 * the very buffer of its own previous state (update in place); any other
 * overlap between outputs and inputs, or between c_next and h_next, is
 * refused with PARARNN_ERR_INVALID_ARG before any launch.  One kernel launch,
 * asynchronous on `stream`, capturable in a CUDA graph; the library keeps no
 * state between calls. */
PARARNN_API pararnn_status pararnn_gru_step(const void* u, pararnn_dtype u_dtype, const float* a,
                                            const float* h_prev, float* h_next, int64_t B,
                                            int64_t D, pararnn_stream_t stream);
PARARNN_API pararnn_status pararnn_lstm_step(const void* u, pararnn_dtype u_dtype, const float* a,
                                             const float* c_prev, const float* h_prev,
                                             float* c_next, float* h_next, int64_t B, int64_t D,
                                             pararnn_stream_t stream);

/* ------------------------------------------------------------- baselines */

/* Naive sequential application ("O compromisso que SSMs fizeram": one step
 * at a time): one GPU thread per (b, d) channel walks l = 1..L.  Same
 * outputs as the solves (to rounding); asynchronous on `stream`. */
PARARNN_API pararnn_status pararnn_gru_sequential(const void* u, pararnn_dtype u_dtype, const float* a,
                                      const float* h0, float* h, int64_t B, int64_t L,
                                      int64_t D, pararnn_stream_t stream);
PARARNN_API pararnn_status pararnn_lstm_sequential(const void* u, pararnn_dtype u_dtype, const float* a,
                                       const float* c0, const float* h0, float* c, float* h,
                                       int64_t B, int64_t L, int64_t D,
                                       pararnn_stream_t stream);

/* Plain diagonal linear scan, the SSM of "O compromisso que SSMs fizeram",
 * as a lower bound on one scan pass over the same [B][L][3][D] input: the
 * GRU with zero recurrence weights,
 *   h_l = (1 - s(u_z)) h_{l-1} + s(u_z) tanh(u_c),
 * which reads two of the three gate streams.  One pass, no Newton;
 * asynchronous on `stream`.  Workspace from
 * pararnn_linear_scan_workspace_size. */
PARARNN_API size_t pararnn_linear_scan_workspace_size(int64_t B, int64_t L, int64_t D);
PARARNN_API pararnn_status pararnn_linear_scan(const void* u, pararnn_dtype u_dtype, const float* h0,
                                   float* h, int64_t B, int64_t L, int64_t D, void* workspace,
                                   size_t workspace_bytes, pararnn_stream_t stream);

/* ------------------------------------------------------------ diagnostics */

PARARNN_API const char* pararnn_status_string(pararnn_status s);
/* Detail of the last error on the calling thread ("" if none). */
PARARNN_API const char* pararnn_last_error(void);
/* Library version as "major.minor.patch". */
PARARNN_API const char* pararnn_version(void);
/* Number of kernels this library has launched in this process (all threads). */
PARARNN_API uint64_t pararnn_kernel_launch_count(void);

/* Failure-detection self tests.  Each launches a small kernel that runs one
 * of the library's bounded waits against a condition nothing will satisfy:
 *   which = 0: the decoupled look-back of a tile whose predecessor never
 *              publishes;
 *   which = 1: the grid barrier (one CTA of a cooperative launch never
 *              arrives).
 * The wait must give up after `limit_ns` nanoseconds and the call must return
 * PARARNN_ERR_TIMEOUT with the context still usable.  Needs a workspace of
 * at least 16384 bytes.  Synchronous. */
PARARNN_API pararnn_status pararnn_selftest_wait_timeout(int which, int64_t limit_ns, void* workspace,
                                             size_t workspace_bytes, pararnn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PARARNN_H */
