/*
 * pararnn_b200.h -- C ABI of libpararnn_b200, the B200 (sm_100a) hot path of
 * ParaRNN: Newton iterations on a whole-trajectory nonlinear system, each
 * linear solve done as a parallel associative scan over time, and the
 * reverse-time adjoint scan for the backward pass.
 *
 * The method (pararnn-torch PyPI page, Method section; ParaRNN thread, tweet
 * [3/8]; ParaRNN abstract on the Hugging Face paper search page):
 *   the recurrence h_t = f(h_{t-1}, x_t), t = 0..T-1, h_{-1} = h0, is the
 *   system F(H)_t = h_t - f(h_{t-1}, x_t) = 0.  Starting from the warm start
 *   h_t^(0) = f(0, x_t) (Method section, "App. A"), each Newton iteration
 *   evaluates f and its Jacobian A_t = df/dh_{t-1} at the current iterate and
 *   solves the lower block-bidiagonal system
 *       delta_t = A_t delta_{t-1} - F_t,  delta_{-1} = 0,
 *   by an associative scan over time with the operator
 *       (A2, b2) o (A1, b1) = (A2 A1, A2 b1 + b2)
 *   (Method section: "each linear solve is an associative scan over time").
 *   The library solves the equivalent direct form
 *       h_t^(k+1) = A_t h_{t-1}^(k+1) + (f(h_{t-1}^(k), x_t) - A_t h_{t-1}^(k)),
 *   h_{-1} = h0, which is the same update without reading h^(k)_t.
 *
 * Cells (diagonal: every channel d is an independent recurrence; p_g are the
 * gate pre-activations, a_g the per-gate, per-channel recurrent weights):
 *   PARARNN_CELL_LINEAR     S=1, G=2 (a, b):   h' = a h + b
 *                           (the affine case the News section says needs no
 *                           Newton iteration beyond one exact scan)
 *   PARARNN_CELL_DIAG_GRU   S=1, G=3 (z, r, c): z = sig(p_z + a_z h),
 *                           r = sig(p_r + a_r h), c = tanh(p_c + a_c r h),
 *                           h' = (1 - z) h + z c          (ParaGRU, Models)
 *   PARARNN_CELL_DIAG_LSTM  S=2 state (c, h), G=4 (i, f, o, c):
 *                           i = sig(p_i + a_i h), f = sig(p_f + a_f h + 1),
 *                           o = sig(p_o + a_o h), g = tanh(p_c + a_c h),
 *                           c' = f c + i g, h' = o tanh(c')  (ParaLSTM)
 *
 * Layouts (row-major, channels fastest, all device memory owned by the
 * caller):
 *   preacts  (B, T, G, D)  float32 or bfloat16 (px_dtype)
 *   diag_w   (G, D)        float32, or NULL for all-zero weights (ignored by
 *                          the linear cell)
 *   h0       (B, S, D)     float32, or NULL for a zero initial state
 *   H        (B, T, S, D)  float32 (LSTM: state order c, h)
 *   dL_dH    (B, T, S, D)  float32
 *   dL_dpx   (B, T, G, D)  float32
 *   dL_da    (G, D)        float32
 *   dL_dh0   (B, S, D)     float32
 * Every pointer must be aligned to its element size.  When D times the
 * pre-activation element size is a multiple of 16 bytes and the row buffers
 * are 16-byte aligned, tiles are staged by the tensor memory accelerator;
 * otherwise the same kernels copy them element by element.
 *
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 * default stream).  Argument errors are detected on the host before anything
 * is launched and return PARARNN_EINVAL (nothing is written).  Conditions the
 * GPU detects -- a non-finite value in the output, a wait between thread
 * blocks that ran past its time limit -- are recorded in the workspace and
 * returned by pararnn_status_sync().  A CUDA launch or copy failure returns
 * PARARNN_ECUDA.  Apart from the fixed scratch array that
 * pararnn_newton_forward_noalloc uses (part of the library's device image),
 * the library allocates no memory; the only state it keeps between calls is a
 * process-wide call counter that tags the scan carries it leaves in a
 * workspace.  pararnn_last_error() describes the last failure on
 * the calling thread.  Results are deterministic: the same inputs give the same bits,
 * whatever the order in which thread blocks run.
 */
#ifndef PARARNN_B200_H
#define PARARNN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PARARNN_OK = 0,
    PARARNN_EINVAL = 1,     /* bad argument; nothing launched */
    PARARNN_ENONFINITE = 2, /* a NaN or Inf reached the output */
    PARARNN_ETIMEOUT = 3,   /* a bounded inter-block wait gave up; outputs invalid */
    PARARNN_ECUDA = 4       /* a CUDA runtime call failed */
} pararnn_status;

typedef enum {
    PARARNN_CELL_LINEAR = 0,
    PARARNN_CELL_DIAG_GRU = 1,
    PARARNN_CELL_DIAG_LSTM = 2
} pararnn_cell;

typedef enum {
    PARARNN_F32 = 0,
    PARARNN_BF16 = 1
} pararnn_dtype;

/* Gate count G (2, 3, 4) and state width S (1, 1, 2) of a cell; -1 if the
 * cell is unknown.  Pure host functions. */
int pararnn_num_gates(pararnn_cell cell);
int pararnn_state_width(pararnn_cell cell);

/* Bytes of device workspace that pararnn_newton_forward (with this K) and
 * pararnn_newton_backward need for a (B, T, D) problem; the same buffer
 * serves both.  0 for an unknown cell or a negative size.  Pure host
 * function.  The workspace holds a status word, a tile counter, the
 * inter-block scan carries and per-block gradient partials.  It needs no
 * initialisation: every call clears, on its stream and before its kernels
 * run, every word of it that the call reads before writing (the status word,
 * the tile counter and all scan carries), so whatever an earlier call -- or
 * any other use of the memory -- left there is never read.  Calls that share
 * a workspace must be ordered (the same stream, or synchronised); calls that
 * overlap on the GPU with one workspace race. */
size_t pararnn_workspace_bytes(pararnn_cell cell, int64_t B, int64_t T, int64_t D, int K);

/* The measured Newton budget K*(cell, T) that K = 0 selects (pararnn-torch
 * page, Method section: K*(T) is the smallest iteration count that matches
 * the sequential unroll within about 1e-4, measured per cell on a T grid,
 * and NewtonConfig(max_iters=None) reads those tables).  Here the table was
 * measured on this library's forward against an fp64 sequential unroll, on
 * synthetic cells (pre-activations ~ N(0,1), diagonal recurrent weights
 * ~ U(-0.5, 0.5), h0 = 0) at T = 16, 64, ..., 262144; a T between grid
 * points takes the entry of the next grid point up, a T past the grid the
 * last entry.  Inputs drawn otherwise (trained weights, saturated gates) can
 * need another K.  Returns 1 for the linear cell (one scan is exact) and -1
 * for an unknown cell or a negative T.  Pure host function. */
int pararnn_kstar(pararnn_cell cell, int64_t T);

/* Newton forward: K iterations from the warm start, output H = h^(K).
 * (Method section; NewtonConfig(max_iters=K), API overview section.)
 *   preacts    (B,T,G,D) in px_dtype, read only
 *   diag_w     (G,D) f32 or NULL (zeros)
 *   h0         (B,S,D) f32 or NULL (zeros)
 *   K          1..64 Newton iterations, or 0 for K = pararnn_kstar(cell, T)
 *              (max_iters=None); the linear cell is exact after one, and
 *              performs exactly one scan for any K
 *   H_out      (B,T,S,D) f32, written
 *   workspace  >= pararnn_workspace_bytes(cell,B,T,D,K) bytes, 16-byte
 *              aligned device memory, any contents (cleared on `stream`)
 *   resid_hist NULL, or K+1 floats of device memory that receive
 *              max_{b,t,s,d} |F(H^(k))| for k = 0..K (the residual history a
 *              NewtonDivergenceError carries, Evaluation section); with
 *              K = 0, pararnn_kstar(cell, T) + 1 floats
 * B, T or D equal to 0 is an empty problem: nothing is launched except the
 * zeroing of resid_hist. */
pararnn_status pararnn_newton_forward(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                      pararnn_dtype px_dtype, const void* preacts, const float* diag_w,
                                      const float* h0, int K, float* H_out, void* workspace,
                                      size_t ws_bytes, float* resid_hist, void* stream);

/* The sequential unroll of a diagonal cell on the GPU: h_t = f(h_{t-1}, x_t)
 * for t = 0..T-1, h_{-1} = h0 -- the one-step recurrence the Newton forward
 * reproduces at convergence (pararnn-torch page, API overview / Quickstart:
 * sequential_apply beside newton_apply), for timing the Newton forward
 * against the sequential recurrence on the same device.  One thread per
 * (batch row, channel) walks the sequence; arguments and layouts as for
 * pararnn_newton_forward (diag_w ignored by the linear cell).
 *   workspace  >= 256 bytes of device memory (only its status word is used;
 *              cleared on `stream`)
 * Errors: PARARNN_EINVAL (nothing launched) for an unknown cell or dtype, bad
 * sizes (B * D at or above 2^37), null, host or misaligned pointers, or a
 * missing workspace; PARARNN_ECUDA if the launch fails.  A non-finite value
 * in H_out is recorded for pararnn_status_sync(workspace, stream). */
pararnn_status pararnn_unroll(pararnn_cell cell, int64_t B, int64_t T, int64_t D, pararnn_dtype px_dtype,
                              const void* preacts, const float* diag_w, const float* h0, float* H_out,
                              void* workspace, size_t ws_bytes, void* stream);

/* The Newton forward with picard_iters Picard sweeps before the Newton
 * iterations (API overview, "Solver": picard_iters warms the first guess;
 * Method section: a zero-hidden start plus Picard).  From the warm start
 * h^(0)_t = f(0, x_t), each sweep forms h^(p+1)_t = f(h^(p)_{t-1}, x_t) for
 * every t at once, with h^(p)_{-1} = h0; sweep p makes the first p rows
 * (p + 1 when h0 is zero) equal to the sequential unroll.  The K Newton
 * iterations then start from h^(P), and resid_hist[0] is the residual of
 * h^(P).  picard_iters is 0..4 (0: exactly pararnn_newton_forward); the
 * linear cell ignores it.  Every other argument, the workspace size and the
 * errors are those of pararnn_newton_forward; a picard_iters outside 0..4
 * returns PARARNN_EINVAL.  The sweeps run inside the same kernel as the
 * Newton iterations: each thread evaluates its rows and the picard_iters + 1
 * rows before them, so no further HBM traffic or look-back is needed. */
pararnn_status pararnn_newton_forward_picard(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                             pararnn_dtype px_dtype, const void* preacts, const float* diag_w,
                                             const float* h0, int picard_iters, int K, float* H_out,
                                             void* workspace, size_t ws_bytes, float* resid_hist,
                                             void* stream);

/* Adjoint (backward) at the trajectory H (normally the forward's output):
 *   lambda_t = dL/dH_t + A_{t+1}^T lambda_{t+1},  lambda_{T-1} = dL/dH_{T-1},
 * with A_{t+1} = df/dh at (h_t, x_{t+1}), a reverse-time scan under the same
 * operator (Method section: "Backward follows paper eq. 2.6"; the ParaRNN
 * thread's "custom parallel reductions").  Then
 *   dL_dpx[b,t,g,d] = lambda_t . df/dp_g at (h_{t-1}, x_t)
 *   dL_da[g,d]      = sum_{b,t} lambda_t . df/da_g at (h_{t-1}, x_t)
 *   dL_dh0[b,:,d]   = A_0^T lambda_0
 * dL_da is reduced in a fixed order without floating-point atomics
 * (Compatibility section: the packed VJP is deterministic).
 *   dL_dpx  (B,T,G,D) f32, written (required)
 *   dL_da   (G,D) f32 or NULL; not written for the linear cell (no weights)
 *   dL_dh0  (B,S,D) f32 or NULL */
pararnn_status pararnn_newton_backward(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                       pararnn_dtype px_dtype, const void* preacts, const float* diag_w,
                                       const float* h0, const float* H, const float* dL_dH, float* dL_dpx,
                                       float* dL_da, float* dL_dh0, void* workspace, size_t ws_bytes,
                                       void* stream);

/* Waits for `stream` and returns what the GPU recorded for the last forward
 * or backward call that used `workspace`: PARARNN_OK, PARARNN_ENONFINITE or
 * PARARNN_ETIMEOUT (ETIMEOUT wins if both happened); PARARNN_ECUDA if the copy
 * or the synchronisation fails. */
pararnn_status pararnn_status_sync(const void* workspace, void* stream);

/* Static, NUL-terminated name of a status code ("PARARNN_OK", ...). */
const char* pararnn_status_string(pararnn_status status);

/* Static, NUL-terminated description of the last EINVAL or ECUDA returned on
 * the calling thread ("" if none). */
const char* pararnn_last_error(void);

/* Test hooks for the bounded waits between thread blocks and for the choice
 * of path (no counterpart on the pages).  They apply to the
 * pararnn_newton_forward and pararnn_newton_backward calls made afterwards on
 * the calling thread:
 *   wait_limit_ns  the limit of every wait of one thread block on another
 *                  (a look-back for a predecessor's carry, a staged tile);
 *                  0 restores the default of 2 s; at most 10 s
 *   flags          PARARNN_HOOK_STALL_FIRST_TILE: the first tile of the scan
 *                  computes as usual but never publishes its carry, so the
 *                  look-back of the tile after it runs out of time.  The
 *                  waiting block then records PARARNN_ETIMEOUT in the
 *                  workspace, takes a zero carry and finishes; the kernel ends
 *                  after about K * wait_limit_ns and pararnn_status_sync()
 *                  reports PARARNN_ETIMEOUT.  Outputs of such a call are
 *                  invalid.  Forwards take the look-back path while it is set.
 *                  PARARNN_HOOK_NO_CLUSTER: forwards never take the
 *                  small-problem path (below), so that both paths can be
 *                  compared on the same small inputs.
 *                  0 clears both.
 * Returns PARARNN_EINVAL (nothing changed) for a limit above 10 s or an
 * unknown flag.  Pure host function.
 *
 * The small-problem path: when every channel group's tiles along T fit in
 * one thread-block cluster (up to 16 tiles where the device allows clusters
 * of 16, else 8) and K <= 8, pararnn_newton_forward runs as one kernel whose
 * thread blocks pass their carries through distributed shared memory; it
 * launches nothing else (no clearing of the workspace) and records its
 * status in a word tagged with its call number, which pararnn_status_sync()
 * reads.  Problems with few channel groups (B * ceil(D/32) <= 18) and
 * T <= 1024 use tiles of 64 steps on both paths.  The small-problem path's
 * results are bit-identical to the look-back path's. */
#define PARARNN_HOOK_STALL_FIRST_TILE 1
#define PARARNN_HOOK_NO_CLUSTER 2
pararnn_status pararnn_debug_hooks(uint64_t wait_limit_ns, int flags);

/* Runs the library's bounded inter-block wait on a flag that nothing sets,
 * with a limit of timeout_ns nanoseconds, so that a test can see the time-out
 * path end cleanly: the kernel records PARARNN_ETIMEOUT in the workspace and
 * returns; pararnn_status_sync() then reports it.  workspace needs at least
 * pararnn_workspace_bytes(PARARNN_CELL_LINEAR, 1, 1, 1, 1) bytes. */
pararnn_status pararnn_probe_wait_timeout(void* workspace, size_t ws_bytes, uint64_t timeout_ns, void* stream);

/* The Newton forward for callers that cannot allocate device memory.  (The
 * ParaRNN pages have no counterpart: this is a deployment convenience.)
 * Some callers cannot call cudaMalloc when they run the forward -- a host
 * framework that owns every device allocation through its own pool, a
 * latency-bound loop that cannot afford cudaMalloc's implicit
 * synchronisation, a process with a device-memory budget fixed at start-up.
 * This entry point computes exactly what pararnn_newton_forward computes, with
 * the same kernels, but keeps its scratch memory (the workspace) in a fixed
 * 32 MiB array inside the library's device image, so it allocates nothing.
 * Every GPU that loads the library holds that array until the process exits.
 *   Arguments are those of pararnn_newton_forward without workspace/ws_bytes.
 *   wait_status  0: return once launched (device-detected conditions are then
 *                not reported); non-zero: wait for `stream` and return the
 *                device status as pararnn_status_sync would.
 * Problems whose pararnn_workspace_bytes(cell, B, T, D, K) exceeds 32 MiB
 * return PARARNN_EINVAL with an explanation in pararnn_last_error().  The
 * first call on a device sets that device up: it looks up the array's device
 * address with cudaGetSymbolAddress (which may load the library's device code
 * onto that device), so make that first call before any stream capture.  A
 * failed look-up returns PARARNN_ECUDA and is tried again on the next call.
 * All calls share the one array, which keeps the last call's contents; each
 * call clears, on `stream`, the part it reads before writing, as
 * pararnn_newton_forward does with its workspace.  Calls that overlap on the
 * GPU race, so order them (one stream, or synchronise between them). */
pararnn_status pararnn_newton_forward_noalloc(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                              pararnn_dtype px_dtype, const void* preacts, const float* diag_w,
                                              const float* h0, int K, float* H_out, float* resid_hist,
                                              int wait_status, void* stream);

/* ---- the forward on host buffers (serving) --------------------------------
 * pararnn_newton_forward for pre-activations and H in host memory (pinned
 * memory lets the copies overlap; pageable memory works, with the copies
 * serialised).  The batch is cut into slices of rows_per_slice rows and,
 * when channels_per_slice is not 0, of channels_per_slice channels each
 * (copied with strided 2-D copies); the slices pass through three device
 * slots on three internal streams -- copy in, solve, copy out -- so that
 * both PCIe directions and the solver work at once.  More, smaller slices
 * shorten the pipeline's fill and drain.  Batch rows and channels are
 * independent recurrences, so every value of H is bit-identical to
 * pararnn_newton_forward's on the whole batch.
 *   channels_per_slice  0 (or >= D): whole rows; otherwise a multiple of 8,
 *                 and D must be a multiple of 8 too (every slice then keeps
 *                 the whole batch's 16-byte row alignment and solver path)
 *   preacts_host  (B, T, G, D) px_dtype, host (or device) memory
 *   diag_w, h0    device memory, as for pararnn_newton_forward
 *   H_host        (B, T, S, D) float32, host (or device) memory
 *   workspace     >= pararnn_newton_forward_host_workspace_bytes(...) bytes,
 *                 256-byte aligned device memory, any contents
 * The work is ordered after what is already queued on `stream`, and work
 * queued on `stream` afterwards runs after it; the call returns once
 * everything is queued.  No residual history is kept.  A non-finite value in
 * any slice's output is reported by pararnn_status_sync(workspace, stream).
 * Errors as for pararnn_newton_forward, plus PARARNN_EINVAL for
 * rows_per_slice < 1 or a channels_per_slice outside the rule above, and
 * PARARNN_ECUDA if the internal streams cannot be created.  The workspace
 * size function returns 0 for the same invalid arguments. */
size_t pararnn_newton_forward_host_workspace_bytes(pararnn_cell cell, int64_t B, int64_t T, int64_t D, int K,
                                                   pararnn_dtype px_dtype, int64_t rows_per_slice,
                                                   int64_t channels_per_slice);
pararnn_status pararnn_newton_forward_host(pararnn_cell cell, int64_t B, int64_t T, int64_t D,
                                           pararnn_dtype px_dtype, const void* preacts_host, const float* diag_w,
                                           const float* h0, int K, float* H_host, void* workspace, size_t ws_bytes,
                                           int64_t rows_per_slice, int64_t channels_per_slice, void* stream);

/* ---- a training step on host buffers --------------------------------------
 * pararnn_newton_forward followed by pararnn_newton_backward, with the
 * pre-activations and dL/dH read from host memory and H and dL/dpx written
 * back to it (pinned memory lets the copies overlap).  The channels are cut
 * into slices of channels_per_slice channels (the first slice a quarter of
 * that, rounded up to a multiple of 8, so that the pipeline fills quickly),
 * each holding every batch row, that pass through three device slots on
 * three internal streams -- copy in, forward + adjoint, copy out -- so that
 * both PCIe directions and the solver work at once.  A slice's dL/da columns are complete sums over (b, t) and
 * are written straight into dL_da.  Channels are independent recurrences and
 * the tiling along T does not depend on the slice, so every output is
 * bit-identical to pararnn_newton_forward + pararnn_newton_backward on the
 * whole batch (Method section: forward by Newton, backward by one linear
 * adjoint scan; the API overview's training use of ParaGRU / ParaLSTM).
 *   channels_per_slice  0 (or >= D): one slice; otherwise a multiple of 8,
 *                 and D must be a multiple of 8 too
 *   preacts_host  (B, T, G, D) px_dtype, host (or device) memory
 *   dL_dH_host    (B, T, S, D) float32, host (or device) memory
 *   diag_w, h0    device memory or NULL, as for pararnn_newton_forward
 *   H_host        (B, T, S, D) float32, host (or device) memory, written
 *   dL_dpx_host   (B, T, G, D) float32, host (or device) memory, written
 *   dL_da         (G, D) float32 device memory or NULL, written (NULL, and
 *                 nothing written, for the linear cell)
 *   workspace     >= pararnn_newton_step_host_workspace_bytes(...) bytes,
 *                 256-byte aligned device memory, any contents
 * K as for pararnn_newton_forward (0 takes pararnn_kstar).  Ordering with
 * `stream`, status reporting and errors as for pararnn_newton_forward_host;
 * dL/dh0 is not computed.  The workspace size function returns 0 for invalid
 * arguments. */
size_t pararnn_newton_step_host_workspace_bytes(pararnn_cell cell, int64_t B, int64_t T, int64_t D, int K,
                                                pararnn_dtype px_dtype, int64_t channels_per_slice);
pararnn_status pararnn_newton_step_host(pararnn_cell cell, int64_t B, int64_t T, int64_t D, pararnn_dtype px_dtype,
                                        const void* preacts_host, const float* diag_w, const float* h0, int K,
                                        const float* dL_dH_host, float* H_host, float* dL_dpx_host, float* dL_da,
                                        void* workspace, size_t ws_bytes, int64_t channels_per_slice, void* stream);

/* ---- head-wise GRU: block-diagonal recurrent weights --------------------
 * ParaGRU(mix='head', n_heads) of the pararnn-torch page (Models / Usage,
 * "Dreamer-style block GRU": block-diagonal A).  The page prints no
 * equations; the cell here is the GRU of torch.nn.GRUCell with its recurrent
 * weight restricted to n_heads dense d x d blocks (D = n_heads * d), in this
 * library's gate convention.  For one head, state s (d values):
 *     z = sig(p_z + U_z s),  r = sig(p_r + U_r s),  n = U_c s,
 *     c = tanh(p_c + r * n), s' = (1 - z) * s + z * c       (* elementwise)
 * -- the diagonal GRU above when every U_g is diagonal.  Its Jacobian is a
 * dense d x d block per head, so each Newton iteration's scan multiplies d x d
 * matrices (d^3 work per step, against d^2 for the sequential unroll).
 * Newton iterations, warm start and K have the meaning of
 * pararnn_newton_forward; each linear solve is done in the update form
 * delta_t = A_t delta_{t-1} - F_t, h^(k+1) = h^(k) + delta.
 *
 * Layouts (row-major, device memory owned by the caller):
 *   preacts  (B, T, 3, D)         float32 or bfloat16 (px_dtype), gates z, r, c
 *   U        (3, n_heads, d, d)   float32: U[g][h][i][j] is the weight of state
 *                                 j of head h in gate g's pre-activation i
 *   h0       (B, D)               float32, or NULL for a zero initial state
 *   H_out    (B, T, D)            float32
 * d = D / n_heads must be 16, 32 or 64.
 *
 * Returns the workspace size for these sizes, or 0 when they are invalid
 * (d not in {16, 32, 64}, D not a multiple of n_heads, K outside 1..64, B*T
 * at or above 2^31).  It holds a second iterate buffer (K >= 2), each
 * chunk's d x d Jacobian product (chunks of 128 steps) and six float row
 * factors per element, which the chunk pass forms and the re-walk reads:
 * about B*T*D*4*7 + B*T*n_heads*(d+2)*d*4/128 bytes. */
size_t pararnn_head_gru_workspace_bytes(int64_t B, int64_t T, int64_t D, int n_heads, int K);

/* K Newton iterations of the head-wise GRU; H_out = h^(K).
 *   workspace  >= pararnn_head_gru_workspace_bytes(B, T, D, n_heads, K)
 *              bytes, 256-byte aligned device memory; no zero-filling needed
 *              (only its 256-byte header is reset, on `stream`).
 *   resid_hist NULL, or K+1 floats: max |F(h^(k))| for k = 0..K.
 * Errors: PARARNN_EINVAL, with nothing launched, for invalid sizes or dtype,
 * a missing or small workspace, and null, host or misaligned pointers;
 * PARARNN_ECUDA if a launch fails.  A non-finite value in H_out is recorded in
 * the workspace and returned by pararnn_status_sync(workspace, stream).  No
 * thread block waits on another, but a block waits on its own tensor-core
 * products; if such a wait runs past 1 s the block stops issuing products and
 * records PARARNN_ETIMEOUT, which pararnn_status_sync() then returns. */
pararnn_status pararnn_head_gru_forward(int64_t B, int64_t T, int64_t D, int n_heads, pararnn_dtype px_dtype,
                                        const void* preacts, const float* U, const float* h0, int K, float* H_out,
                                        void* workspace, size_t ws_bytes, float* resid_hist, void* stream);

/* The adjoint of the head-wise GRU at a trajectory H (normally H_out of
 * pararnn_head_gru_forward), the head-wise counterpart of
 * pararnn_newton_backward: with g_t = dL/dH_t,
 *     lambda_t = g_t + A_{t+1}^T lambda_{t+1},   lambda_{T-1} = g_{T-1},
 * A_{t+1} the head's Jacobian block at (h_t, x_{t+1}); then
 *     dL/dp_z = lambda * alpha, dL/dp_r = lambda * beta,
 *     dL/dp_c = lambda * z (1 - c^2)                     (at (h_{t-1}, x_t)),
 *     dL/dU_g[i][j] = sum over b, t of lambda_i f_{g,i} h_{t-1,j}
 *                     (f = alpha, beta, gamma for g = z, r, c),
 *     dL/dh0 = A_0^T lambda_0,
 * alpha, beta, gamma as in the Jacobian above.  Layouts: H, dL_dH (B, T, D);
 * dL_dpx (B, T, 3, D); dL_dU (3, n_heads, d, d) or NULL; dL_dh0 (B, D) or
 * NULL; all float32 device memory owned by the caller.  dL_dU is summed in a
 * fixed order (no floating-point atomics): repeated calls give identical
 * bits.  Returns the workspace size, or 0 for invalid sizes (as for the
 * forward): about B*T*D*4*6 + B*T*n_heads*(d+2)*d*4/128 bytes (lambda * gamma
 * and five float row factors per element, and the chunk products) plus
 * 12 n_heads d^2 * min(64, B*T/256) * 4 bytes of split partials. */
size_t pararnn_head_gru_backward_workspace_bytes(int64_t B, int64_t T, int64_t D, int n_heads);

/* Errors as for pararnn_head_gru_forward; a non-finite value in dL_dpx is
 * recorded in the workspace for pararnn_status_sync(). */
pararnn_status pararnn_head_gru_backward(int64_t B, int64_t T, int64_t D, int n_heads, pararnn_dtype px_dtype,
                                         const void* preacts, const float* U, const float* h0, const float* H,
                                         const float* dL_dH, float* dL_dpx, float* dL_dU, float* dL_dh0,
                                         void* workspace, size_t ws_bytes, void* stream);

/* The sequential unroll of the head-wise GRU, s_t = f(s_{t-1}, x_t) for
 * t = 0..T-1 with s_{-1} = h0: the one-step recurrence that the Newton
 * forward reproduces at convergence (pararnn-torch page, API overview /
 * Quickstart: sequential_apply beside newton_apply).  One thread block per
 * (batch row, head) walks the sequence with the head's d x d blocks in
 * registers (3 d^2 multiply-adds per step, against the Newton scan's d x d x d
 * products), so it suits problems with many sequences; the Newton forward
 * suits few long ones.  Same layouts and head widths (16, 32, 64) as
 * pararnn_head_gru_forward; preacts must be 16-byte aligned.
 *   workspace  >= 256 bytes of device memory (only its status word is used;
 *              cleared on `stream`)
 * Errors: PARARNN_EINVAL (nothing launched) for bad sizes, dtype, pointers or
 * workspace; PARARNN_ECUDA if the launch fails.  A non-finite value in H_out
 * is recorded for pararnn_status_sync(workspace, stream).  No block waits on
 * another. */
pararnn_status pararnn_head_gru_unroll(int64_t B, int64_t T, int64_t D, int n_heads, pararnn_dtype px_dtype,
                                       const void* preacts, const float* U, const float* h0, float* H_out,
                                       void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PARARNN_B200_H */
