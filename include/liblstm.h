/*
 * liblstm.h -- C ABI of liblstm: the LSTM forward pass and backpropagation
 * through time on one NVIDIA B200 (sm_100a).  lstm_fwd / lstm_bwd run the
 * single-layer, unidirectional operation; lstm_fwd_ex / lstm_bwd_ex add the
 * operator's options (variable length, reverse direction, gate order);
 * lstm_stack_fwd / lstm_stack_bwd run a stack of layers.
 *
 * The operation is the one defined on the "SingleLayerLstmGrad" operator page
 * (CANN ops-nn):
 *   forward-formula table      z_t = [h_{t-1}; x_t]
 *                              i,f,o = sigmoid(W_* z_t + b_*), g = tanh(W_g z_t + b_g)
 *                              c_t = f (.) c_{t-1} + i (.) g,  h_t = o (.) tanh(c_t)
 *   backward algorithm         steps 1-6 (time step t -> t-1), which return the
 *                              gradients of x, W, b, initH and initC.
 *
 * Conventions (all entry points):
 *   - W is the packed weight [4H][H+I], row-major.  Rows are grouped by gate in
 *     the order [i | f | g | o] (gate_order "ifjo", j = g); columns are [h | x],
 *     i.e. W = [W_h | W_x] applied to z_t = [h_{t-1}; x_t].
 *   - One bias b[4H] (same gate grouping); the page's db shape [4, H] is the
 *     same memory.
 *   - Sequences are time-major and row-major: x[T][B][I], y[T][B][H], ...
 *     Row r = t*B + n of a [T*B][.] view is time step t of sequence n.
 *   - "compute type" (lstm_dims.dtype) is the element type of x, W, b, h0, y,
 *     hT, gates, dy and dhT: LSTM_F32 (float, the page's FLOAT), LSTM_BF16
 *     (bfloat16) or LSTM_F16 (IEEE binary16, the page's FLOAT16).  The cell
 *     state (c0, cT, cells, dcT) and every gradient output (dx, dW, db, dh0,
 *     dc0) are float.  Products accumulate in float.  In LSTM_F16 the saved
 *     gates and the gate gradients dG are stored in binary16: gradients below
 *     its range (about 6e-8) flush to zero, as in any fp16 backward without
 *     loss scaling.
 *   - Every pointer is a DEVICE pointer into memory the caller allocated and
 *     owns; it must be 16-byte aligned.  The library allocates no device memory
 *     and keeps no device state between calls; all scratch lives in the
 *     caller's workspace.  (Its process state: the optional profiling record,
 *     a launch counter (see lstm_profile_begin), and per device two internal
 *     streams and a few events that lstm_bwd creates on first use and keeps.)
 *   - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *     stream).  Argument errors are returned synchronously before anything is
 *     enqueued.  Device-side waits that give up record LSTM_ERR_TIMEOUT in the
 *     workspace's status word, which lstm_status() reports.
 *   - Two calls that share a workspace must not run concurrently.
 */
#ifndef LIBLSTM_H
#define LIBLSTM_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define LSTM_OK 0
#define LSTM_ERR_INVALID_ARG 1    /* bad dims, dtype, NULL or misaligned pointer */
#define LSTM_ERR_UNSUPPORTED 2    /* valid arguments this build cannot run */
#define LSTM_ERR_WORKSPACE 3      /* workspace NULL, too small or misaligned */
#define LSTM_ERR_CUDA 4           /* a CUDA runtime call or launch failed */
#define LSTM_ERR_TIMEOUT 5        /* a device-side wait gave up (see lstm_status) */
#define LSTM_ERR_NOT_CORESIDENT 6 /* a persistent grid cannot be fully resident */

/* Compute types. */
#define LSTM_F32 0
#define LSTM_BF16 1
#define LSTM_F16 2

/* Problem sizes: T time steps, B sequences, I input features, H hidden units
 * (parameter table: x [T, batch, input_size], w [4*hidden, input+hidden]).
 * All must be >= 0; T, B or I may be 0 (empty problems are valid). */
typedef struct lstm_dims {
    int T;
    int B;
    int I;
    int H;
    int dtype; /* LSTM_F32, LSTM_BF16 or LSTM_F16 */
} lstm_dims;

/* Workspace bytes lstm_fwd / lstm_bwd need for these dims (0 on invalid dims).
 * The workspace must be 256-byte aligned.
 *
 * The forward's size depends on the plan the call takes on the CURRENT device:
 * when the fused forward kernel runs (the input projection contracted inside
 * the recurrence: 16-bit compute types with H a multiple of 32, I a multiple
 * of 8, and a grid that fits the device) it needs the 256-byte control block
 * only; every other plan also needs the fp32 input projection Gx [T*B][4H].
 *   lstm_fwd_workspace_size     the plan of a call with default options
 *   lstm_fwd_workspace_size_ex  the plan of a call with these options (a
 *                               seq_mask selects other kernel instantiations)
 *   lstm_fwd_workspace_size_max enough for every plan on every device
 * Without a usable device the first two return the _max size.  A forward call
 * whose plan needs more than ws_bytes returns LSTM_ERR_WORKSPACE; if the fused
 * kernel is planned but cannot be launched (LSTM_ERR_NOT_CORESIDENT inside the
 * library), the call falls back to a Gx plan and returns LSTM_ERR_WORKSPACE
 * when ws_bytes is below the _max size.  lstm_bwd_workspace_size does not
 * depend on the device. */
size_t lstm_fwd_workspace_size(const lstm_dims *d);
size_t lstm_bwd_workspace_size(const lstm_dims *d);
size_t lstm_fwd_workspace_size_max(const lstm_dims *d);

/*
 * lstm_fwd -- forward pass ("SingleLayerLstmGrad", forward-formula table).
 *
 *   x     [T][B][I]   compute type  input sequence
 *   W     [4H][H+I]   compute type  packed weights [W_h | W_x], gate rows i,f,g,o
 *   b     [4H]        compute type  bias, or NULL for zero
 *   h0    [B][H]      compute type  initH (h_{-1}), or NULL for zero
 *   c0    [B][H]      float         initC (c_{-1}), or NULL for zero
 * outputs (overwritten):
 *   y     [T][B][H]   compute type  h_t for every step
 *   hT    [B][H]      compute type  h_{T-1} (h0 when T == 0)
 *   cT    [B][H]      float         c_{T-1} (c0 when T == 0)
 *   gates [T][B][4H]  compute type  post-activation i,f,g,o of every step, kept
 *                                    for lstm_bwd (the page's i, j, f, o inputs)
 *   cells [T][B][H]   float         c_t of every step, kept for lstm_bwd
 *   ws / ws_bytes                   scratch, >= lstm_fwd_workspace_size(d) (see there)
 *
 * y, gates and cells must stay unchanged until the matching lstm_bwd has run.
 * Returns LSTM_OK or an LSTM_ERR_* code.
 */
int lstm_fwd(const lstm_dims *d, const void *x, const void *W, const void *b,
             const void *h0, const float *c0, void *y, void *hT, float *cT,
             void *gates, float *cells, void *ws, size_t ws_bytes, void *stream);

/*
 * lstm_bwd -- backpropagation through time ("SingleLayerLstmGrad", backward
 * algorithm steps 1-6 and gradient derivation).  It returns the gradients of
 * the loss L whose partial derivatives the page's dy, dh and dc inputs give:
 *   L = sum_t <dy_t, h_t> + <dhT, h_{T-1}> + <dcT, c_{T-1}>.
 *
 *   dy    [T][B][H]   compute type  dL/dh_t of every step, or NULL for zero
 *   dhT   [B][H]      compute type  gradient at h_{T-1} (page input dh), or NULL
 *   dcT   [B][H]      float         gradient at c_{T-1} (page input dc), or NULL
 *   x, W, h0, c0                    the forward's inputs (h0, c0 may be NULL)
 *   y, gates, cells                 the forward's saved outputs
 * outputs (overwritten, never accumulated):
 *   dx    [T][B][I]   float         dL/dx
 *   dW    [4H][H+I]   float         dL/dW, same layout as W
 *   db    [4H]        float         dL/db (the page's db [4, H])
 *   dh0   [B][H]      float         dL/dinitH (the page's dh_prev at t = 0)
 *   dc0   [B][H]      float         dL/dinitC (the page's dc_prev at t = 0)
 *   ws / ws_bytes                   scratch, >= lstm_bwd_workspace_size(d)
 *
 * On the tensor-core path lstm_bwd may run its recurrence and its dW / dx
 * products on two internal streams of the library (the recurrence at the
 * device's highest stream priority), so that the products of finished time
 * chunks run beside the rest of the recurrence.  Those streams start after
 * the work already enqueued in `stream`, and `stream` waits for both before
 * anything enqueued after the call: the ordering seen on `stream` is that of
 * a single-stream call.  Calls from several host threads are serialised while
 * they enqueue.
 *
 * Returns LSTM_OK or an LSTM_ERR_* code.
 */
int lstm_bwd(const lstm_dims *d, const void *dy, const void *dhT, const float *dcT,
             const void *x, const void *W, const void *h0, const float *c0,
             const void *y, const void *gates, const float *cells, float *dx,
             float *dW, float *db, float *dh0, float *dc0, void *ws, size_t ws_bytes,
             void *stream);

/*
 * lstm_fwd_ex / lstm_bwd_ex -- lstm_fwd / lstm_bwd with the optional input and
 * the attribute of the "SingleLayerLstmGrad" parameter table that plain calls
 * leave at their defaults.  opt NULL (or zero-initialised) = lstm_fwd /
 * lstm_bwd.
 *
 * seq_mask  [T][B][H], compute type: the variable-length input seq_length,
 *   1 = real step, 0 = padding (no other values); NULL = every step real.
 *   The page gives no formula for it.  Reading: at a padded element the state
 *   does not move -- c_t = m c~_t + (1 - m) c_prev, h_t = m h~_t +
 *   (1 - m) h_prev with c~, h~ the unmasked update -- y_t = h_t and
 *   cells_t = c_t (gates are stored as computed), and the backward returns the
 *   exact gradient of that function: padding passes delta h and delta c on
 *   unchanged and has no gate gradient.  With per-sequence lengths
 *   (mask[t][n][:] = t < L_n) every sequence behaves as the LSTM run on its
 *   first L_n steps, carrying its final state through the padding.
 *
 * direction  LSTM_DIR_FORWARD ("UNIDIRECTIONAL": the recurrence runs over
 *   t = 0 .. T-1) or LSTM_DIR_REVERSE ("REDIRECTIONAL": t = T-1 .. 0; h0 / c0
 *   precede the step at t = T-1, hT / cT follow the step at t = 0, dh0 / dc0
 *   are the gradients at h0 / c0).  Tensor layouts are unchanged: y[t], gates[t],
 *   dx[t] ... belong to time t in both directions.  A bidirectional layer is
 *   one call in each direction.  Other values: LSTM_ERR_INVALID_ARG.
 *
 * gate_order  LSTM_GATES_IFJO (the default, "ifjo": the 4H rows of W, b, gates
 *   and dG are the row blocks [i | f | g | o]) or LSTM_GATES_IJFO ("ijfo":
 *   [i | g | f | o], the candidate j = g in block 1 and the forget gate in
 *   block 2).  The attribute only names which row block plays which role; the
 *   arithmetic of every gate is unchanged.  Other values: LSTM_ERR_INVALID_ARG.
 *
 * The backward must receive the options the forward received, and the
 * forward's saved y, gates and cells.  Other arguments, ownership, workspace
 * sizes and errors are those of lstm_fwd / lstm_bwd.
 */
#define LSTM_DIR_FORWARD 0
#define LSTM_DIR_REVERSE 1
#define LSTM_GATES_IFJO 0
#define LSTM_GATES_IJFO 1
typedef struct {
    const void *seq_mask;
    int direction;
    int gate_order;
} lstm_options;

size_t lstm_fwd_workspace_size_ex(const lstm_dims *d, const lstm_options *opt);
int lstm_fwd_ex(const lstm_dims *d, const lstm_options *opt, const void *x, const void *W,
                const void *b, const void *h0, const float *c0, void *y, void *hT, float *cT,
                void *gates, float *cells, void *ws, size_t ws_bytes, void *stream);
int lstm_bwd_ex(const lstm_dims *d, const lstm_options *opt, const void *dy, const void *dhT,
                const float *dcT, const void *x, const void *W, const void *h0,
                const float *c0, const void *y, const void *gates, const float *cells,
                float *dx, float *dW, float *db, float *dh0, float *dc0, void *ws,
                size_t ws_bytes, void *stream);

/*
 * lstm_stack_fwd / lstm_stack_bwd -- a stack of L >= 1 LSTM layers (the
 * multi-layer LSTM module of the "cmu 10-414 HW4" page; "Stack Multiple RNN
 * Cells" of the "mxnet-lstm" page).  Layer 0 reads x [T][B][I]; layer l > 0
 * reads the outputs y of layer l-1.  Every layer has its own weights, bias
 * and initial state, and its final state is an output of its own; only y
 * passes upward.  The stack computes what one lstm_fwd_ex / lstm_bwd_ex call
 * per layer (in that order) computes, with those calls' options, precision
 * and errors.  For 16-bit stacks without a length mask whose layers each fit
 * on half the device, the layers run as a layer wavefront: each layer in
 * chunks of consecutive steps on an internal stream of its own, a layer's
 * chunk after the same chunk of the layer below (forward) or above
 * (backward), all ordered after earlier work on `stream` and before later
 * work on it.  The wavefront's forward plans each layer on half the SMs,
 * whose summation order may differ from the whole-device plan (results
 * within the compute type's tolerance); its backward gives the bits of the
 * layer-by-layer backward.
 *
 * d       sizes and compute type of layer 0; layer l > 0 has I = H.
 * L       number of layers (< 1: LSTM_ERR_INVALID_ARG).
 * W, b    HOST arrays of L DEVICE pointers: W[l] [4H][H + I_l] (I_0 = d->I,
 *         I_l = d->H), b[l] [4H].  b may be NULL (no bias), as may any b[l].
 * h0 [L][B][H] (compute type), c0 [L][B][H] (float): initial states, layer
 *         after layer; either may be NULL (zeros).
 * y [L][T][B][H], gates [L][T][B][4H], cells [L][T][B][H]: every layer's
 *         saved state (the backward reads them); the stack's output is the
 *         slice y[L-1].  hT [L][B][H], cT [L][B][H] (float): final states.
 * opt     as for lstm_fwd_ex, applied to every layer (NULL = defaults).
 * ws      at least lstm_stack_fwd_workspace_size(d, L) bytes.
 * With L > 1 every [L][...] slice must start 16-byte aligned: B*H a
 * multiple of 8 for the 16-bit types, of 4 for float (else
 * LSTM_ERR_UNSUPPORTED).
 *
 * lstm_stack_bwd: dy [T][B][H] (compute type, or NULL) is the gradient at the
 * top layer's outputs; dhT [L][B][H] (compute type) and dcT [L][B][H]
 * (float), either NULL, the gradients at every layer's final state.  Outputs
 * (float): dx [T][B][I]; dW and db, HOST arrays of L DEVICE pointers to
 * dW[l] [4H][H + I_l] and db[l] [4H]; dh0, dc0 [L][B][H].  Layer l-1's dy is
 * layer l's dx rounded to the compute type.  ws:
 * lstm_stack_bwd_workspace_size(d, L) bytes (with the layer wavefront, one
 * layer workspace per layer); a workspace of at least
 * lstm_stack_bwd_workspace_size_min(d, L) bytes (one layer workspace and the
 * dx / dy buffers between two layers) runs the layers one after another,
 * L-1 .. 0; a smaller one is LSTM_ERR_WORKSPACE.
 */
/* (The stack's forward workspace covers every plan of every layer, like
 * lstm_fwd_workspace_size_max.) */
size_t lstm_stack_fwd_workspace_size(const lstm_dims *d, int L);
size_t lstm_stack_bwd_workspace_size(const lstm_dims *d, int L);
size_t lstm_stack_bwd_workspace_size_min(const lstm_dims *d, int L);
int lstm_stack_fwd(const lstm_dims *d, int L, const lstm_options *opt, const void *x,
                   const void *const *W, const void *const *b, const void *h0, const float *c0,
                   void *y, void *hT, float *cT, void *gates, float *cells, void *ws,
                   size_t ws_bytes, void *stream);
int lstm_stack_bwd(const lstm_dims *d, int L, const lstm_options *opt, const void *dy,
                   const void *dhT, const float *dcT, const void *x, const void *const *W,
                   const void *h0, const float *c0, const void *y, const void *gates,
                   const float *cells, float *dx, float *const *dW, float *const *db,
                   float *dh0, float *dc0, void *ws, size_t ws_bytes, void *stream);

/*
 * lstm_status -- synchronise `stream`, then read and clear the device status
 * word kept in the first bytes of a workspace used by lstm_fwd / lstm_bwd.
 * Every call zeroes the word when it starts (in stream order), so it reports
 * the most recent call on that workspace; a fresh workspace needs no
 * initialisation.  Returns LSTM_OK, LSTM_ERR_TIMEOUT (a device-side wait gave
 * up; the results of that call are invalid), LSTM_ERR_CUDA, or
 * LSTM_ERR_INVALID_ARG.
 */
int lstm_status(void *ws, size_t ws_bytes, void *stream);

/*
 * Per-phase device timing (diagnostics, not thread-safe).  Between
 * lstm_profile_begin() and lstm_profile_end(), every lstm_fwd / lstm_bwd call
 * records a CUDA event pair around each phase of the path on its stream and
 * counts the kernels it launches.  lstm_profile_end() waits for those events
 * and writes, per phase, the summed device milliseconds and kernel launches
 * (arrays of LSTM_NUM_PHASES entries; either may be NULL).  Phases:
 */
#define LSTM_PHASE_INPUT_PROJ 0 /* Gx = X W_x^T + b over all T*B rows          */
#define LSTM_PHASE_FWD_RECUR 1  /* the forward recurrence over t = 0..T-1      */
#define LSTM_PHASE_BWD_RECUR 2  /* the backward recurrence over t = T-1..0     */
#define LSTM_PHASE_DW 3         /* dW = dG^T [h_prev | x]                       */
#define LSTM_PHASE_DB 4         /* db = column sums of dG                       */
#define LSTM_PHASE_DX 5         /* dx = dG W_x                                  */
#define LSTM_PHASE_OTHER 6      /* copies, pass-through and set-up launches     */
#define LSTM_NUM_PHASES 7
int lstm_profile_begin(void);
int lstm_profile_end(double *ms, long long *launches);

/* Kernel launches issued by this process's liblstm calls so far. */
long long lstm_launch_count(void);

/*
 * lstm_fwd_noalloc -- the forward pass for callers that may not allocate
 * device memory.  (The paper has no counterpart; this is a deployment aid.)
 *
 * Some callers cannot call cudaMalloc: a plugin inside a host program that owns
 * the whole device-memory budget and forbids allocations it does not make
 * itself, or a latency-critical loop that cannot afford cudaMalloc's implicit
 * device synchronisation.  This entry point takes the same inputs and outputs
 * as lstm_fwd, but instead of a caller workspace it uses a scratch buffer of
 * LSTM_NOALLOC_SCRATCH_BYTES that is a static device array inside the library:
 * every GPU on which the library is loaded holds that buffer until the
 * process exits.  It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 *   - Problems whose lstm_fwd_workspace_size() on the current device exceeds
 *     LSTM_NOALLOC_SCRATCH_BYTES are rejected with LSTM_ERR_UNSUPPORTED
 *     before anything is enqueued.  (Where the fused forward kernel runs the
 *     call needs only the 256-byte control block, at any T and B; other plans
 *     need T*B*4H floats of Gx as well.)
 *   - The first call on a device (the current device) looks up that device's
 *     address of the buffer and keeps it for the life of the process; make
 *     that first call before any stream capture, and do not use this entry
 *     point across a cudaDeviceReset of that device (the kept address would
 *     then be stale).
 *   - All calls share the one buffer per device, which keeps the previous
 *     call's contents; each call clears the parts that must start at zero (the
 *     status word and barrier counters), after its arguments are checked and
 *     in stream order.  Calls whose executions overlap on the GPU (different
 *     streams, or different host threads) race on the buffer: serialise them.
 *   - lstm_fwd_noalloc_status(stream) synchronises `stream` and reads and
 *     clears the buffer's status word on the current device, like lstm_status
 *     does for a caller workspace: it reports a device-side wait that gave up
 *     (LSTM_ERR_TIMEOUT) in the most recent call.
 * Returns LSTM_OK or an LSTM_ERR_* code, like lstm_fwd.
 */
#define LSTM_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int lstm_fwd_noalloc(const lstm_dims *d, const void *x, const void *W, const void *b,
                     const void *h0, const float *c0, void *y, void *hT, float *cT,
                     void *gates, float *cells, void *stream);
int lstm_fwd_noalloc_status(void *stream);

/* Static description of a status code. */
const char *lstm_strerror(int code);

/* ABI version: 100 * major + minor (1.1: lstm_options with gate_order, the
 * LSTM_F16 compute type and the stack entry points; 1.2: the plan-aware
 * forward workspace sizes and lstm_fwd_noalloc_status; 1.3: the stacked
 * layer wavefront and lstm_stack_bwd_workspace_size_min). */
#define LSTM_ABI_VERSION 103
int lstm_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBLSTM_H */
