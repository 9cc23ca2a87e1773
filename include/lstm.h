/*
 * lstm.h -- C ABI of the B200 (sm_100a) LSTM library liblstm_b200.so.
 *
 * Computes the multi-layer, optionally bidirectional 4-gate LSTM forward and
 * its back-propagation-through-time backward on one GPU, asynchronously on a
 * caller-supplied CUDA stream.  Sources of the definitions (web pages, cited
 * by title and section):
 *
 *   [warp_nn]   "Long Short-Term Memory (LSTM)", warp_nn API page: equation
 *               block (gates i, f, g, o; c' = f*c + i*g; h' = o*tanh(c')),
 *               the "Learnable parameters" table (shapes, i|f|g|o row
 *               stacking, _reverse parameters), __call__ parameters/returns
 *               (x (B,T,I); h0/c0/h_n/c_n (D*L,B,H); out (B,T,D*H); zero
 *               default state; ValueError conditions).
 *   [trace]     "Complete Trace: nn.LSTM": Step 1 (batch_first handling,
 *               zero hx default), Step 3 (lstm.input schema: input, hx,
 *               params, has_biases, num_layers, dropout, train,
 *               bidirectional, batch_first -> output, h_n, c_n), Step 5
 *               (workspace / reserveSpace sizing, the backward split into a
 *               data phase and a weight phase).
 *   [mxnet]     "LSTM Forward Computation": Stack Multiple RNN Cells (layer
 *               k+1 reads layer k's output sequence only), Loop Unroll (the
 *               backward is reverse-mode differentiation of the unrolled
 *               loop).
 *   [pulsatrix] pulsatrix LSTMModule: backward() sums every weight and bias
 *               gradient over all timesteps.
 *
 * Notation: L = num_layers, D = 1 + bidirectional, B = batch, T = seq_len,
 * I = input_size, H = hidden_size, G = 4H, in_l = I for l = 0 else D*H.
 *
 * Memory and ownership.  Every data pointer is DEVICE memory owned by the
 * caller; the library never allocates device memory and keeps no state between
 * calls.  The pointer ARRAYS (w_ih, w_hh, b_ih, b_hh, dw_ih, ...) are HOST
 * arrays of length L*D, indexed l*D + d (d = 0 forward, d = 1 reverse, the
 * [warp_nn] _reverse parameters), each entry a device pointer.  Scratch comes
 * from a caller-allocated workspace (size from lstm_workspace_size); training
 * additionally needs a reserve (size from lstm_reserve_size) that the forward
 * fills and the matching backward reads.  Calls that may overlap on the GPU
 * need distinct workspaces.
 *
 * Layouts (row-major, contiguous):
 *   x     (B, T, I) if batch_first else (T, B, I)
 *   out   (B, T, D*H) / (T, B, D*H); forward direction in [0,H), reverse in
 *         [H,2H) at the same time position ([warp_nn])
 *   h0, c0, h_n, c_n, dh0, dc0, grad_hn, grad_cn: (L*D, B, H), index l*D+d
 *   w_ih[l*D+d] (G, in_l); w_hh[l*D+d] (G, H); b_ih, b_hh: G values.  The G
 *   rows are the four gate blocks in the order i, f, g, o.
 *
 * Types: lstm_desc.dtype selects the storage type of x, h0, weights, biases,
 * out, h_n, grad_out, grad_hn, dx and dh0 (float32 or bf16).  Cell states
 * (c0, c_n, grad_cn, dc0) are always float32, and so are the weight and bias
 * gradients.  Arithmetic accumulates in float32.
 *
 * Errors: functions return an lstm_status.  Argument errors are detected on
 * the host before anything is enqueued.  Kernel-side failures (a bounded wait
 * that gave up) are written to a status word inside the workspace and read by
 * lstm_query_status.
 */
#ifndef LSTM_B200_H
#define LSTM_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

typedef enum {
    LSTM_OK = 0,
    LSTM_ERR_INVALID_ARG = 1,  /* bad size, NULL required pointer, num_layers < 1
                                  ([warp_nn] ValueError cases) */
    LSTM_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
    LSTM_ERR_WORKSPACE = 3,    /* workspace or reserve smaller than the query */
    LSTM_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    LSTM_ERR_TIMEOUT = 5       /* a kernel's bounded inter-block wait gave up */
} lstm_status;

typedef enum { LSTM_F32 = 0, LSTM_BF16 = 1 } lstm_dtype;

typedef struct {
    int input_size;     /* I >= 1 */
    int hidden_size;    /* H >= 1 */
    int num_layers;     /* L >= 1 ([warp_nn]: ValueError if < 1) */
    int bidirectional;  /* 0 or 1 */
    int bias;           /* 0: b_ih/b_hh ignored and treated as zero, db not written */
    int batch_first;    /* 1: x/out/grad_out/dx are (B,T,.); 0: (T,B,.) */
    int batch;          /* B >= 0 */
    int seq_len;        /* T >= 0; T == 0 gives h_n = h0, c_n = c0 */
    lstm_dtype dtype;
    /* Inter-layer dropout of the training forward ([trace] Step 3: the
     * dropout argument of the LSTM op), 0 <= dropout < 1; 0 = none.  Applied
     * only when lstm_forward gets a reserve, to the outputs of layers
     * 0..L-2 before they enter the next layer; the backward replays the
     * same mask.  Element e = (t*B + b)*(D*H) + k of layer l's time-major
     * output is kept iff (w >> 11) >= ceil(dropout * 2^53), w = word e mod 4
     * of Philox4x64-10 (Salmon et al. 2011) with key (dropout_seed, l) and
     * counter (e / 4, 0, 0, 0); kept elements are scaled by 1/(1-dropout). */
    float dropout;
    unsigned long long dropout_seed;
} lstm_desc;

/* Workspace bytes needed by lstm_forward and lstm_backward for this
 * description (one size serves both).  0 if the description is invalid. */
size_t lstm_workspace_size(const lstm_desc* desc);

/* Reserve bytes a training forward fills for the backward: per (layer,
 * direction) the gate activations i, f, g, o and the cell state c of every
 * step, and per layer its output sequence ([trace] Step 5, reserveSpace).
 * 0 if the description is invalid. */
size_t lstm_reserve_size(const lstm_desc* desc);

/*
 * Forward ([warp_nn] equation block, [mxnet] Stack Multiple RNN Cells).
 *   x, w_ih, w_hh (and b_ih, b_hh when desc->bias): inputs, required.
 *   h0, c0: initial states or NULL for zeros ([trace] Step 1; [warp_nn]).
 *   out, h_n, c_n: outputs, required when B*T (resp. B) > 0.
 *   workspace/ws_bytes: scratch, at least lstm_workspace_size bytes,
 *     256-byte aligned.
 *   reserve/rs_bytes: NULL for inference; otherwise at least
 *     lstm_reserve_size bytes, filled for lstm_backward.
 * Enqueued on `stream`; returns before the GPU finishes.  Only
 * stream-ordered work is enqueued (no host synchronisation), so a call may be
 * captured into a CUDA graph and replayed.
 * LSTM_F32 runs the input projection, and where a tensor-core plan fits (H a
 * multiple of 128 from 256 to 1024, batch groups of at most 64 rows) the
 * recurrent product W_hh h_{t-1} too, as 3xTF32: each operand is split into
 * its tf32 part and the float32 remainder and the three larger cross
 * products are summed in float32 (the remainder-by-remainder term, relative
 * size 2^-22, is dropped); gates and cell update in float32.  LSTM_BF16
 * multiplies bf16 operands on the tensor cores with float32 sums and cell
 * arithmetic; h_t is rounded to bf16 where it is stored.  (Other shapes, or
 * LSTM_B200_REC=simt, run the recurrence on the CUDA cores in float32.)
 */
lstm_status lstm_forward(const lstm_desc* desc, const void* x, const void* h0, const float* c0,
                         const void* const* w_ih, const void* const* w_hh,
                         const void* const* b_ih, const void* const* b_hh,
                         void* out, void* h_n, float* c_n,
                         void* workspace, size_t ws_bytes,
                         void* reserve, size_t rs_bytes, cudaStream_t stream);

/*
 * Backward (BPTT, [mxnet] Loop Unroll; [pulsatrix] backward(); data then
 * weight phase as in [trace] Step 5, cuDNN Backward).  Must follow an
 * lstm_forward with a reserve, on the same x, h0, c0 and weights.
 *   grad_out: gradient of the loss w.r.t. out (same layout), required.
 *   grad_hn, grad_cn: gradients w.r.t. h_n, c_n or NULL for zeros.
 *   dx (layout of x), dh0, dc0 (L*D, B, H): input-gradient outputs.
 *   dw_ih, dw_hh, db_ih, db_hh: host arrays of L*D device pointers to float32
 *     gradients, OVERWRITTEN (not accumulated); db arrays ignored if !bias.
 *     db_ih and db_hh receive the same values (the biases enter as a sum).
 * LSTM_F32 computes in float32: 3xTF32 tensor-core products in the weight
 * phase and, where a tensor-core plan fits (H = 128, 256 or 512, batch groups
 * of at most 64 rows), in the recurrent products W_hh^T da too (operands
 * split as in the forward); gate derivatives, carries and sums in float32.
 * LSTM_BF16 keeps the cell arithmetic, the dc carry and every sum in
 * float32, with bf16 products on the tensor cores: the recurrent products
 * W_hh^T da take the previous step's gate gradients rounded to bf16, and the
 * weight phase takes the gate gradients rounded to bf16 (x, the saved layer
 * outputs and W_ih are exact in bf16); dx and dh0 are rounded to bf16
 * (nearest even) at the end, the weight and bias gradients stay float32.
 * (Shapes outside the tensor-core plans, or LSTM_B200_REC=simt, run the
 * recurrence on the CUDA cores in float32.)  LSTM_ERR_UNSUPPORTED only when
 * no recurrent plan fits the device.
 */
lstm_status lstm_backward(const lstm_desc* desc, const void* x, const void* h0, const float* c0,
                          const void* const* w_ih, const void* const* w_hh,
                          const void* grad_out, const void* grad_hn, const float* grad_cn,
                          const void* reserve, size_t rs_bytes,
                          void* workspace, size_t ws_bytes,
                          void* dx, void* dh0, float* dc0,
                          float* const* dw_ih, float* const* dw_hh,
                          float* const* db_ih, float* const* db_hh, cudaStream_t stream);

/*
 * Variable-length batches ([trace] Step 3: the packed-sequence overload of
 * the LSTM op; [mxnet] Sequence Buckets: sequences padded to a fixed
 * length).  `lengths` is a device array of desc->batch int32 values: row b
 * of the padded x holds lengths[b] valid steps (values above seq_len act as
 * seq_len, below 0 as 0); NULL means every row has seq_len steps, which is
 * lstm_forward / lstm_backward.  Row b is the ordinary problem on its first
 * lengths[b] steps: the reverse direction starts at step lengths[b] - 1, out
 * is 0 at padded positions, h_n / c_n hold each row's final states, the
 * padding of grad_out is ignored and dx is 0 there.  Arguments, buffers and
 * errors are otherwise those of lstm_forward / lstm_backward; the backward
 * takes the same lengths as its forward.
 */
lstm_status lstm_forward_varlen(const lstm_desc* desc, const int* lengths, const void* x, const void* h0,
                                const float* c0, const void* const* w_ih, const void* const* w_hh,
                                const void* const* b_ih, const void* const* b_hh,
                                void* out, void* h_n, float* c_n,
                                void* workspace, size_t ws_bytes,
                                void* reserve, size_t rs_bytes, cudaStream_t stream);
lstm_status lstm_backward_varlen(const lstm_desc* desc, const int* lengths, const void* x, const void* h0,
                                 const float* c0, const void* const* w_ih, const void* const* w_hh,
                                 const void* grad_out, const void* grad_hn, const float* grad_cn,
                                 const void* reserve, size_t rs_bytes,
                                 void* workspace, size_t ws_bytes,
                                 void* dx, void* dh0, float* dc0,
                                 float* const* dw_ih, float* const* dw_hh,
                                 float* const* db_ih, float* const* db_hh, cudaStream_t stream);

/*
 * Inference forward that allocates nothing and takes no workspace.  The pages
 * have no counterpart: this is an integration aid.  It exists for callers
 * that cannot call cudaMalloc or size a workspace for us, such as a plugin
 * running inside a host application that owns every byte of device memory
 * and forbids its plugins to allocate, or a loop on a fixed memory budget
 * where an allocation could fail or stall at an unpredictable moment.
 *
 * Same arguments and results as lstm_forward with reserve == NULL; the caller
 * still passes every input and output.  The scratch is one fixed array of
 * LSTM_NOALLOC_SCRATCH_BYTES (32 MiB) of device memory inside the library,
 * present on every GPU where the library's device code is loaded until the
 * process exits.  Problems whose inference workspace exceeds it return
 * LSTM_ERR_WORKSPACE; use lstm_forward with your own workspace for those.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call shares the one array: calls that may overlap on the
 * GPU (other streams, other host threads) race and must be serialised by the
 * caller.  The status word of a call (LSTM_ERR_TIMEOUT after a bounded wait
 * gave up) lives in the array too; read it with lstm_noalloc_query_status.
 * Errors: LSTM_ERR_INVALID_ARG for an invalid description or pointer,
 * LSTM_ERR_UNSUPPORTED when no recurrent plan fits the device,
 * LSTM_ERR_WORKSPACE as above, LSTM_ERR_CUDA when the array's address cannot
 * be looked up.  A cudaDeviceReset invalidates the address cached for that
 * device; do not call this entry point on a device after resetting it.
 */
#define LSTM_NOALLOC_SCRATCH_BYTES (32u << 20)

lstm_status lstm_forward_noalloc(const lstm_desc* desc, const void* x, const void* h0,
                                 const float* c0, const void* const* w_ih, const void* const* w_hh,
                                 const void* const* b_ih, const void* const* b_hh,
                                 void* out, void* h_n, float* c_n, cudaStream_t stream);

/* Synchronises `stream` and returns the kernel-side status that the last
 * lstm_forward_noalloc on the current device recorded in the library's
 * scratch array (LSTM_OK or LSTM_ERR_TIMEOUT), or LSTM_ERR_CUDA if the stream
 * reports an error.  No counterpart on the pages (see lstm_forward_noalloc). */
lstm_status lstm_noalloc_query_status(cudaStream_t stream);

/* Synchronises `stream` and returns the kernel-side status recorded in
 * `workspace` by the last call that used it (LSTM_OK or LSTM_ERR_TIMEOUT), or
 * LSTM_ERR_CUDA if the stream reports an error.  A kernel's inter-block or
 * barrier wait gives up after 2 s, or after LSTM_B200_WAIT_TIMEOUT_NS
 * nanoseconds when that environment variable is set (read once per
 * process); the kernel then records LSTM_ERR_TIMEOUT, drains the copies it
 * has in flight and returns, leaving the CUDA context usable. */
lstm_status lstm_query_status(void* workspace, cudaStream_t stream);

/* Static string naming a status code. */
const char* lstm_status_string(lstm_status status);

/*
 * Kernel timing (instrumentation; the pages define no counterpart).  While
 * enabled, the library brackets every kernel it launches with a pair of CUDA
 * events on the launching stream.  lstm_timing_read waits for the recorded
 * events, adds their durations to per-kind totals and copies up to
 * max_entries {name, launches, total_ms} records into `out` (a host array);
 * it returns the number of records written (the number of kinds when out is
 * NULL), or -1 if an event could not be read.  Kinds (the suffix names the
 * engine: _tc tensor cores, _ffma / _simt CUDA cores): pack, proj_gemm_tc,
 * proj_gemm_simt, fwd_rec_tc, fwd_rec_ffma, bwd_rec_tc, bwd_rec_ffma,
 * dw_gemm_tc, dw_gemm_simt, dx_gemm_tc, dx_gemm_simt, db_reduce, seq_copy,
 * transpose, dropout.
 * lstm_timing_reset
 * zeroes the totals.  Process-wide and thread-safe; event recording adds a
 * few microseconds per launch, so leave it off outside measurements.
 */
typedef struct {
    const char* name;       /* static string */
    long long launches;
    double total_ms;
} lstm_kernel_time;

lstm_status lstm_timing_enable(int enable);
int lstm_timing_read(lstm_kernel_time* out, int max_entries);
void lstm_timing_reset(void);

/*
 * Per-step timeline of a recurrent kernel (instrumentation; the pages define
 * no counterpart).  While enabled, every recurrent launch has thread(s) of
 * block 0 stamp %globaltimer (ns) at fixed points of each step into a static
 * device buffer of LSTM_TRACE_MAX_STEPS x LSTM_TRACE_EVENTS entries, zeroed
 * before the launch; each launch overwrites the previous one, so after a
 * multi-layer call the buffer holds the last recurrent launch.
 * lstm_trace_read copies min(max_steps, steps of that launch) rows of
 * LSTM_TRACE_EVENTS values into `out` (host memory) and returns the number of
 * rows (0 if nothing was traced, -1 on a CUDA error); *kind (if non-null)
 * receives the kernel, LSTM_TRACE_*.  The caller synchronises the launch's
 * stream first.  Unused events stay 0.  Events by kernel:
 *   LSTM_TRACE_FWD_REC_FFMA: 0 step start, 1 group wait done, 2 h tile in
 *     shared memory, 3 matvec done (first batch sub-tile), 4 cell update
 *     done, 5 arrival published.
 *   LSTM_TRACE_BWD_REC_FFMA: 0 step start, 1 group wait done, 2 partial-dh
 *     gather done, 3 gate gradients done (first sub-tile), 4 partial dh
 *     products done, 5 arrival published.
 *   LSTM_TRACE_FWD_REC_TC: 0 producer passed the group wait, 1 last h TMA
 *     issued, 2 accumulator initialised (MMA thread), 9 first h chunk landed,
 *     3 MMAs committed, 4 epilogue saw the MMAs complete, 5 partial sums sent
 *     to the partner block, 6 partner's partial sums received, 7 cell update
 *     done, 8 h_t published, 10 Gx of this step loaded into the accumulator
 *     (stamped at the end of the previous step).
 *   LSTM_TRACE_FWD_REC_TC32: 0 producer passed the group wait, 9 h tiles
 *     landed (first issuer), 3 its MMAs committed, 4 epilogue saw all MMAs
 *     complete, 5 partial sums sent to the column owners, 6 the owners'
 *     partial sums received, 7 cell update done, 8 h_t published.
 *   LSTM_TRACE_BWD_REC_TC32 (row s = iteration s, 1..T): 0 producer passed
 *     the group wait, 9 da tiles landed (first issuer), 3 its MMAs
 *     committed, 4 epilogue saw all MMAs complete, 5 partial sums sent to the
 *     unit owners, 6 the owners' partial sums received, 7 gate gradients
 *     done; 8 (stamped in the next row) gate gradients published.
 * Process-wide; tracing adds one timer read and store per event to block 0.
 */
#define LSTM_TRACE_MAX_STEPS 512
#define LSTM_TRACE_EVENTS 16
enum {
    LSTM_TRACE_FWD_REC_FFMA = 1,
    LSTM_TRACE_BWD_REC_FFMA = 2,
    LSTM_TRACE_FWD_REC_TC = 3,
    LSTM_TRACE_FWD_REC_TC32 = 4,
    LSTM_TRACE_BWD_REC_TC32 = 5
};

lstm_status lstm_trace_enable(int enable);
int lstm_trace_read(unsigned long long* out, int max_steps, int* kind);

#ifdef __cplusplus
}
#endif

#endif /* LSTM_B200_H */
