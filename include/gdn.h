/*
 * gdn.h -- C ABI of libgdn: the Gated DeltaNet gated delta-rule recurrence on
 * NVIDIA B200 (sm_100a).
 *
 * The operation.  A Gated DeltaNet layer keeps, per value head, a fixed-size
 * state S (d_v x d_k, float32) and updates it once per token with the delta
 * rule of the Qwen3.8-27B architecture page (2kiu.com, "From parameter race to
 * efficiency revolution: dissecting Qwen3.8-27B's dense architecture and
 * long-context hybrid attention", section 2.2): the value stored under key k_t
 * is erased and v_t written with strength beta_t.  The layer is gated: a decay
 * alpha_t scales the erased state,
 *
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = scale * S_t q_t,
 *     alpha_t = exp(-exp(A_log) * softplus(a_t + dt_bias)),  beta_t = sigmoid(b_t),
 *
 * with the per-layer parameters A_log, dt_bias and the per-token inputs a, b
 * named by that page's weight list (A_log, dt_bias, in_proj_a, in_proj_b,
 * section 2.1; the page gives no gate formula, this is the reading the library
 * implements).  Section 2.1 fixes the shape this library is built for: 16 key
 * heads (q, k), 48 value heads, head width 128; value head h reads key head
 * h / (Hv / Hqk).  Section 2.2 keeps the state in float32.  Before the
 * recurrence, q, k and v go through a causal depthwise convolution of width 4
 * (linear_conv_kernel_dim = 4 and conv1d.weight, section 2.1), SiLU, and an L2
 * normalisation of q and k per head.
 *
 * Conventions for every entry point.
 *  - Memory.  Every pointer argument is a DEVICE pointer unless stated
 *    otherwise; the caller owns all memory.  The library never allocates,
 *    frees or synchronises, and enqueues all work on `stream` (NULL = the
 *    legacy default stream).  Results are ready when the stream reaches them.
 *    (gdn_layer_prefill_host also uses two caller-given copy streams and
 *    creates and releases CUDA events to order them; gdn_prefill_status waits
 *    for its stream, as documented there.)
 *  - Types.  bf16 tensors are passed as uint16_t bit patterns.  Layouts are
 *    dense row-major in the order written; "[T, H, d]" means d is contiguous.
 *  - Alignment.  Every tensor pointer must be 16-byte aligned
 *    (GDN_ERR_MISALIGNED otherwise).
 *  - Aliasing.  Inputs and outputs must not overlap, except where stated.
 *  - Errors.  Arguments are checked on the host first; on any error nothing is
 *    launched and the status says why.  A failed launch returns GDN_ERR_CUDA.
 *    Device code never traps or asserts.
 *  - Sequences.  cu_seqlens (int32, device, [n_seq + 1], non-decreasing,
 *    cu_seqlens[0] = 0, cu_seqlens[n_seq] = T) packs n_seq sequences along the
 *    token axis; NULL means one sequence of length T (n_seq must be 1).  No
 *    state, history or chunk crosses a sequence boundary.  Sequences of
 *    length 0 are allowed.  The library trusts cu_seqlens' contents.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA stream type (cudaStream_t / CUstream), declared without CUDA headers. */
struct CUstream_st;
typedef struct CUstream_st* gdn_stream_t;

typedef enum gdn_status {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* NULL required pointer, negative size, inconsistent sizes */
    GDN_ERR_UNSUPPORTED = 2,   /* a shape the kernels do not implement (d != 128, Hv % Hqk != 0) */
    GDN_ERR_MISALIGNED = 3,    /* a tensor pointer that is not 16-byte aligned */
    GDN_ERR_CUDA = 4,          /* a CUDA call or kernel launch failed (see gdn_last_cuda_error) */
    GDN_ERR_TIMEOUT = 5,       /* a bounded wait inside a kernel ran out (prefill only) */
    GDN_ERR_WORKSPACE = 6      /* workspace NULL or below the least size gdn_prefill accepts */
} gdn_status;

/* Version of this ABI; bumped when a signature or a layout changes. */
#define GDN_ABI_VERSION 1
int gdn_abi_version(void);

/* Static, NUL-terminated description of a status code (never NULL). */
const char* gdn_status_string(int status);

/* The last CUDA error code seen by a call that returned GDN_ERR_CUDA in this
 * process (0 if none), and its name.  Informational; not thread-safe. */
int gdn_last_cuda_error(void);
const char* gdn_last_cuda_error_string(void);

/*
 * gdn_conv1d_silu -- the layer's front end: causal depthwise 4-tap convolution
 * over time for every channel, SiLU on every channel, then q and k divided per
 * head by sqrt(sum of squares + 1e-6).  Width-4 causal convolution and
 * conv1d.weight: architecture page section 2.1.
 *
 *  qkv            [T, Ctot] bf16, Ctot = (2 Hqk + Hv) d; channels ordered
 *                 [q heads 0..Hqk-1 | k heads 0..Hqk-1 | v heads 0..Hv-1],
 *                 each head d channels.
 *  conv_w         [Ctot, 4] float32; tap j multiplies x[t - 3 + j] (tap 3 is
 *                 the current token).  No bias.
 *  conv_state_in  [n_seq, Ctot, 3] float32 or NULL: the three inputs before
 *                 each sequence's first token, oldest first (NULL: zeros).
 *  conv_state_out [n_seq, Ctot, 3] float32 or NULL: receives the last three
 *                 inputs of each sequence, oldest first (positions before the
 *                 sequence start come from conv_state_in), so that a later
 *                 call can continue the sequences.  Must not overlap
 *                 conv_state_in.
 *  q, k           [T, Hqk, d] bf16 outputs;  v  [T, Hv, d] bf16 output.
 * Arithmetic is float32; outputs are rounded to bf16 (nearest even).
 * Supported: d = 128, Hqk >= 1, Hv >= 1.
 */
gdn_status gdn_conv1d_silu(const uint16_t* qkv, const float* conv_w, const int32_t* cu_seqlens,
                           int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv, int32_t d,
                           const float* conv_state_in, float* conv_state_out,
                           uint16_t* q, uint16_t* k, uint16_t* v, gdn_stream_t stream);

/*
 * gdn_conv1d_silu_backward_workspace_size -- bytes of device workspace
 * gdn_conv1d_silu_backward needs: per-tile sums of the weight gradient,
 * ceil(T / 32) * (2 Hqk + Hv) * d * 4 floats, rounded up to 256 bytes (0 for
 * T = 0).  Host-only.
 */
size_t gdn_conv1d_silu_backward_workspace_size(int64_t T, int32_t Hqk, int32_t Hv, int32_t d);

/*
 * gdn_conv1d_silu_backward -- the gradient of gdn_conv1d_silu (the front end:
 * 4-tap causal depthwise conv1d, SiLU, L2 norm of each q and k head; the
 * architecture page, section 2.1, gives the conv width) given dL/dq, dL/dk and
 * dL/dv.  Reverse mode, recomputing the forward from qkv:
 *     da = (dout - out <dout, out>) / n  for q and k heads (n the head's norm),
 *     da = dout for v;  dy = da (sigma(y) + a (1 - sigma(y))) with a = silu(y);
 *     d qkv[t] = sum_j w[c, j] dy[t + 3 - j] over tokens of t's sequence;
 *     d conv_w[c, j] = sum over all tokens of dy[t] x~[t - 3 + j];
 *     d conv_state: the taps of a sequence's first three tokens that read its
 *     history (x~ is the history, or zero, before the first token).
 * Inputs as for gdn_conv1d_silu (qkv [T, Ctot] bf16, conv_w [Ctot, 4],
 * cu_seqlens, conv_state [n_seq, Ctot, 3] or NULL for a zero history), plus
 *  dq, dk  [T, Hqk, d] float32,  dv [T, Hv, d] float32.
 * Outputs (float32, overwritten; caller-owned):
 *  d_qkv        [T, Ctot]
 *  d_conv_w     [Ctot, 4]
 *  d_conv_state [n_seq, Ctot, 3] or NULL (not written); with conv_state NULL
 *               it is the gradient at a zero history.
 * workspace: gdn_conv1d_silu_backward_workspace_size() bytes, 256-byte aligned
 * (may be NULL when that is 0).  Supported: d = 128.  CUDA cores, float32, one
 * CTA per (32-token tile, head); sums in a fixed order, so the result is
 * deterministic.  Errors as for gdn_conv1d_silu, plus GDN_ERR_WORKSPACE.
 */
gdn_status gdn_conv1d_silu_backward(const uint16_t* qkv, const float* conv_w, const int32_t* cu_seqlens,
                                    int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv, int32_t d,
                                    const float* conv_state, const float* dq, const float* dk, const float* dv,
                                    float* d_qkv, float* d_conv_w, float* d_conv_state, void* workspace,
                                    size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_prefill_workspace_size -- bytes of device workspace with which
 * gdn_prefill runs its fastest kernel for these sizes (a multiple of 256; never
 * 0).  Host-only, no CUDA calls.  That kernel passes each chunk's
 * state-independent operands from producer to consumer CTAs through a ring of
 * 8 slots of 49664 bytes plus 128 bytes of counters per (sequence, value head)
 * of one launch, and a launch holds at most 64 of them, so the size is
 * 256 + 397440 * min(n_seq * Hv, 64) bytes (rounded up to 256).  A smaller
 * workspace that holds at least one such ring runs fewer (sequence, value head)
 * pairs per launch.  gdn_prefill also accepts a workspace as small as
 * 256 + 4 * n_seq * Hv bytes (rounded up to 256) and then runs a single-CTA
 * kernel with the same results up to rounding.
 */
size_t gdn_prefill_workspace_size(int32_t n_seq, int64_t T, int32_t Hqk, int32_t Hv, int32_t d);

/*
 * gdn_prefill -- the recurrence over packed sequences, computed in chunks of
 * 64 tokens (WY / UT form: decay-masked beta K K^T, (I + A)^{-1} by forward
 * substitution, W and U, the intra-chunk output, then the inter-chunk state
 * scan), with products on the tensor cores in bf16 and float32 accumulation,
 * and the state carried in float32 (architecture page section 2.2: float32
 * state).
 *
 *  q, k           [T, Hqk, d] bf16 (the recurrence uses them as given; the
 *                 front end normalises them).
 *  v              [T, Hv, d] bf16.
 *  a, b           [T, Hv] float32 per-token gate inputs.
 *  A_log, dt_bias [Hv] float32 per-head gate parameters.
 *  scale          output scale (1/sqrt(d) for the layer).
 *  initial_state  [n_seq, Hv, d_v, d_k] float32 (d_k contiguous) or NULL (zeros).
 *  final_state    [n_seq, Hv, d_v, d_k] float32 or NULL (not written).  May be
 *                 the same pointer as initial_state (updated in place).
 *  o              [T, Hv, d] float32 output.
 *  workspace      device scratch, 256-byte aligned, of
 *                 gdn_prefill_workspace_size() bytes (or at least the smaller
 *                 size given there, for the single-CTA kernel); its contents
 *                 on entry do not matter.  Calls that share a workspace must be
 *                 ordered on one stream.
 * A sequence of length 0 leaves final_state = initial_state (or zeros).
 * Supported: d = 128, Hv % Hqk == 0.
 * Kernel choice: with a workspace that holds at least one ring (see
 * gdn_prefill_workspace_size), a cooperative grid of one consumer CTA (the
 * state chain) and two or one producer CTAs (the state-independent chunk
 * algebra) per (sequence, value head), in launches of as many pairs as fit on
 * the device at once; otherwise one CTA per (sequence, value head, half of d).
 * The environment variables GDN_PREFILL_KERNEL (=pc or =single) and
 * GDN_PREFILL_PRODUCERS (=1 or =2) force a choice; a forced producer /
 * consumer kernel that cannot run returns GDN_ERR_UNSUPPORTED.
 * GDN_ERR_TIMEOUT is not returned here (the kernel does not stop the host):
 * a kernel that gave up on a bounded wait records it in the workspace, and
 * gdn_prefill_status() reports it.
 */
gdn_status gdn_prefill(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                       const float* b, const float* A_log, const float* dt_bias,
                       const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                       int32_t Hv, int32_t d, float scale, const float* initial_state,
                       float* final_state, float* o, void* workspace, size_t workspace_bytes,
                       gdn_stream_t stream);

/*
 * gdn_prefill_bf16 -- gdn_prefill with the output o stored as bf16 (rounded to
 * nearest even from the same float32 values) instead of float32: the bf16
 * output variant.  The architecture page (section 2.2) puts the layer's state
 * in float32 and gives a ~75 MB figure for the 48 layers' state at 2 bytes per
 * element; o is the activation that leaves the recurrence, and halving its
 * bytes cuts the prefill's algorithmic traffic from 45,440 to 33,152 bytes per
 * token (16 / 48 heads, d = 128).  Arguments, layouts, ownership and errors as
 * gdn_prefill, except
 *  o  [T, Hv, d] bf16 (uint16 bits), written; 16-byte aligned.
 * The state (initial_state, final_state) stays float32.
 */
gdn_status gdn_prefill_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                            const float* b, const float* A_log, const float* dt_bias,
                            const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                            int32_t Hv, int32_t d, float scale, const float* initial_state,
                            float* final_state, uint16_t* o, void* workspace, size_t workspace_bytes,
                            gdn_stream_t stream);

/*
 * gdn_layer_prefill_host_workspace_size -- bytes of device workspace that
 * gdn_layer_prefill_host needs for T tokens cut into n_blocks ranges: a prefill
 * workspace for one range (first, so that its error word is this workspace's
 * first word), two input buffers of a range (qkv, a, b), q/k/v of a range, two
 * output buffers of a range, two conv histories and two states.  0 for
 * unsupported arguments.  Host-only.
 */
size_t gdn_layer_prefill_host_workspace_size(int64_t T, int32_t Hqk, int32_t Hv, int32_t d, int32_t n_blocks);

/*
 * gdn_layer_prefill_host -- gdn_conv1d_silu then gdn_prefill for one sequence,
 * from HOST inputs to HOST outputs, with the host<->device copies overlapped
 * with the compute (the operation is that of the two calls; architecture page
 * sections 2.1 and 2.2).  The T tokens are cut into n_blocks ranges of whole
 * 64-token chunks, the first a quarter as long as the others (so that the first
 * download, the longer copy direction, starts early): range r's inputs are
 * copied up on `upload_stream` into one of two device buffers; its front end
 * (continuing range r-1's conv history) and prefill (continuing range r-1's
 * state) run on `stream`; its output is copied down on `download_stream` from
 * one of two output buffers.  Range r+1's upload and range r-1's download thus
 * run while range r computes.  The result equals the two device calls on the
 * whole sequence within the prefill's tolerance (the state is handed between
 * ranges in float32; gdn_prefill's own chunking runs unchanged inside each).
 *  h_qkv          [T, (2 Hqk + Hv) d] bf16, HOST (pinned: page-locked host
 *                 memory is what lets the copies overlap)
 *  h_a, h_b       [T, Hv] float32, HOST (pinned)
 *  conv_w, A_log, dt_bias   device, as for gdn_conv1d_silu / gdn_prefill
 *  conv_state_in  [(2 Hqk + Hv) d, 3] float32 device, or NULL (zero history)
 *  initial_state  [Hv, d, d] float32 device, or NULL (zero state)
 *  h_o            [T, Hv, d] float32, HOST (pinned), written
 *  h_final_state  [Hv, d, d] float32, HOST (pinned), written
 *  conv_state_out [(2 Hqk + Hv) d, 3] float32 device, or NULL
 *  workspace      gdn_layer_prefill_host_workspace_size() bytes, 256-byte aligned
 *  stream, upload_stream, download_stream: three distinct streams.
 * The call only enqueues work and returns; everything it enqueues is ordered
 * before work enqueued on `stream` afterwards (the host outputs are ready when
 * `stream` reaches that point), and its device-side reads of the workspace wait
 * for work enqueued on `stream` before the call.  It creates CUDA events for
 * the ordering and releases them before returning (the driver keeps them until
 * the work they mark completes); it allocates no memory.  n_blocks in
 * [1, 4096].  Errors as for gdn_prefill; a timeout inside a range's prefill sets
 * the workspace's error word (gdn_prefill_status / gdn_check_async on this
 * workspace).  Supported: d = 128.
 */
gdn_status gdn_layer_prefill_host(const uint16_t* h_qkv, const float* h_a, const float* h_b, const float* conv_w,
                                  const float* A_log, const float* dt_bias, const float* conv_state_in,
                                  const float* initial_state, int64_t T, int32_t Hqk, int32_t Hv, int32_t d,
                                  float scale, int32_t n_blocks, float* h_o, float* h_final_state,
                                  float* conv_state_out, void* workspace, size_t workspace_bytes,
                                  gdn_stream_t stream, gdn_stream_t upload_stream, gdn_stream_t download_stream);

/*
 * gdn_prefill_status -- waits for `stream`, then reads the error word that the
 * last gdn_prefill on this workspace left: GDN_OK, or GDN_ERR_TIMEOUT if a
 * bounded wait inside the kernel ran out (the outputs are then invalid).
 * workspace NULL: the library-owned array that gdn_prefill_noalloc uses on the
 * current device.  Synchronises the stream; not for use inside stream capture
 * (gdn_check_async is the form that does not wait).
 */
gdn_status gdn_prefill_status(const void* workspace, gdn_stream_t stream);

/*
 * gdn_check_async -- the non-waiting error check (library error reporting; the
 * pages define no interface).  Enqueues on `stream` a copy of the workspace's
 * error word into *status_word and returns at once: nothing is synchronised,
 * so it may follow gdn_prefill inside a stream capture.  Once the stream has
 * passed that point, *status_word is 0 if every bounded wait of the prefills
 * that used this workspace before it succeeded, nonzero if one ran out (their
 * outputs are then invalid; gdn_prefill_status would report GDN_ERR_TIMEOUT).
 *  workspace    the prefill's workspace, or NULL for the library-owned array
 *               of gdn_prefill_noalloc on the current device.
 *  status_word  4-byte aligned uint32 in device memory or in page-locked host
 *               memory (with pageable host memory the copy may wait for the
 *               stream); owned by the caller.
 * Errors: GDN_ERR_INVALID_ARG (status_word NULL), GDN_ERR_MISALIGNED,
 * GDN_ERR_CUDA (the copy could not be enqueued).
 */
gdn_status gdn_check_async(const void* workspace, uint32_t* status_word, gdn_stream_t stream);

/*
 * gdn_prefill_noalloc -- gdn_prefill for callers that cannot allocate device
 * memory (the pages describe no such variant; it has no counterpart there).
 * Some callers own no allocator for the GPU: a host framework that manages
 * all device memory in its own arena and passes in only the model's tensors,
 * a plugin that is handed input and output pointers, or a latency-critical
 * loop where cudaMalloc (which can synchronise the device) is not allowed.
 * This entry point takes the same arguments as gdn_prefill minus the
 * workspace, and calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * The workspace lives instead in a fixed array of 64 KiB inside the library's
 * device image (every GPU that loads the library holds it until the process
 * exits).  That bounds n_seq * Hv to 16320 (for example 340 sequences of 48
 * value heads); larger problems are rejected with GDN_ERR_WORKSPACE before
 * anything touches the GPU.
 *
 * The array holds less than one producer / consumer ring, so this entry point
 * always runs the single-CTA prefill kernel: about 0.77 ms at T = 8192 (16 / 48
 * heads) against 0.30 ms for gdn_prefill with a full workspace.  With
 * GDN_PREFILL_KERNEL=pc set it returns GDN_ERR_UNSUPPORTED.
 *
 * The first call on each device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture.  The cache lasts as long as the process: after a cudaDeviceReset of
 * a device, do not call this entry point on that device again.  All calls in
 * the process share the one array, which keeps what the last call left there:
 * calls that overlap on the GPU (different streams, devices not involved) race
 * on it, so order them on one stream.  A bounded device wait that times out is
 * recorded in that shared array: gdn_prefill_status(NULL, stream) and
 * gdn_check_async(NULL, word, stream) read it.
 */
gdn_status gdn_prefill_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const float* a, const float* b, const float* A_log,
                               const float* dt_bias, const int32_t* cu_seqlens, int32_t n_seq,
                               int64_t T, int32_t Hqk, int32_t Hv, int32_t d, float scale,
                               const float* initial_state, float* final_state, float* o,
                               gdn_stream_t stream);

/*
 * gdn_decode_step -- one token of the recurrence for many independent units
 * (sequence s, layer l), unit u = s * layers + l, state updated in place.
 * This is the constant-memory, O(d^2)-per-token step the pages contrast with a
 * growing KV cache.
 *
 *  q, k           [U, Hqk, d] bf16, U = n_seq * layers.
 *  v              [U, Hv, d] bf16.
 *  a, b           [U, Hv] float32.
 *  A_log, dt_bias [layers, Hv] float32 (unit u uses row u % layers).
 *  state          [U, Hv, d_v, d_k] float32, read and overwritten in place.
 *  o              [U, Hv, d] float32 output (o from the updated state).
 * All arithmetic float32.  Supported: d = 128, Hv % Hqk == 0.
 */
gdn_status gdn_decode_step(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const float* a, const float* b, const float* A_log,
                           const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                           int32_t Hv, int32_t d, float scale, float* state, float* o,
                           gdn_stream_t stream);

/*
 * gdn_decode_step_fused -- one decode step with the layer's front end fused
 * in: for each (sequence, layer) unit the token's packed projection goes
 * through the causal width-4 convolution, SiLU and the q / k L2 norm
 * (gdn_conv1d_silu's arithmetic, architecture page section 2.1), then one step
 * of the recurrence (as gdn_decode_step, section 2.2).  q, k and v stay in
 * float32 between the two (no bf16 rounding).  The convolution history and the
 * state are updated in place.
 *
 *  qkv            [n_seq, layers, Ctot] bf16, Ctot = (2 Hqk + Hv) d, channels
 *                 ordered as in gdn_conv1d_silu.
 *  conv_w         [layers, Ctot, 4] float32 (tap 3 multiplies the current input).
 *  conv_state     [n_slots, layers, Ctot, 3] float32 in place: the three previous
 *                 inputs of each channel, oldest first.
 *  a, b           [n_seq, layers, Hv] float32;  A_log, dt_bias [layers, Hv] float32.
 *  slot           [n_seq] int32 (device): the slot holding sequence n's states,
 *                 or NULL for slot n (then n_slots >= n_seq).  Slots must be
 *                 distinct and < n_slots; the library trusts them.
 *  state          [n_slots, layers, Hv, d_v, d_k] float32 in place.
 *  o              [n_seq, layers, Hv, d] float32 output.
 * Slots not named by `slot` are not touched.  Supported: d = 128, Hv % Hqk == 0.
 */
gdn_status gdn_decode_step_fused(const uint16_t* qkv, const float* conv_w, float* conv_state,
                                 const float* a, const float* b, const float* A_log,
                                 const float* dt_bias, const int32_t* slot, int32_t n_seq,
                                 int32_t layers, int32_t Hqk, int32_t Hv, int32_t d, float scale,
                                 int32_t n_slots, float* state, float* o, gdn_stream_t stream);

/*
 * gdn_decode_step_bf16, gdn_decode_step_fused_bf16 -- gdn_decode_step and
 * gdn_decode_step_fused with the state stored as bf16 (uint16_t bit patterns)
 * instead of float32; every other argument as there.  The page's ~75 MB of
 * state for 48 layers (architecture page section 2.2) is this 2-byte size.
 * The arithmetic is float32; each updated state element is rounded to bf16
 * (nearest even) when stored.  This halves the bytes of the step, which is
 * bound by HBM bandwidth, at the price of one bf16 rounding of the state per
 * token.
 */
gdn_status gdn_decode_step_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                const float* a, const float* b, const float* A_log,
                                const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                                int32_t Hv, int32_t d, float scale, uint16_t* state, float* o,
                                gdn_stream_t stream);
gdn_status gdn_decode_step_fused_bf16(const uint16_t* qkv, const float* conv_w, float* conv_state,
                                      const float* a, const float* b, const float* A_log,
                                      const float* dt_bias, const int32_t* slot, int32_t n_seq,
                                      int32_t layers, int32_t Hqk, int32_t Hv, int32_t d, float scale,
                                      int32_t n_slots, uint16_t* state, float* o, gdn_stream_t stream);

/*
 * gdn_prefill_gated -- gdn_prefill followed by gdn_gated_norm on its output, in
 * one pass: y = norm_w * o / sqrt(mean_v o^2 + eps) * silu(z) per token and
 * value head (see gdn_gated_norm for the formula and the reading of the pages),
 * written as bf16 by the same kernel that computes o, so that o need not go
 * through memory.  Arguments as for gdn_prefill, plus
 *  z       [T, Hv, d] bf16, norm_w [d] float32, eps >= 0, y [T, Hv, d] bf16.
 *  o       may be NULL: the norm then runs inside the producer / consumer
 *          kernel and o is not written (no o buffer at all).  If o is given,
 *          the prefill writes o and gdn_gated_norm runs on it (two launches;
 *          measured faster on B200 at T = 8192: 0.38 ms against 0.46 ms for
 *          the fused kernel, whose exponentials on the consumer's SM lengthen
 *          the state chain).  GDN_PREFILL_NORM=fused in the environment forces
 *          the fused kernel with o written too.
 * The fused kernel needs a workspace that holds the producer / consumer
 * kernel's ring (see gdn_prefill_workspace_size); with a smaller one the
 * single-CTA kernel runs, o must be given (else GDN_ERR_WORKSPACE), and
 * gdn_gated_norm runs on it.
 */
gdn_status gdn_prefill_gated(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                             const float* b, const float* A_log, const float* dt_bias,
                             const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                             int32_t Hv, int32_t d, float scale, const float* initial_state,
                             float* final_state, float* o, const uint16_t* z, const float* norm_w,
                             float eps, uint16_t* y, void* workspace, size_t workspace_bytes,
                             gdn_stream_t stream);

/*
 * gdn_decode_step_gated -- gdn_decode_step (state_bf16 = 0, float32 state) or
 * gdn_decode_step_bf16 (state_bf16 = 1, bf16 state) with the gated output norm
 * of gdn_gated_norm applied to each (unit, value head)'s output in the same
 * kernel:  y = norm_w[l] * o / sqrt(mean_v o^2 + eps) * silu(z).
 *  state   [n_seq * layers, Hv, d, d] float32 or bf16 bits, updated in place.
 *  o       [n_seq * layers, Hv, d] float32, or NULL (not written).
 *  z       [n_seq * layers, Hv, d] bf16; norm_w [layers, d] float32 (unit u
 *          uses layer u % layers); eps >= 0; y [n_seq * layers, Hv, d] bf16.
 * Every other argument as for gdn_decode_step.
 */
gdn_status gdn_decode_step_gated(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 const float* a, const float* b, const float* A_log,
                                 const float* dt_bias, int32_t n_seq, int32_t layers, int32_t Hqk,
                                 int32_t Hv, int32_t d, float scale, void* state, int32_t state_bf16,
                                 float* o, const uint16_t* z, const float* norm_w, float eps,
                                 uint16_t* y, gdn_stream_t stream);

/*
 * gdn_prefill_backward_workspace_size -- bytes of device workspace
 * gdn_prefill_backward needs (a multiple of 256): a float32 state checkpoint per
 * 64-token chunk ((T / 64 + n_seq + 1) * Hv * d * d * 4), the 64 states of one
 * chunk per (sequence, value head) (n_seq * Hv * 64 * d * d * 4), dq and dk per
 * value head (2 * T * Hv * d * 4) and the gate-parameter sums.  Host-only.
 */
size_t gdn_prefill_backward_workspace_size(int32_t n_seq, int64_t T, int32_t Hv, int32_t d);

/*
 * gdn_prefill_backward -- the gradient of a scalar loss L through the
 * recurrence of gdn_prefill (reverse-mode, one token at a time):
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = scale S_t q_t,  alpha = exp(-exp(A_log) softplus(a + dt_bias)),
 *     beta = sigmoid(b)   (architecture page section 2.2, gate reading as for
 *     gdn_prefill).
 * Inputs as for gdn_prefill, plus
 *  d_o            [T, Hv, d] float32: dL/do.
 *  d_final_state  [n_seq, Hv, d_v, d_k] float32 or NULL (zero): dL/dS_T.
 * Outputs (float32, written in full; caller-owned):
 *  dq, dk         [T, Hqk, d] (summed over the value heads of each key head)
 *  dv             [T, Hv, d];  da, db [T, Hv];  dA_log, ddt_bias [Hv]
 *  d_initial_state [n_seq, Hv, d_v, d_k] or NULL (not written).
 * workspace: gdn_prefill_backward_workspace_size() bytes, 256-byte aligned.
 * The kernel runs on CUDA cores (one CTA per (sequence, value head), every
 * token in turn, float32 arithmetic); the result is deterministic.
 */
gdn_status gdn_prefill_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                                const float* b, const float* A_log, const float* dt_bias,
                                const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                                int32_t Hv, int32_t d, float scale, const float* initial_state,
                                const float* d_o, const float* d_final_state, float* dq, float* dk,
                                float* dv, float* da, float* db, float* dA_log, float* ddt_bias,
                                float* d_initial_state, void* workspace, size_t workspace_bytes,
                                gdn_stream_t stream);

/*
 * gdn_prefill_backward_chunked_workspace_size -- bytes of device workspace
 * gdn_prefill_backward_chunked needs (a multiple of 256).  A 256-byte header
 * whose first word is the error word (as in the prefill's workspace); with
 * slots = T / 64 + n_seq + 1: per (slot, value head) W and U' (2 * 64 * d
 * floats), T (64 * 64), Y, the chunk-start state and the chunk-end gradient
 * (3 * d * d) and 65 decay floats; dq and dk per value head (2 * T * Hv * d
 * floats); the chunk list and the gate-parameter sums.  About 256 KiB per
 * (chunk, value head).  Host-only.
 */
size_t gdn_prefill_backward_chunked_workspace_size(int32_t n_seq, int64_t T, int32_t Hv, int32_t d);

/*
 * gdn_prefill_backward_chunked -- the same gradient as gdn_prefill_backward,
 * taken through the chunked (WY / UT) form of the recurrence with 64-token
 * chunks (architecture page section 2.2 for the recurrence; the chunk algebra
 * is that of gdn_prefill).  The sequential work is two chains over chunks
 * instead of one over tokens: the chunk-start states, and the gradient at each
 * chunk end, dS_{c-1} = gam dS_c - (diag(kap) K dS_c^T)^T W + Y_c, whose
 * state-free term Y_c is computed for all chunks at once; everything else (dq,
 * dk, dv, the gates) is computed per (chunk, value head) in parallel.  The
 * per-chunk preparation, both chains and the per-chunk gradient step run their
 * products on the tensor cores (tcgen05, bf16 operands, float32 accumulation;
 * the chains carry the state in float32; the bf16 tensor-core prefill's
 * tolerance, 1e-2 relative to the largest reference element, applies), or all
 * in float32 on the CUDA cores when the environment variable
 * GDN_BACKWARD_GRAD=simt is set (2e-3).  No atomics: the result is
 * deterministic.
 * Arguments, layouts, outputs and errors as for gdn_prefill_backward, with the
 * workspace sized by gdn_prefill_backward_chunked_workspace_size().  The
 * tensor-core step waits (bounded, 2 s) for its products; if a wait gives up
 * it sets the workspace's error word, which gdn_prefill_status and
 * gdn_check_async read, and its outputs are not valid.  The call clears the
 * word first.
 */
gdn_status gdn_prefill_backward_chunked(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* a,
                                        const float* b, const float* A_log, const float* dt_bias,
                                        const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Hqk,
                                        int32_t Hv, int32_t d, float scale, const float* initial_state,
                                        const float* d_o, const float* d_final_state, float* dq, float* dk,
                                        float* dv, float* da, float* db, float* dA_log, float* ddt_bias,
                                        float* d_initial_state, void* workspace, size_t workspace_bytes,
                                        gdn_stream_t stream);

/*
 * gdn_gated_norm_backward_workspace_size -- bytes of device workspace
 * gdn_gated_norm_backward needs: per-tile partial sums of the weight gradient
 * (ceil(T / 8) * ceil(Hv / 8) * 8 * d floats) and per-chunk sums
 * (layers * ceil(ceil(T / layers) / 64) * d floats), each rounded up to 256
 * bytes; 0 for T = 0.  Host-only.
 */
size_t gdn_gated_norm_backward_workspace_size(int64_t T, int32_t Hv, int32_t d, int32_t layers);

/*
 * gdn_gated_norm_backward -- the gradient of gdn_gated_norm
 *     y = norm_w[l] * o * r * silu(z),  r = 1 / sqrt(mean_v o^2 + eps),  l = t % layers
 * given dL/dy (the same reading of the architecture page, section 2.1):
 *     d_o = r u - (r^3 / d) o <o, u>  with u = norm_w silu(z) dy,
 *     d_z = dy norm_w r o sigma(z) (1 + z (1 - sigma(z))),
 *     d_norm_w[l] = sum over the rows of layer l of dy r o silu(z).
 *  o, z, norm_w, T, Hv, d, layers, eps as for gdn_gated_norm;
 *  dy          [T, Hv, d] float32.
 * Outputs (float32, overwritten; caller-owned): d_o, d_z [T, Hv, d],
 * d_norm_w [layers, d].  workspace: gdn_gated_norm_backward_workspace_size()
 * bytes, 256-byte aligned (may be NULL when that is 0).  Supported: d = 128.
 * CUDA cores, float32, sums in a fixed order (deterministic).  Errors as for
 * gdn_gated_norm, plus GDN_ERR_WORKSPACE.
 */
gdn_status gdn_gated_norm_backward(const float* o, const uint16_t* z, const float* norm_w, const float* dy,
                                   int64_t T, int32_t Hv, int32_t d, int32_t layers, float eps, float* d_o,
                                   float* d_z, float* d_norm_w, void* workspace, size_t workspace_bytes,
                                   gdn_stream_t stream);

/*
 * gdn_selftest_bounded_wait -- failure detection check.  Runs, in one small
 * kernel, one of the bounded waits the prefill's CTAs use, on something that
 * never happens: which = 0 waits for a counter in global memory (as on the
 * producer / consumer ring) that no thread raises, which = 1 for an mbarrier
 * phase that never completes.  After limit_us microseconds (1 ms .. 2 s) the
 * wait gives up and the kernel records the error in the workspace's error word
 * as the prefill does, so that gdn_prefill_status(workspace) then returns
 * GDN_ERR_TIMEOUT.  Nothing faults or hangs; the context stays usable.
 * workspace: at least 256 bytes, 256-byte aligned (its header is cleared), or
 * NULL for the library-owned array of gdn_prefill_noalloc.
 */
gdn_status gdn_selftest_bounded_wait(int32_t which, int64_t limit_us, void* workspace, gdn_stream_t stream);

/*
 * gdn_gated_norm -- the gated output norm that follows the recurrence in a
 * linear-attention layer:
 *     y[t, h, :] = norm_w[l] * o[t, h, :] / sqrt(mean_v o[t, h, v]^2 + eps)
 *                  * silu(z[t, h, :]),      silu(x) = x / (1 + e^{-x}).
 * The architecture page (section 2.1) lists `norm` and `in_proj_z` among each
 * linear-attention layer's weights but prints no formula; this is the reading
 * used: an RMS norm over the d_v channels of each value head, one weight
 * vector per layer shared by all heads, gated by SiLU of z = in_proj_z(x).
 *
 *  o       [T, Hv, d] float32 (the output of gdn_prefill or of a decode step).
 *  z       [T, Hv, d] bf16.
 *  norm_w  [layers, d] float32; row t uses layer t % layers (1 for a prefill;
 *          for a decode batch, rows are units s * layers + l).
 *  eps     >= 0 (the layer uses 1e-6).
 *  y       [T, Hv, d] bf16 output (round to nearest even); must not overlap o
 *          or z.
 * Supported: d = 128.  T = 0 does nothing.  All pointers 16-byte aligned.
 * One launch, bound by HBM bandwidth (1024 bytes per (token, head)).
 */
gdn_status gdn_gated_norm(const float* o, const uint16_t* z, const float* norm_w, int64_t T, int32_t Hv,
                          int32_t d, int32_t layers, float eps, uint16_t* y, gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
