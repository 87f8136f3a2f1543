/*
 * gdn_cpr.h -- C ABI of the CPR Gated DeltaNet library for B200 (sm_100a).
 *
 * The layer is the gated delta rule with an fp32 state, per sequence and head
 * (IsoExec summary page, section "Chunkwise-Parallel Recurrent (CPR) Gated
 * DeltaNet"; commentary blog, section 10 "Gated DeltaNet"):
 *
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t
 *
 * It is evaluated chunkwise-parallel recurrent (CPR).  The recurrence is the
 * primary computation.  It runs in parallel across chunks of C tokens, each chunk
 * starting from its boundary state.  Decode re-synchronises its running state
 * with the boundary state every C tokens (same page and section; daily.dev
 * digest, "What is chunkwise-parallel recurrent (CPR)").
 *
 * Every entry point executes one written-down fp32 arithmetic schedule.  The
 * schedule fixes an 8-leaf reduction tree over d_k, the operation order and the
 * rounding (IsoExec summary page, "Achieving Parallelism Invariance";
 * commentary blog, section 8).  The forward and the decode step therefore give
 * bit-identical outputs and states.  gdn_contract_id() names the schedule.
 *
 * Conventions common to every call:
 *  - All tensors are caller-owned device memory unless marked "host".
 *    The library never allocates device memory and never synchronises the
 *    device.  It keeps global mutable state in two places only:
 *    gdn_cpr_forward_noalloc (end of this file) uses a fixed device array
 *    inside the library and caches that array's address per device, and
 *    gdn_test_fault_injection holds a process-wide test setting.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *    The call returns once the kernels are enqueued.
 *  - Layouts are row-major and densely packed:
 *      q, k   [T_total, H, d_k]      v, o [T_total, H, d_v]
 *      alpha, beta [T_total, H] fp32  (alpha in [0, 1], beta in [0, 1])
 *      states [.., H, d_v, d_k] fp32  (row i of a state = value channel i)
 *  - Every device pointer must be 16-byte aligned.
 *  - Supported shapes: d_k == d_v in {16, 32, 64, 128}; C in {16, 32, 64}.
 *    Any other shape returns GDN_ERR_UNSUPPORTED.
 *  - Inputs must be finite.  The results for NaN or Inf inputs are unspecified.
 *  - Errors are reported through status codes only: no exceptions, no exit,
 *    and no device trap or assert.  There are two places:
 *      1. The return code.  Invalid arguments and failed launches are caught on
 *         the host before or while the kernels are enqueued.
 *      2. The device status word.  Two errors can only be seen on the GPU
 *         while the kernels run: a device cu_seqlens that disagrees with the
 *         host copy (GDN_ERR_DEVICE_INPUT), and a bounded wait that ran out
 *         (GDN_ERR_TIMEOUT).  The kernels record the first such error in a
 *         status word.  For gdn_cpr_forward and gdn_cpr_backward that word
 *         sits in the workspace; gdn_read_device_status copies it out.  For
 *         gdn_decode_step it is gdn_cache_t.status.  A call whose return code
 *         is GDN_OK can still have failed on the device: read the status word
 *         after the stream has run the call.
 */
#ifndef GDN_CPR_H
#define GDN_CPR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* NULL/misaligned pointer, bad size, bad cu_seqlens */
    GDN_ERR_UNSUPPORTED = 2,   /* (d_k, d_v, C, dtype) not compiled in */
    GDN_ERR_CUDA = 3,          /* a CUDA launch or attribute call failed */
    GDN_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than gdn_cpr_workspace_size() */
    GDN_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out; the outputs are incomplete */
    GDN_ERR_DEVICE_INPUT = 6   /* device: cu_seqlens on the device disagrees with the host copy, or a
                                  decode position outside [0, C); nothing was written for it */
} gdn_status_t;

typedef enum {
    GDN_F32 = 0,               /* IEEE binary32 */
    GDN_BF16 = 1               /* bfloat16; widened exactly to fp32 on load, stored round-to-nearest-even */
} gdn_dtype_t;

/*
 * Decode cache of N sequences.  It is the complete resumable state of a CPR
 * layer at any token position.  All fields are caller-owned device memory.
 *   S_b  [N, H, d_v, d_k] fp32   the last chunk-boundary state (position floor(p/C)*C)
 *   R    [N, H, d_v, d_k] fp32   the running per-token state divided by rscale
 *   rscale [N, H] fp32           the running state's scale: the running state is
 *                                rscale * R.  The per-token step keeps the decay
 *                                in this scale and folds it into R when it would
 *                                fall below 2^-64 (R == S_b and rscale == 1 when
 *                                pos == 0)
 *   kbuf [N, H, C, d_k]  in_dtype  the tokens since the last boundary ...
 *   vbuf [N, H, C, d_v]  in_dtype
 *   abuf [N, H, C] fp32, bbuf [N, H, C] fp32   ... their gates
 *   pos  [N, H] int32            tokens since the last boundary, 0 <= pos < C
 *   status  one int32, or NULL   the decode step's device status word: the
 *                                kernels store the first error they detect
 *                                (GDN_ERR_DEVICE_INPUT for a pos outside [0, C),
 *                                GDN_ERR_TIMEOUT for a resync whose tensor-core
 *                                wait ran out; that pair's pos becomes -1).
 *                                The library never clears it: the caller sets
 *                                it to GDN_OK (0) and reads it back.  NULL: not
 *                                recorded.  gdn_cpr_forward ignores it.
 * A fresh cache for an initial state S_0 is S_b = R = S_0 with rscale = 1 and
 * pos = 0.  The buffer contents do not matter while pos == 0.
 */
typedef struct {
    float*   S_b;
    float*   R;
    float*   rscale;
    void*    kbuf;
    void*    vbuf;
    float*   abuf;
    float*   bbuf;
    int32_t* pos;
    int32_t* status;
} gdn_cache_t;

/* Name of the arithmetic schedule every kernel executes (static string). */
const char* gdn_contract_id(void);

/*
 * Contract identities.  Runtimes that must give the same bits compare SHA-256
 * identities of the contract they execute, in three parts (IsoExec summary
 * page, "Contract Structure and Enforcement", Identities; commentary blog,
 * section 6):
 *   GDN_ID_SEMANTIC          what the layer computes: the recurrence, the CPR
 *                            composition, layouts, shapes and dtypes;
 *   GDN_ID_NUMERICAL_POLICY  how: the fp32 rules, the reduction tree, the
 *                            operation order, the split products and the
 *                            instruction shapes of every step (it names
 *                            gdn_contract_id());
 *   GDN_ID_DEPLOYMENT        which build: target, a SHA-256 of the kernel
 *                            sources, the compiler version.
 * Two runtimes with equal semantic and numerical-policy identities for the
 * same (d_k, d_v, C, dtypes) produce bit-identical results.
 */
typedef enum {
    GDN_ID_SEMANTIC = 0,
    GDN_ID_NUMERICAL_POLICY = 1,
    GDN_ID_DEPLOYMENT = 2
} gdn_identity_kind_t;

/*
 * The canonical text an identity digests.  Writes at most cap bytes
 * (NUL-terminated, truncated if cap is too small) and returns the full length
 * without the NUL, or -1 for an unsupported shape, a bad kind, or buf == NULL
 * with cap != 0.  gdn_contract_text(kind, ..., NULL, 0) returns the length.
 */
int64_t gdn_contract_text(gdn_identity_kind_t kind, int32_t d_k, int32_t d_v, int32_t C,
                          gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, char* buf, size_t cap);

/*
 * SHA-256 of gdn_contract_text as 64 lowercase hex digits plus NUL into
 * out_hex (65 bytes, host memory).  GDN_ERR_UNSUPPORTED for a shape or dtype
 * that is not compiled in; GDN_ERR_INVALID_ARG for out_hex == NULL or a bad kind.
 */
gdn_status_t gdn_contract_identity(gdn_identity_kind_t kind, int32_t d_k, int32_t d_v, int32_t C,
                                   gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, char* out_hex);

/* SHA-256 (FIPS 180-4) of n bytes of host memory as 64 hex digits plus NUL. */
gdn_status_t gdn_sha256_hex(const void* data, size_t n, char* out_hex);

/* Human-readable text for a status code (static string). */
const char* gdn_status_string(gdn_status_t status);

/*
 * Device status of the last gdn_cpr_forward or gdn_cpr_backward call that used
 * `workspace` (NULL: the fixed array of gdn_cpr_forward_noalloc on the current
 * device).  The call enqueues on `stream` one 4-byte copy of the workspace's
 * status word into *status_out, which may be host or device memory.  Once the
 * stream has run it (cudaStreamSynchronize), *status_out holds a gdn_status_t:
 *   GDN_OK               the kernels detected nothing;
 *   GDN_ERR_DEVICE_INPUT the device cu_seqlens disagreed with the host copy;
 *                        the kernels wrote no output;
 *   GDN_ERR_TIMEOUT      a bounded device wait ran out (about a second of GPU
 *                        clocks); some outputs were not written.
 * Every forward and backward call resets the word at its start, on the
 * stream, so the copy must be enqueued after the call it reports on and
 * before the next call that uses the same workspace.  Returns
 * GDN_ERR_INVALID_ARG for status_out == NULL and GDN_ERR_CUDA if the copy
 * cannot be enqueued.  Host-side errors are not recorded here: they are the
 * return codes of the calls themselves.
 */
gdn_status_t gdn_read_device_status(const void* workspace, int32_t* status_out, void* stream);

/*
 * Failure-detection hook, for tests of the status reporting.  It is
 * process-wide and off by default.
 *   mode 0: normal operation (wait_clocks is ignored);
 *   mode 1: every later gdn_cpr_forward call that runs the fused chain +
 *           intra-chunk kernel (d_v = 128 and fewer (sequence, head) pairs
 *           than SMs) withholds the publication of its boundary states.  Each
 *           intra-chunk task then waits for a state that never arrives.  The
 *           wait gives up after wait_clocks GPU clocks (1 .. 2^31), the task
 *           records GDN_ERR_TIMEOUT and ends, and the call's outputs are
 *           incomplete.  Nothing on the GPU faults or hangs.
 * Returns GDN_ERR_INVALID_ARG for another mode or a wait_clocks out of range.
 */
gdn_status_t gdn_test_fault_injection(int32_t mode, int64_t wait_clocks);

/*
 * Number of chunk states the forward writes.  That is
 * sum_n (floor(L_n / C) + 1), with L_n = cu_seqlens_host[n+1] - cu_seqlens_host[n].
 * cu_seqlens_host is host memory with num_seqs + 1 entries.  Returns -1 if
 * the arguments are invalid (see gdn_cpr_forward).
 */
int64_t gdn_num_chunk_states(const int32_t* cu_seqlens_host, int32_t num_seqs, int32_t C);

/*
 * Device workspace, in bytes, that gdn_cpr_forward needs for a batch of at most
 * total_tokens tokens in num_seqs sequences.  Returns 0 for invalid sizes.
 */
size_t gdn_cpr_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H,
                              int32_t d_k, int32_t d_v, int32_t C);

/*
 * CPR forward: rollout prefill and trainer forward are the same call.
 *
 * Inputs:
 *   q, k [T_total,H,d_k], v [T_total,H,d_v] in in_dtype;  alpha, beta [T_total,H] fp32.
 *   state_in [num_seqs,H,d_v,d_k] fp32 is the state at each sequence's
 *     position 0, which is a chunk boundary.  NULL means zeros.
 *   cu_seqlens      device [num_seqs+1] int32, packed sequence offsets
 *   cu_seqlens_host host   [num_seqs+1] int32, the same values.  It sizes the
 *     launch grids and is validated on the host: cu[0] == 0, non-decreasing,
 *     cu[num_seqs] == total_tokens.  The kernels check the device copy against
 *     the host copy: chunk totals and a 64-bit position-sensitive hash of
 *     the values.  If the two copies disagree, the kernels write nothing, the
 *     outputs keep their previous contents, and the workspace's device status
 *     word becomes GDN_ERR_DEVICE_INPUT (gdn_read_device_status).
 *   Chunks are aligned to each sequence's own token 0, so results do not
 *   depend on batch composition or packing.
 * Outputs:
 *   o [T_total,H,d_v] in out_dtype (fp32, or bf16 with nearest-even rounding)
 *   chunk_states [gdn_num_chunk_states(),H,d_v,d_k] fp32: for sequence n,
 *     entries s_n + c (c = 0..floor(L_n/C)) hold the state at position c*C,
 *     where s_n = sum_{m<n}(floor(L_m/C)+1).  Entry s_n is a copy of state_in.
 *   cache_out (optional; NULL to skip): filled for a decode continuation of
 *     every sequence, in the layout of gdn_cache_t with N = num_seqs.  Its
 *     buffers take in_dtype.
 *   workspace: at least gdn_cpr_workspace_size(total_tokens, num_seqs, H, d_k,
 *     d_v, C) bytes of device memory, owned by the caller.  The call may
 *     overwrite it freely.  It must not be shared with a concurrent call.
 */
gdn_status_t gdn_cpr_forward(const void* q, const void* k, const void* v,
                             const float* alpha, const float* beta,
                             const float* state_in,
                             const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                             int32_t num_seqs, int64_t total_tokens, int32_t H,
                             int32_t d_k, int32_t d_v, int32_t C,
                             gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                             void* o, float* chunk_states, const gdn_cache_t* cache_out,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Device workspace, in bytes, that gdn_cpr_backward needs for a batch of
 * total_tokens tokens in num_seqs sequences.  It holds the tables, the
 * recomputation checkpoints (one state row tile per 8 tokens of a chunk for
 * every (sequence, head, row tile)) and the per-row-tile partial sums of
 * dq, dk, dalpha and dbeta.  Returns 0 for invalid sizes.
 */
size_t gdn_cpr_backward_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H,
                                       int32_t d_k, int32_t d_v, int32_t C);

/*
 * CPR backward (trainer): the gradients of L = sum_t dO_t . o_t for the layer
 * of gdn_cpr_forward, with the gated delta rule
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t
 * (IsoExec summary page, section "Chunkwise-Parallel Recurrent (CPR) Gated
 * DeltaNet"; commentary blog, section 10), differentiated in reverse token
 * order.  A serial scan carries dL/dS back to every chunk boundary; then the
 * chunks run in parallel, each from the boundary state the forward stored and
 * the adjoint at its end, as dense products of chunk matrices on the tensor
 * cores (tf32 with a hi/lo split of every fp32 operand).
 * Inputs:
 *   q, k, v, alpha, beta, cu_seqlens, cu_seqlens_host, num_seqs, total_tokens,
 *     H, d_k, d_v, C, in_dtype: as given to gdn_cpr_forward.
 *   dO [T_total,H,d_v] in in_dtype: the gradient of the loss for o.
 *   chunk_states: the forward's chunk_states output for these inputs.
 *   dstate_out [num_seqs,H,d_v,d_k] fp32, or NULL for zeros: the gradient of
 *     the loss for each sequence's final state (the state after its last
 *     token).  A sequence split at a chunk boundary runs its later part's
 *     backward first and passes that call's dstate_in here to the earlier
 *     part: the result equals the unsplit backward bit for bit.
 * Outputs (fp32, device, caller-owned, every element written):
 *   dq, dk [T_total,H,d_k]; dv [T_total,H,d_v]; dalpha, dbeta [T_total,H];
 *   dstate_in [num_seqs,H,d_v,d_k]: the gradient for the forward's state_in.
 * The result is deterministic: every sum has a fixed order and there are no
 * atomics, so repeats give the same bits.
 *   workspace: at least gdn_cpr_backward_workspace_size(...) bytes of device
 *     memory, 256-byte aligned, not shared with a concurrent call.
 * Errors: as gdn_cpr_forward.  If the device copy of cu_seqlens disagrees
 * with the host copy, the kernels write nothing and the workspace's device
 * status word becomes GDN_ERR_DEVICE_INPUT (gdn_read_device_status).
 */
gdn_status_t gdn_cpr_backward(const void* q, const void* k, const void* v,
                              const float* alpha, const float* beta, const void* dO,
                              const float* chunk_states, const float* dstate_out,
                              const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                              int32_t num_seqs, int64_t total_tokens, int32_t H,
                              int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype,
                              float* dq, float* dk, float* dv, float* dalpha, float* dbeta,
                              float* dstate_in, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * gdn_cpr_backward with events: events (host array of 4 cudaEvent_t, or NULL)
 * are recorded on the stream before the boundary-adjoint scan, after it,
 * after the chunk-local precompute and after the per-chunk gradients.
 */
gdn_status_t gdn_cpr_backward_timed(const void* q, const void* k, const void* v,
                                    const float* alpha, const float* beta, const void* dO,
                                    const float* chunk_states, const float* dstate_out,
                                    const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                    int32_t num_seqs, int64_t total_tokens, int32_t H,
                                    int32_t d_k, int32_t d_v, int32_t C, gdn_dtype_t in_dtype,
                                    float* dq, float* dk, float* dv, float* dalpha, float* dbeta,
                                    float* dstate_in, void* workspace, size_t workspace_bytes,
                                    void* stream, void* const* events);

/*
 * One decode step: one new token for each of num_seqs sequences.
 *   q, k [num_seqs,H,d_k], v [num_seqs,H,d_v] in in_dtype; alpha, beta [num_seqs,H] fp32
 *   cache: updated in place (see gdn_cache_t).  For each (sequence, head):
 *     the running state R takes one per-token step and gives o.  The token is
 *     appended to the buffer.  When the buffer then holds C tokens, the
 *     boundary state is advanced over them (S_b <- P_chunk(S_b, buffer)),
 *     R <- S_b, and pos wraps to 0 (the resync).
 *   o [num_seqs,H,d_v] out_dtype.
 * The call enqueues two kernels: the per-token step, then the resync.  The
 * resync exits at once for sequences that are not at a boundary.  A prefill
 * of L tokens followed by m decode steps gives bit-identical o and cache to a
 * prefill of L + m tokens.
 * A pos outside [0, C) is not written through.  That (sequence, head) is left
 * unchanged, its o is unspecified, and cache->status (when non-NULL) records
 * GDN_ERR_DEVICE_INPUT.  A resync whose tensor-core completion wait runs out
 * (about a second of GPU clocks) records GDN_ERR_TIMEOUT and sets the pos of
 * the pairs it had not finished to -1.
 */
gdn_status_t gdn_decode_step(const void* q, const void* k, const void* v,
                             const float* alpha, const float* beta,
                             const gdn_cache_t* cache,
                             int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v, int32_t C,
                             gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                             void* o, void* stream);

/*
 * gdn_decode_step with a host-side hint and optional events.
 *   may_resync = 0: the caller guarantees that no (sequence, head) buffer
 *     fills in this step, i.e. every pos is below C - 1 before the call (the
 *     positions follow from the prefill lengths: pos = L mod C after a prefill
 *     of L tokens, then + 1 per step, wrapping to 0 at C).  Only the per-token
 *     kernel is enqueued; the resync launch is skipped.
 *   may_resync != 0: exactly gdn_decode_step.
 *   events: NULL, or 3 events as for gdn_decode_step_timed (with the resync
 *     skipped, events[1] and events[2] are recorded back to back).
 * A wrong guarantee does not write out of bounds: a pair whose buffer filled
 * is left at pos = C, and the next step's per-token kernel treats that as an
 * invalid position (GDN_ERR_DEVICE_INPUT in cache->status, nothing written
 * for it) until a call with may_resync != 0 runs its resync.
 */
gdn_status_t gdn_decode_step_ex(const void* q, const void* k, const void* v,
                                const float* alpha, const float* beta,
                                const gdn_cache_t* cache,
                                int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v, int32_t C,
                                gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                                void* o, int32_t may_resync, void* stream, void* const* events);

/*
 * Per-kernel timing variants, for benchmarks and profilers.  These are the
 * same calls with the same launches and the same results.  In addition they
 * record caller-created CUDA events (cudaEvent_t, created on the current
 * device) on `stream` between the kernels:
 *   gdn_cpr_forward_timed: events[0..5] around, in order, the offsets
 *     kernel, the chunk precompute (w, u0, decays), the boundary-state chain,
 *     the intra-chunk recurrence and the cache fill.  Kernel i ran between
 *     events[i] and events[i+1].  A kernel that has no work still gets both
 *     of its events, so its time is zero.  When the chain and the
 *     intra-chunk recurrence run as one kernel (batches with d_v = 128 and
 *     fewer (sequence, head) pairs than SMs), events[2] and events[3] are
 *     recorded back to back and events[3..4] span that kernel.
 *   gdn_decode_step_timed: events[0..2] around the per-token step and then the
 *     resync.
 * events == NULL behaves exactly like the untimed call.
 */
gdn_status_t gdn_cpr_forward_timed(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta,
                                   const float* state_in,
                                   const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                   int32_t num_seqs, int64_t total_tokens, int32_t H,
                                   int32_t d_k, int32_t d_v, int32_t C,
                                   gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                                   void* o, float* chunk_states, const gdn_cache_t* cache_out,
                                   void* workspace, size_t workspace_bytes, void* stream,
                                   void* const* events);

gdn_status_t gdn_decode_step_timed(const void* q, const void* k, const void* v,
                                   const float* alpha, const float* beta,
                                   const gdn_cache_t* cache,
                                   int32_t num_seqs, int32_t H, int32_t d_k, int32_t d_v, int32_t C,
                                   gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                                   void* o, void* stream, void* const* events);

/*
 * Forward without any device allocation, for callers that cannot allocate
 * device memory at the point of the call.  Examples: a plugin whose host
 * framework owns all device memory and forbids allocation inside its execute
 * callback; a process that has already reserved the whole device for its own
 * memory pool; a latency-critical loop that cannot take the implicit device
 * synchronisation of cudaMalloc.  The pages have no counterpart to this call;
 * it exists for such integrations only.
 *
 * It is gdn_cpr_forward, with the same arguments, results and errors, except
 * that its workspace is a fixed array of GDN_NOALLOC_SCRATCH_BYTES inside the
 * library.  The caller still passes every input and output.
 *  - Limit: the batch must fit the fixed array, i.e.
 *    gdn_cpr_workspace_size(total_tokens, num_seqs, H, d_k, d_v, C) <=
 *    GDN_NOALLOC_SCRATCH_BYTES.  At d_k = d_v = 128 and C = 64 that is about
 *    65,000 (token, head) pairs, for example 4,000 tokens with 16 heads.  Larger
 *    batches return GDN_ERR_WORKSPACE before anything is enqueued.
 *  - Every device that uses the library holds the array until the process
 *    exits.  CUDA loads modules lazily by default, so the array is committed on
 *    a device at the first call there (unless CUDA_MODULE_LOADING=EAGER): a
 *    caller that reserves the whole device for its own pool makes one call
 *    first.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it per device
 *    ordinal for the life of the process.  Make that first call before any
 *    stream capture begins.  The cache does not survive cudaDeviceReset (the
 *    module is reloaded at another address): do not use this entry point after
 *    a device reset in the same process.
 *  - All calls on a device share the one array, and it keeps the last call's
 *    contents; no part of it needs to start at zero.  Calls whose work
 *    overlaps on the GPU (different streams, or different host threads)
 *    race on the array and give wrong results; serialise them.
 *  - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (64u << 20)

gdn_status_t gdn_cpr_forward_noalloc(const void* q, const void* k, const void* v,
                                     const float* alpha, const float* beta,
                                     const float* state_in,
                                     const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                     int32_t num_seqs, int64_t total_tokens, int32_t H,
                                     int32_t d_k, int32_t d_v, int32_t C,
                                     gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                                     void* o, float* chunk_states, const gdn_cache_t* cache_out,
                                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_CPR_H */
