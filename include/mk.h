/*
 * mk.h - C ABI of the persistent decode megakernel for NVIDIA B200 (sm_100a).
 *
 * One call evaluates one whole decoder step (embedding -> every layer's
 * attention and FFN / MoE -> final norm -> LM head -> greedy argmax) as a
 * single persistent kernel.  Source of the operation: "700 TPS on Kimi K3:
 * A Case for TPU Megakernels" (Inferact blog), section "Why megakernels?"
 * (the whole decoder step inside one program, weight loads decoupled from
 * their consumers), section "Our Kimi K3 megakernel" (phase order attention
 * -> router -> shared expert -> routed experts; the next layer's attention
 * weights are fetched while the current layer's MoE runs) and section
 * "DSpark" (one launch checks 1 anchor + 7 proposals).
 *
 * Conventions for every entry point:
 *   - Return MK_OK or an error code; no exception crosses the ABI.
 *   - Argument errors are detected on the host and returned synchronously;
 *     nothing is launched then.
 *   - Compute calls are asynchronous on the caller's stream.  Errors found
 *     on the device (a bounds violation in device-resident inputs, a
 *     dependency wait that timed out) are recorded in a device status word
 *     and read with mk_sync_status() after the stream has been synchronised.
 *     They are sticky: later compute calls return MK_ERR_STATE until
 *     mk_reset() is called.
 *   - Pointers marked "dev" are CUDA device pointers owned by the caller;
 *     "host" pointers are host memory owned by the caller.  The library never
 *     frees caller memory and never keeps a caller pointer after a call
 *     returns.  Weights, KV caches and scratch are owned by the library.
 *   - mk_last_error() returns a static description of the last failure of a
 *     handle (valid until the next call on that handle).
 */
#ifndef MK_H
#define MK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MK_OK = 0,
  MK_ERR_INVALID = 1,        /* bad argument or unsupported shape */
  MK_ERR_OOM = 2,            /* device allocation failed */
  MK_ERR_CUDA = 3,           /* a CUDA runtime call failed */
  MK_ERR_DEVICE_TIMEOUT = 4, /* a dependency wait inside the kernel ran out */
  MK_ERR_DEVICE_BOUNDS = 5,  /* token / position out of range in device inputs */
  MK_ERR_STATE = 6           /* handle is in the sticky error state, or wrong order of calls */
} mk_status;

/* Shape of the decoder.  A dense model has n_routed == 0 (then ffn > 0).
 * A MoE model has n_routed > 0, top_k in [1, 8], expert_ffn > 0, n_shared >= 0.
 * kv_lora_rank > 0 selects multi-head latent attention: query heads have
 * head_dim "nope" dims + rope_dim rotary dims, values have head_dim dims, and
 * the cache keeps kv_lora_rank + rope_dim values per position (n_kv_heads is
 * ignored).  expert_fp8 != 0 stores shared and routed expert weights as OCP
 * FP8 E4M3 with one fp32 scale per 128x128 block of each [out, in] matrix.
 * max_batch (<= 8) bounds S * Q rows of one step; max_ctx bounds positions. */
typedef struct {
  int32_t layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  float rope_theta, rms_eps;
  int32_t n_routed, n_shared, top_k, expert_ffn;
  int32_t kv_lora_rank, rope_dim;
  int32_t expert_fp8;
  int32_t max_batch, max_ctx;
} mk_model_desc;

/* Parameters of the seeded synthetic weights (see synth/synth.h for the
 * counter-based generator): weights ~ N(0, w_sigma^2) rounded to bf16, router
 * ~ N(0, router_sigma^2), norm gains 1 + N(0, gain_sigma^2), fp8 expert codes
 * e4m3(16 N(0,1)) with block scales fp8_block_base * (1 + j/8). */
typedef struct {
  uint64_t seed;
  float w_sigma, router_sigma, gain_sigma, fp8_block_base;
} mk_synth_params;

typedef struct mk_handle mk_handle;
typedef struct mk_kv mk_kv;

/* Create a model on `device` (weights allocated, not initialised).
 * Fails with MK_ERR_INVALID for unsupported shapes (e.g. head_dim other than
 * 64 or 128, hidden not a multiple of 16, n_q_heads not a multiple of
 * n_kv_heads) and MK_ERR_OOM when the weights do not fit. */
mk_status mk_create(const mk_model_desc* desc, int device, mk_handle** out);

/* Fill every weight from the seeded generator, directly on the device and
 * already in the kernel's streaming layout.  Synchronous. */
mk_status mk_init_random(mk_handle* h, const mk_synth_params* p);

/* Weight tensor for mk_load_weights, in logical row-major [rows][cols]
 * layout ([out, in] for projections).  `kind` and `layer`/`expert` name the
 * tensor with the same ids as synth/synth.h (SYN_WQKV, SYN_EX_GATE, ...).
 * data: bf16 bits (uint16) for bf16 tensors, e4m3 bytes for fp8 expert
 * tensors (then `scales` = fp32 [ceil(rows/128)][ceil(cols/128)]).
 * on_device != 0 means data/scales are device pointers, else host. */
typedef struct {
  int32_t kind, layer, expert;
  int64_t rows, cols;
  const void* data;
  const float* scales;
  int32_t on_device;
} mk_tensor_src;

/* Copy and re-tile `n` tensors into the model's weights.  The caller keeps
 * ownership of the sources.  Shapes must match the descriptor exactly.
 * Synchronous. */
mk_status mk_load_weights(mk_handle* h, const mk_tensor_src* tensors, int n);

/* A KV cache for up to `max_seqs` sequences of `max_ctx` positions, owned by
 * the library, zero-filled.  Layout (device, bf16): GQA keys and values
 * [layers][max_seqs][n_kv_heads][max_ctx][head_dim] each, with the 16-byte
 * groups of each row permuted by the position (group c at c ^ (pos & 7), so
 * that the kernel's shared-memory reads are free of bank conflicts); MLA
 * latent [layers][max_seqs][max_ctx][kv_lora_rank + rope_dim]. */
mk_status mk_kv_create(mk_handle* h, int max_seqs, int max_ctx, mk_kv** out);

/* Fill positions [0, length) of every sequence with seeded bf16 values
 * ~ N(0, sigma^2) (a synthetic pre-filled context).  Synchronous. */
mk_status mk_kv_fill_random(mk_kv* kv, uint64_t seed, float sigma, int32_t length);

/* Copy the whole cache into caller device memory of mk_kv_bytes() bytes, in
 * logical order (rows not permuted; keys first, then values, for GQA).
 * Synchronous. */
mk_status mk_kv_copy_out(mk_kv* kv, void* dst_dev);
int64_t mk_kv_bytes(const mk_kv* kv);

/* The inverse of mk_kv_copy_out: replace the whole cache with caller device
 * memory of mk_kv_bytes() bytes in logical order (the copy-out layout), for
 * example a context computed elsewhere.  The source is only read; the
 * caller keeps it.  Synchronous. */
mk_status mk_kv_copy_in(mk_kv* kv, const void* src_dev);

/* One decode step for B sequences (B <= max_batch): sequence b consumes
 * tokens[b] at positions[b], writes its K/V there and attends over
 * positions 0..positions[b].
 *   tokens, positions: dev int32 [B]
 *   logits_out: dev fp32 [B][vocab], or NULL
 *   argmax_out: dev int32 [B] (greedy token; ties -> lower index)
 *   stream: a cudaStream_t (NULL = default stream)
 * Device-side bounds errors: token outside [0, vocab) or position outside
 * [0, kv max_ctx). */
mk_status mk_decode_step(mk_handle* h, const int32_t* tokens, const int32_t* positions, int B,
                         mk_kv* kv, float* logits_out, int32_t* argmax_out, void* stream);

/* The same decode step as mk_decode_step, run the way the pages describe a
 * GPU serving stack doing it ("Why megakernels?": one kernel per operation,
 * launch overhead hidden with CUDA Graphs and programmatic dependent launch),
 * for comparison with the persistent kernel.  The step's tasks are split at
 * every phase boundary of the single kernel (each projection's row split,
 * each layer's attention items, ...) into one launch of the same kernel code
 * per phase; a phase waits for the previous one through the launch order,
 * and its weight stream starts before that wait (programmatic dependent
 * launch lets it begin while the previous phase drains).  The launches are
 * recorded once per (batch size, cache, logits wanted, router trace) as a
 * CUDA graph; each call copies tokens and positions into fixed device
 * buffers, launches the graph and copies the argmax (and logits) out.  The
 * arithmetic is the persistent kernel's, task for task: results are
 * bit-identical to mk_decode_step.  Allocates on its first call (fixed
 * buffers) and on the first call of each key (the graph).  Arguments as for
 * mk_decode_step; the task trace and the stall hook are not supported
 * (MK_ERR_STATE). */
mk_status mk_decode_step_multikernel(mk_handle* h, const int32_t* tokens, const int32_t* positions, int B,
                                     mk_kv* kv, float* logits_out, int32_t* argmax_out, void* stream);

/* Size of the static device array behind mk_decode_step_noalloc, in bytes.
 * Every GPU that loads this library holds it until the process exits. */
#define MK_NOALLOC_SCRATCH_BYTES (16u << 20)

/* mk_decode_step that allocates no device memory.  The pages this library
 * follows have no counterpart; it is here for callers that cannot call
 * cudaMalloc while they step the model: a process whose device memory is all
 * owned by its own allocator (a framework's caching allocator, a serving
 * engine that sizes its KV pool to fill the GPU), or a latency-critical loop
 * that must not let cudaMalloc / cudaFree synchronise the device.
 * (mk_decode_step allocates the device task list of a batch size the first
 * time that size is used.)
 *   Arguments, results and device-error reporting are those of
 *   mk_decode_step (errors through mk_sync_status on the same handle).
 *   The task list, activations, partial sums, split-KV partials and
 *   inter-CTA counters live in one file-scope device array of
 *   MK_NOALLOC_SCRATCH_BYTES, shared by every handle on the device and
 *   keeping the last call's contents.  The counters must start at zero: each
 *   call clears them on `stream` before its launch; nothing else needs it.
 *   The task list is rebuilt on the host and copied in (from pageable host
 *   memory, on `stream`) only when another handle or batch size used the
 *   array last.
 *   The first call on a device looks up the array's device address (a
 *   one-time set-up); make that first call before any stream capture.  A
 *   call that has to install a task list (its handle or batch size differs
 *   from the last call's on this device) while `stream` is capturing returns
 *   MK_ERR_STATE: the list is copied from host memory that the call frees.
 *   Work enqueued by a call reads, when it runs on the GPU, whatever task
 *   list the array holds then, so it is correct only while no call of
 *   another handle or batch size has installed its own list in between.
 *   Calls that overlap on the GPU (other streams, other handles on the same
 *   device, or mk_decode_step_noalloc from several host threads without
 *   ordering their streams) race on the array: order them.
 *   A model and batch size whose scratch exceeds MK_NOALLOC_SCRATCH_BYTES
 *   are rejected with MK_ERR_INVALID (mk_last_error gives the bytes needed).
 *   mk_debug_inject_stall does not apply to this entry point (its waits keep
 *   their ordinary limit). */
mk_status mk_decode_step_noalloc(mk_handle* h, const int32_t* tokens, const int32_t* positions, int B,
                                 mk_kv* kv, float* logits_out, int32_t* argmax_out, void* stream);

/* Speculative verify of one sequence (sequence 0 of the cache): tokens8 =
 * anchor followed by n_prop (<= 7) proposals, dev int32 [n_prop + 1], placed
 * at positions position .. position + n_prop, causal within the chunk.  K/V
 * are written for every position; the caller rewinds its length to
 * position + accepted + 1 (later entries are overwritten by the next step).
 *   logits_out: dev fp32 [n_prop + 1][vocab] or NULL
 *   argmax_out: dev int32 [n_prop + 1] (greedy token after each position)
 *   accepted_out: dev int32 [1] = largest n <= n_prop with
 *                 tokens8[j] == argmax_out[j - 1] for all 1 <= j <= n. */
mk_status mk_verify(mk_handle* h, const int32_t* tokens8, int n_prop, int32_t position, mk_kv* kv,
                    float* logits_out, int32_t* argmax_out, int32_t* accepted_out, void* stream);

/* Prefill: run the model over a prompt of n tokens of cache sequence `seq`
 * at positions start .. start + n - 1, writing their K/V (or latent rows)
 * into the cache.  The prompt is processed in chunks of min(8, max_batch)
 * positions, each one launch of the verify form (the positions of a chunk as
 * the rows of one step, causal within the chunk; section "DSpark" of the
 * pages checks 8 positions per launch the same way).  Asynchronous on
 * `stream`; device errors as for mk_decode_step.
 *   tokens: dev int32 [n]
 *   argmax_last: dev int32 [1] (greedy token after the last position) or NULL
 * Positions outside [0, kv max_ctx) or seq outside [0, kv max_seqs) are
 * rejected on the host (MK_ERR_INVALID). */
mk_status mk_prefill(mk_handle* h, const int32_t* tokens, int n, int seq, int32_t start, mk_kv* kv,
                     int32_t* argmax_last, void* stream);

/* Speculative greedy generation ("DSpark" section of the pages: each launch
 * checks an anchor and up to 7 proposed continuations, keeps the accepted
 * prefix plus one greedy "bonus" token, and rewinds the rest).  Runs on
 * cache sequence 0, which holds positions 0 .. position - 1.
 *
 * The draft is the caller's: before every verify launch the library calls
 *   draft(user, history, n_history, proposals, max_k)
 * with history = the anchor followed by every token emitted so far (host
 * memory, valid during the call); it writes up to max_k (<= 7) proposed
 * next tokens into proposals (host) and returns how many it wrote (values
 * outside [0, max_k] are clamped).  The verify launch (mk_verify) places the
 * anchor at the current position and the proposals after it; with `a`
 * proposals accepted, the emitted tokens are those a proposals and the greedy
 * token after the last accepted one, which becomes the next anchor one
 * position past them (later cache rows are overwritten by the next launch).
 * The emitted sequence is the one plain greedy decoding (mk_decode_step fed
 * its own argmax) produces, whatever the draft proposes.
 *   out_tokens: host int32 [n_out], the emitted tokens in order
 *   stats: host, optional: launches, proposed, accepted and emitted tokens
 * Synchronous: the host reads each launch's accepted count before the next.
 * MK_ERR_INVALID when the cache cannot hold the next launch's positions;
 * device errors are returned as by mk_sync_status. */
typedef int32_t (*mk_draft_fn)(void* user, const int32_t* history, int32_t n_history, int32_t* proposals,
                               int32_t max_k);
typedef struct {
  int64_t launches, proposed, accepted, emitted;
} mk_spec_stats;
mk_status mk_spec_generate(mk_handle* h, mk_kv* kv, int32_t anchor, int32_t position, int32_t n_out,
                           mk_draft_fn draft, void* user, int32_t* out_tokens, mk_spec_stats* stats, void* stream);

/* Debug outputs of the next compute calls (dev pointers, or NULL to stop):
 * router expert indices int32 [layers][rows][top_k] and weights fp32 (same
 * shape) in top-k order. */
mk_status mk_set_router_trace(mk_handle* h, int32_t* idx_dev, float* w_dev);

/* Debug trace of the next compute calls.  While a buffer is set, steps run
 * an instrumented instance of the kernel (same arithmetic and results; the
 * ordinary instance carries no tracing code).  For every task of every CTA it
 * writes 20 int64 into trace_dev[cta][task][20]:
 *   0-2   %globaltimer (ns) at task start, when its dependency was met, at its end;
 *   3-4   SM cycles spent waiting for weight tiles, for activation slices;
 *   5-7   chunks consumed, layer (+ the task's phase << 16: the tasks between
 *         two dependency points, one kernel of the multi-kernel path),
 *         type * 16 + epilogue;
 *   8-11  cycles in fragment preparation, mma, epilogue, release;
 *   12-15 (record 0) producer cycles blocked on a full ring, chunks issued,
 *         first and last issue time (ns); (record 1) producer cycles and ns
 *         over its lifetime (the SM clock); (later records) field 12 holds
 *         the cycles spent waiting for the MoE route;
 *   16-19 cycles in the chunk loop, before it, after it, signalling.
 * The buffer holds ctas x max_tasks_per_cta records (mk_launch_info gives the
 * CTA count); later tasks are not recorded.  NULL disables. */
mk_status mk_set_trace(mk_handle* h, int64_t* trace_dev, int32_t max_tasks_per_cta);

/* Read the device status word (call after the stream has been synchronised).
 * Returns MK_OK or the recorded device error; errors stay until mk_reset. */
mk_status mk_sync_status(mk_handle* h);

/* Clear a sticky device error and all inter-CTA counters.  Synchronous. */
mk_status mk_reset(mk_handle* h);

/* Number of persistent CTAs (one per SM) and dynamic shared memory per CTA. */
mk_status mk_launch_info(mk_handle* h, int32_t* ctas, int32_t* smem_bytes, int32_t* threads);

/* Bytes of device memory held for weights. */
int64_t mk_weight_bytes(const mk_handle* h);

/* Test hook: make the next compute call wait on a dependency counter that
 * nothing signals, with a wait limit of `timeout_ns`, so that it returns
 * MK_ERR_DEVICE_TIMEOUT through mk_sync_status.  0 disables. */
mk_status mk_debug_inject_stall(mk_handle* h, int64_t timeout_ns);

/* The description of h's last failure; with h == NULL, why the calling
 * thread's last mk_create failed. */
const char* mk_last_error(const mk_handle* h);
void mk_kv_destroy(mk_kv* kv);
void mk_destroy(mk_handle* h);

#ifdef __cplusplus
}
#endif
#endif /* MK_H */
