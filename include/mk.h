/*
 * mk.h -- C ABI of the B200 decode megakernel for parallel-layer MoE decoders.
 *
 * One call of mk_decode_step runs one whole small-batch (B <= 8) decode step
 * of a parallel-transformer MoE decoder as ONE persistent kernel with one
 * resident CTA per SM.  Each CTA interprets a host-built list of fixed-size
 * int32 task descriptors (one opcode per tile of an operation); tasks wait on
 * and signal global-memory counters instead of kernel boundaries, and weight
 * tiles are streamed into shared memory by TMA ahead of their activation
 * dependency.
 *
 * Sources (the method this library implements):
 *  - agenticcommons.xyz, "Cohere North Mini Code megakernel serving engine":
 *    section "How the megakernel works" (one persistent block per SM, a task
 *    list in global memory, one task = one tile of one operation, counters
 *    incremented on completion and spun on by consumers); section "Three
 *    sources of speedup", items 1-3 (backfill across a parallel transformer
 *    layer whose attention and MoE read the same normalized input and merge
 *    through a fused residual add + RMSNorm; per-KV-group O-proj and
 *    per-expert down-projection dependencies; weight prefetch before the
 *    activation dependency resolves).
 *  - aimodeling.com, "Cohere megakernel engine: one CUDA file, 1.58x vLLM on H100":
 *    sections "One persistent kernel for the whole decode step" and "From
 *    demo to a full serving system" (continuous batching, paged attention,
 *    ragged sequence lengths, at most 8 sequences, one calling convention).
 *
 * Conventions for every entry point:
 *  - All tensors are owned by the caller; the library never frees them and
 *    keeps the pointers for the lifetime of the context.  Device pointers are
 *    plain CUDA device addresses on the context's device.
 *  - Every entry point returns an mk_status; nothing is thrown or aborted.
 *    Arguments are validated before any launch.  Failures detected on the
 *    device (a counter wait that exceeded its deadline, an out-of-range page
 *    id or position) are latched in a device status word read by mk_check.
 *  - bf16 tensors are IEEE binary16-brain (upper half of a binary32), row
 *    major, dense, 16-byte aligned base addresses.
 */
#ifndef MK_H_
#define MK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mk_status {
  MK_OK = 0,
  MK_ERR_INVALID = 1,   /* bad argument (shape, pointer, batch, length, page id) */
  MK_ERR_CUDA = 2,      /* a CUDA runtime/driver call failed                      */
  MK_ERR_OOM = 3,       /* device allocation failed                               */
  MK_ERR_TIMEOUT = 4,   /* a device-side wait exceeded its deadline (mk_check)    */
  MK_ERR_CAPACITY = 5,  /* request exceeds a compiled-in or configured capacity   */
  MK_ERR_STATE = 6,     /* call out of order (no schedule, schedule outgrown)     */
  MK_ERR_DEVICE = 7     /* device-side validation failed (mk_check detail)        */
} mk_status;

/* Model shape.  Requirements (checked by mk_create): head_dim in {64, 128};
 * d_model, d_ff multiples of 64 with d_model / 64 <= 64 tiles; n_q_heads a
 * multiple of n_kv_heads; n_q_heads / n_kv_heads <= 4; n_experts <= 256 and
 * a multiple of 4 (the router logits are summed as float4 columns);
 * top_k <= 8; page_size == 64; max_batch in [1, 8].  n_pages is the number
 * of physical pages in each layer's K and V pool.                           */
typedef struct mk_config {
  int32_t n_layers;
  int32_t d_model;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t n_experts;
  int32_t top_k;
  int32_t d_ff;
  int32_t vocab;
  int32_t page_size;
  int32_t max_batch;
  int32_t n_pages;
  float rope_theta;
  float rms_eps;
} mk_config;

/* Model tensors (device pointers, bf16 unless noted).  Arrays of per-layer
 * pointers are HOST arrays of n_layers device pointers.
 *   embed       [vocab][d_model]
 *   lm_head     [vocab][d_model]               (untied)
 *   final_norm  [d_model]
 *   attn_norm[l][d_model]                      (the one RMSNorm gain of layer l,
 *                                               read by both branches)
 *   w_qkv[l]    [(Hq + 2 Hkv) * hd][d_model]   rows: q heads, k heads, v heads
 *   w_o[l]      [d_model][Hq * hd]
 *   w_router[l] [n_experts][d_model]
 *   router_bias NULL, or host array of n_layers device pointers to float32
 *               [n_experts] (an entry may be NULL: no bias for that layer)
 *   w_gate[l]   [n_experts][d_ff][d_model]
 *   w_up[l]     [n_experts][d_ff][d_model]
 *   w_down[l]   [n_experts][d_model][d_ff]
 *   k_pool[l], v_pool[l]  [n_pages][Hkv][page_size][hd]  (post-RoPE K, raw V;
 *               written in place: the step appends the new token's K and V) */
typedef struct mk_tensors {
  const void* embed;
  const void* lm_head;
  const void* final_norm;
  const void* const* attn_norm;
  const void* const* w_qkv;
  const void* const* w_o;
  const void* const* w_router;
  const float* const* router_bias;
  const void* const* w_gate;
  const void* const* w_up;
  const void* const* w_down;
  void* const* k_pool;
  void* const* v_pool;
} mk_tensors;

typedef struct mk_ctx mk_ctx;

/* Create a context on `device`: validates the shape, encodes the TMA tensor
 * maps of every weight and KV pool, allocates the context-owned device
 * memory (descriptors, counters, per-layer activation buffers, status word).
 * On success *out receives the context; on failure *out is set to NULL.     */
mk_status mk_create(const mk_config* cfg, const mk_tensors* tensors, int device,
                    mk_ctx** out);

/* Build and upload the task schedule for `batch` sequences (1..max_batch).
 * seq_lens: HOST int32[batch], tokens already cached per sequence.
 * max_pages_per_seq: row stride of the page table later passed to
 * mk_decode_step.  The schedule's attention chunk plan covers sequences up to
 * `plan_len` cached tokens each (HOST int32[batch]; NULL means seq_lens + 64),
 * so one schedule serves many consecutive steps.  Zeroes the counters.
 * Synchronizes the device.                                                  */
mk_status mk_build_schedule(mk_ctx* ctx, int batch, const int32_t* seq_lens,
                            const int32_t* plan_len, int32_t max_pages_per_seq);

/* Run one decode step on `stream` (a cudaStream_t; NULL = legacy stream).
 * Device inputs:
 *   tokens     int32[batch]    token fed to each entry
 *   positions  int32[batch]    position of each entry's token: seq_lens[b],
 *              or seq_lens[b] + g for the (g+1)-th token of a prefill group
 *   page_table int32[batch][max_pages_per_seq]  logical page -> physical page;
 *              the entry for page positions[b] / page_size must already be a
 *              valid page (the step writes the new K/V there)
 *   seq_lens   int32[batch]    cached tokens before the step
 * Device output:
 *   logits     float32[batch][vocab]
 * Chunked prefill: up to `batch` consecutive prompt tokens of one sequence
 * run as consecutive entries b0 .. b0 + M - 1 with equal seq_lens (the cached
 * prefix, possibly 0), positions seq_lens + 0 .. M - 1 and the same
 * page-table row.  Entry b0 + g attends to the prefix and to tokens b0 ..
 * b0 + g (causal), so its logits are those of a decode step at its position
 * after the tokens before it; all M tokens' K/V are appended.  Groups and
 * single decode entries mix freely in one batch.  A position that breaks
 * these rules (positions[b] - seq_lens[b] outside 0 .. b, or an entry whose
 * predecessor is not the previous token of its group) stops the step with a
 * device-side error before any attention reads out of the group.
 * Asynchronous: returns after the launch.  Returns MK_ERR_STATE before any
 * schedule was built.  Device-side errors surface through mk_check.         */
mk_status mk_decode_step(mk_ctx* ctx, const int32_t* tokens, const int32_t* positions,
                         const int32_t* page_table, const int32_t* seq_lens,
                         float* logits, void* stream);

/* Greedy decoding: n_steps fused steps back to back on `stream`, with no host
 * round trip between them.  Step i reads tokens, positions and seq_lens as
 * mk_decode_step does and writes logits; its last LM-head tile to finish also
 * writes each sequence's greedy token (the largest logit, the lowest token id
 * among equal ones) to out_tokens[i][b] and to tokens[b], the next step's
 * input, and advances positions[b] and seq_lens[b] by one (once if both
 * pointers name the same buffer).  Each LM-head tile folds its rows' best
 * logit per sequence into a 64-bit key with one atomicMax, so the step's
 * argmax costs no extra pass over the logits.  This is the greedy step after
 * the LM head of the pages' serving loop (aimodeling.com, "Cohere megakernel
 * engine: one CUDA file, 1.58x vLLM on H100", "From demo to a full serving
 * system"), done on the device.
 *   tokens, positions, seq_lens  int32[batch], device, read and updated;
 *               positions must equal seq_lens (no prefill groups)
 *   page_table  as for mk_decode_step; it must already map the page of every
 *               token the n_steps steps append
 *   logits      float32[batch][vocab], device: the last step's logits
 *   out_tokens  int32[n_steps][batch], device
 * The schedule's plan length must cover seq_lens + n_steps (else the step
 * that outgrows it latches MK_ERR_STATE).  Asynchronous like mk_decode_step;
 * n_steps == 0 does nothing.                                               */
mk_status mk_decode_greedy(mk_ctx* ctx, int32_t n_steps, int32_t* tokens, int32_t* positions,
                           const int32_t* page_table, int32_t* seq_lens, float* logits,
                           int32_t* out_tokens, void* stream);

/* Same step as mk_decode_step, but issued as one launch of the same task
 * interpreter per operation phase (about nine per layer), so kernel
 * boundaries replace the cross-SM counters.  This is the unfused per-op
 * baseline built from the library's own tile routines.                      */
mk_status mk_decode_step_unfused(mk_ctx* ctx, const int32_t* tokens,
                                 const int32_t* positions, const int32_t* page_table,
                                 const int32_t* seq_lens, float* logits, void* stream);

/* Capacity of the fixed scratch array used by mk_decode_step_static. */
#define MK_STATIC_SCRATCH_MAX_BYTES (32u * 1024u * 1024u)

/* The same fused step as mk_decode_step, for callers that must not allocate
 * device memory while they run: for example a serving process whose own
 * memory pool has already reserved the device's free memory, or code that
 * runs where an allocation's implicit device synchronization would stall
 * other streams.  The pages describe no such entry point; it is an addition
 * of this library.
 *
 * The step's scratch (counters, routing words, activations, attention and
 * expert partials) lives in one file-scope device array of
 * MK_STATIC_SCRATCH_MAX_BYTES (32 MiB) instead of the context's buffers.
 * mk_create looks up the array's device address (cudaGetSymbolAddress, with
 * the device current), which loads the array on that device if it is not
 * loaded yet; it then stays reserved there until the process exits.  This
 * call itself loads nothing and allocates nothing.  The context (from
 * mk_create and mk_build_schedule, which do allocate) supplies the schedule,
 * tensor maps and status word; arguments and device inputs are those of
 * mk_decode_step.
 *  - Returns MK_ERR_CUDA, before any launch, if mk_create could not resolve
 *    the array on this device (for example when no room was left for it).
 *  - Every call, from every context, shares the one array and leaves its
 *    contents in place; each call clears the counters and routing words on
 *    `stream` before the launch.  Calls that overlap on the GPU (other
 *    streams, other contexts on the same device) race on the array: order
 *    them on one stream.
 *  - Returns MK_ERR_CAPACITY, before any launch, when the current schedule
 *    needs more than MK_STATIC_SCRATCH_MAX_BYTES (the 30B-MoE shape fits at
 *    batch 1, not at batch 8); MK_ERR_STATE before any schedule was built.
 *  - It records no trace and does not update the buffers mk_debug_read
 *    returns; device errors surface through mk_check as usual.             */
mk_status mk_decode_step_static(mk_ctx* ctx, const int32_t* tokens, const int32_t* positions,
                                const int32_t* page_table, const int32_t* seq_lens,
                                float* logits, void* stream);

/* Synchronize the stream of the context's last step (the whole device when no
 * step has been launched yet) and read the device status word.
 * device_status (may be NULL) receives MK_OK or the latched device error;
 * detail (may be NULL) receives int32[8]: {code, cta, task, opcode, counter,
 * observed, target, aux}.  Returns MK_OK if the device status is clean, else
 * the device status.  Clears the latched status.                           */
mk_status mk_check(mk_ctx* ctx, int32_t* device_status, int32_t* detail);

/* Failure-detection self-test: runs the task interpreter on a one-task list
 * whose only dependency is a counter that nothing signals, with a deadline
 * of `timeout_ms` per device wait.  The wait runs out by design (no fault,
 * no trap, no unbounded spin): the kernel latches MK_ERR_TIMEOUT in the
 * status word, every CTA leaves its task loop, and this call synchronizes,
 * reads and clears the status (device_status and detail as for mk_check).
 * Returns MK_ERR_TIMEOUT when detection works, MK_ERR_STATE before any
 * schedule was built.  Uses its own counters: the step's counters, epoch and
 * outputs are untouched, and the next mk_decode_step runs normally.
 * (The pages describe no failure handling; the bounded waits are this
 * library's own.)                                                           */
mk_status mk_selftest_timeout(mk_ctx* ctx, int32_t timeout_ms, int32_t* device_status,
                              int32_t* detail);

/* Record per-task timestamps in every following fused step (enable != 0),
 * readable with mk_debug_read(MK_BUF_TRACE).  Costs a few global stores per
 * task.  Default off.                                                       */
mk_status mk_set_trace(mk_ctx* ctx, int32_t enable);

/* Per-wait deadline in milliseconds for device-side spins (default 2000). */
mk_status mk_set_timeout_ms(mk_ctx* ctx, int32_t ms);

/* Copy one of the context's per-step buffers to host memory (synchronous),
 * for per-operation parity checks and statistics.  `which` selects:
 *   MK_BUF_X        float [L+1][B][d]        residual entering each layer
 *                                            (index L: entering the final norm)
 *   MK_BUF_QKV      float [L][B][(Hq+2Hkv)hd] QKV projection (before RoPE)
 *   MK_BUF_ATTN_O   float [L][B][Hq*hd]      attention output per head
 *   MK_BUF_RLOGITS  float [L][B][E]          router logits (bias included)
 *   MK_BUF_TOPK     int32 [L][B][k] expert ids, then float [L][B][k] weights
 *   MK_BUF_NSLOTS   int32 [L]                experts touched per layer
 *   MK_BUF_EXPERT_A float [L][S][B][F]       SwiGLU activation per slot
 *   MK_BUF_MOE      float [L][k][B][d]       weighted expert outputs by rank
 *   MK_BUF_OPART    float [L][Hkv][B][d]     O-proj output per KV group
 *   MK_BUF_TRACE    uint32 [n_tasks][18] per task of the last traced step (see
 *                   mk_set_trace): globaltimer stamps (ns, low 32 bits) of
 *                   producer resolved, producer issued last stage, loader
 *                   deps met, loader activation issued, consumer picked up,
 *                   consumer has activation, consumer math done, consumer
 *                   epilogue done; then the CTA that ran it, plus one; then
 *                   SM clock cycles the consumer waited for stage data, of
 *                   the consumer's whole stage loop, and the producer waited
 *                   for free stages; then the consumer's SM clock (low 32
 *                   bits) at pickup, activation ready, tile routine entry,
 *                   stage loop end, reduction end, epilogue end
 *   MK_BUF_PLAN     int32 [n_tasks][32] descriptors of the schedule
 * `bytes` must equal the buffer's size for the current schedule.            */
enum {
  MK_BUF_X = 0,
  MK_BUF_QKV = 1,
  MK_BUF_ATTN_O = 2,
  MK_BUF_RLOGITS = 3,
  MK_BUF_TOPK = 4,
  MK_BUF_NSLOTS = 5,
  MK_BUF_EXPERT_A = 6,
  MK_BUF_MOE = 7,
  MK_BUF_OPART = 8,
  MK_BUF_TRACE = 9,
  MK_BUF_PLAN = 10
};
mk_status mk_debug_read(mk_ctx* ctx, int which, void* host_dst, size_t bytes);
size_t mk_debug_size(mk_ctx* ctx, int which);

/* Host-only schedule planner (no GPU needed): the task list mk_build_schedule
 * would upload, sized for `n_ctas` CTAs (attention chunks are cut so the KV
 * stream spreads over them).  The list is in topological priority order; at
 * run time every CTA takes the next task with an atomic add.
 *   meta (HOST int32[16]) receives {n_tasks, n_counters, n_slots, max_chunks,
 *   desc_words, n_phases, qkv_rows_per_tile, pages_per_chunk, dispenser
 *   counter, first phase dispenser counter, ring stages per CTA, 1 if an
 *   attention chunk works in its own activation buffer (else 0), 0...}.
 *   desc (HOST int32[n_tasks][desc_words] or NULL) receives the descriptors;
 *   pass NULL first to learn n_tasks from meta.
 *   targets (HOST int32[n_counters] or NULL) receives each counter's
 *   per-step arrival count.                                                 */
mk_status mk_plan_schedule(const mk_config* cfg, int n_ctas, int batch,
                           const int32_t* seq_lens, const int32_t* plan_len,
                           int32_t* meta, int32_t* desc, int32_t* targets);

const char* mk_strerror(mk_status s);

/* Release everything the context owns (not the caller's tensors). */
void mk_destroy(mk_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* MK_H_ */
