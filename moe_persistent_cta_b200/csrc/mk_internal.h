// mk_internal.h -- task descriptor format, opcodes, counter layout and the
// kernel parameter block shared by the host planner, the host library and the
// persistent interpreter.
//
// The descriptor format follows the pages' "uniform ABI" of fixed-size int32
// task records (aimodeling.com, "Cohere megakernel engine: one CUDA file,
// 1.58x vLLM on H100", section "Caveats and takeaways": 32 int32 per task); the field
// assignment below is this library's own.
#pragma once

#include <stdint.h>
#include <stddef.h>

#if defined(__CUDACC__)
#define MK_HD __host__ __device__
#else
#define MK_HD
#endif

namespace mk {

constexpr int kDescWords = 32;
constexpr int kPage = 64;            // tokens per KV page
constexpr int kMaxBatch = 8;         // mma N (token columns) and the pages' batch cap
constexpr int kMaxTopK = 8;
constexpr int kStageBytes = 16384;   // one ring stage = 8 units of 16 rows x 64 k (bf16)
constexpr int kUnitBytes = 2048;
constexpr int kConsumerWarps = 8;
constexpr int kProducerWarp = 0;     // TMA weight/KV streamer + task resolver
constexpr int kLoaderWarp = 1;       // dependency waits + activation loads
constexpr int kSignalWarp = 2;       // completion signals (release adds)
constexpr int kEpilogueWarp = 3;     // GEMV partial reduction and outputs
constexpr int kFirstConsumerWarp = 4;   // warps 4..11: two whole warpgroups
constexpr int kThreads = (kFirstConsumerWarp + kConsumerWarps) * 32;   // 384
// Registers per thread after the split (setmaxnreg) of the launch's
// kThreads x 168 = 64,512: warpgroup 0 (the single-warp roles) keeps
// kRoleRegs, the consumers get kConsumerRegs, 63,488 in all.  A split above
// the launch's registers would leave the increase waiting forever.
constexpr int kRoleRegs = 80;
constexpr int kConsumerRegs = 208;
static_assert(128 * kRoleRegs + 256 * kConsumerRegs <= kThreads * 168,
              "register split exceeds the launch's registers");
static_assert(kRoleRegs % 8 == 0 && kConsumerRegs % 8 == 0 && kConsumerRegs <= 256,
              "setmaxnreg takes multiples of 8 up to 256");
constexpr int kRstdRing = 4;         // per-level 1/rms slots (levels in flight)
constexpr int kMaxParts = 1 + 16 + kMaxTopK;   // residual + O-proj groups + expert ranks
constexpr int kFifo = 16;            // task entries in flight per CTA
constexpr int kFifoEntryWords = 64;  // 32 descriptor words + 32 resolved words
constexpr int kMapsPerLayer = 8;     // qkv, o, router, gate, up, down, kpool, vpool
constexpr int kMapRouter = 2;
// Activation rows are padded by 8 floats so that the 8 columns a warp reads
// at one k land in different shared-memory banks.
constexpr int kActPad = 8;
constexpr int kRnStage = 1536;       // floats of the norm tile's staging area (group sums, gamma x, part pointers)
constexpr int kRouterRowsPerStage = 128;   // router weight rows (x 64 columns) per ring stage
constexpr int kMaxAttnOut = 512;    // G x hd floats of one (token, KV head) output (G <= 4, hd <= 128)
// Batch sizes up to which each producer computes a layer's routing table
// itself from the norm tiles' accumulators (one warp, a few microseconds),
// instead of waiting for the layer's top-k task and copying its table.
constexpr int kLocalRouteMaxB = 4;
// Attention chunks of up to this many pages let their CTA take its next task
// before the chunk's stages are issued; longer chunks take it afterwards.
constexpr int kEarlyTakeMaxPages = 32;
// expert bitmasks of the routing compaction: the union (8 words, E <= 256),
// then one per token
constexpr int kRouteMaskWords = 8 + 8 * kMaxBatch;
// words of the producer's routing scratch after its copy of the routing
// table: selections and weights [8][8] each, and the expert bitmasks
constexpr int kRouteTmpWords = 64 + 64 + kRouteMaskWords;
// Per-layer pointer table in shared memory: norm weights of levels 0..L (the
// final norm last), then router bias, K pool and V pool of layers 0..L-1.  A
// task reads its layer's pointers from there, so its first global loads need
// no dependent pointer load.
MK_HD constexpr int ptr_table_words(int L) { return 4 * L + 1; }
constexpr int kTraceWords = 18;      // per task: see TraceField

// Per-task trace words: globaltimer stamps (low 32 bits, ns) and the CTA
// that ran the task.
enum TraceField : int {
  T_P_RESOLVED = 0,   // producer wrote the task's entry
  T_P_ISSUED = 1,     // producer issued the task's last stage
  T_L_DEPS = 2,       // loader saw the task's counters satisfied
  T_L_ACT = 3,        // loader issued the task's activation copy
  T_C_READY = 4,      // consumers picked the task up
  T_C_ACT = 5,        // consumers have the activation
  T_C_MATH = 6,       // consumers finished the streamed stages
  T_C_END = 7,        // consumers finished the epilogue
  T_CTA = 8,          // CTA index + 1
  T_C_WAITCYC = 9,    // SM cycles consumer warp 0 waited for stage data
  T_C_LOOPCYC = 10,   // SM cycles of the consumer's stage loop
  T_P_WAITCYC = 11,   // SM cycles the producer waited for free stages
  T_K0 = 12,          // SM clock (low 32 bits) at: consumer pickup,
  T_K1 = 13,          //   activation ready,
  T_K2 = 14,          //   tile routine entry,
  T_K3 = 15,          //   stage loop end,
  T_K4 = 16,          //   cross-warp reduction end,
  T_K5 = 17           //   epilogue end
};

// ---------------------------------------------------------------- opcodes --
enum Op : int32_t {
  OP_NONE = 0,
  OP_RN = 1,        // fused residual add + RMSNorm statistics for one 64-row tile
  OP_QKV = 2,       // QKV projection tile (RoPE/append happen in OP_ATTN)
  OP_ROUTER = 3,    // (unused: the norm tiles produce the router logits)
  OP_TOPK = 4,      // top-k + softmax + expert-slot compaction
  OP_ATTN = 5,      // paged GQA decode attention over one KV chunk (+RoPE, append)
  OP_COMBINE = 6,   // (unused: the last-arriving attention chunk of (b, g) merges)
  OP_OPROJ = 7,     // O-proj tile, split-K by KV group
  OP_GATEUP = 8,    // expert gate+up tile with SwiGLU epilogue
  OP_DOWN = 9,      // expert down tile with weighted scatter into rank slots
  OP_LMHEAD = 10,   // LM head tile
  OP_COUNT = 11
};

// ------------------------------------------------------- descriptor words --
enum DescField : int {
  D_OP = 0,
  D_LAYER = 1,
  D_A = 2,          // tile / batch index / slot
  D_B = 3,          // tile / group
  D_C = 4,          // attention: chunk; expert tiles: list index one past the
                    // layer's last tile of the same operation (see D_A)
  D_D = 5,          // chunk count
  D_FLAGS = 6,
  D_NWAIT = 7,
  D_W0 = 8, D_W0N = 9, D_W1 = 10, D_W1N = 11,   // loader waits (counter, arrivals/step)
  D_PW = 12, D_PWN = 13,                        // producer wait (-1: none)
  D_NSIG = 14, D_S0 = 15, D_S1 = 16,            // signalled counters
  D_NSTAGE = 17,    // ring stages streamed (static part)
  D_ROW0 = 18,      // GEMV: first row (per-expert offset added at run time)
  D_K0 = 19,        // GEMV: first column
  D_KCH = 20,       // GEMV: 64-column chunks
  D_R = 21,         // GEMV: rows per tile (TMA box height)
  D_NMAT = 22,      // GEMV: matrices per tile (2 = gate+up)
  D_MAP0 = 23, D_MAP1 = 24,                     // tensor-map indices
  D_ACT = 25,       // activation: 0 none, 1 normalized input of level D_LAYER
                    // (slot A, reused while the level repeats), 2 small (slot B)
  D_PPC = 27,       // attention: pages per chunk
  D_PHASE = 28,     // operation phase (for the unfused launcher)
  D_X0 = 29, D_X1 = 30, D_X2 = 31   // last-arriver: arrival counter, arrivals, join signal
};

enum ActKind : int32_t { ACT_NONE = 0, ACT_A = 1, ACT_B = 2 };

enum Flags : int32_t {
  F_LAST_CHUNK = 8,  // attention chunk that owns the new token (and appends it)
  F_SINGLE = 16,     // attention of (b, g) in one chunk: write the final output
  // Last-arriver work: after its own outputs, the task adds 1 to counter
  // D_X0 (D_X1 arrivals per step); the task that completes the count does the
  // join below and then signals counter D_X2.
  F_COMBINE = 128,   // attention chunk: log-sum-exp merge of the (b, g) chunks
  F_ARGMAX = 512     // LM-head tile: in a greedy step, the tokens of the step
};

// ------------------------------------------------- resolved entry words ---
// Written by the producer into the FIFO entry after the 32 descriptor words.
enum ResolvedField : int {
  R_NSTAGE = 0,     // stages actually streamed for this task
  R_EXPERT = 1,     // expert id (-1: empty slot)
  R_NTOK = 2,       // tokens in the slot / pages in the chunk
  R_P0 = 3,         // attention: first logical page of the chunk
  R_SEQLEN = 4,     // attention: cached tokens of the sequence
  R_PHYS_NEW = 5,   // attention: physical page receiving the new token
  R_TASK = 6,       // index of the task in the step's list (-1: no more tasks)
  R_POS = 7,        // attention: position of the new token (seq_len + its index
                    //   in a prefill group)
  R_TOK = 8,        // [8] slot token ids
  R_RANK = 16,      // [8] rank of the expert in each token's top-k
  R_W = 24          // [8] routing weight (float bits)
};

// ------------------------------------------------------------- params -----
struct Params {
  // shape
  int L, d, Hq, Hkv, hd, E, k, F, V, B, S, G, NR, qkvR;
  int max_chunks, max_pages, n_pages, part_stride;
  float eps;
  // byte sizes of the activation formats
  int actA_bytes;      // per level: rows of gamma*x (fp32) + ss partials
  int actA_rows_bytes; // per level: the rows part, B x (d + kActPad) floats
  int ofrag_bytes;     // per (layer, group): B x (G*hd + kActPad) floats
  int afrag_bytes;     // per (layer, slot): B x (F + kActPad) floats
  int route_words;     // per layer
  // schedule: one list in topological priority order; CTAs take the next
  // task with an atomic add on counters[grab].  The dispenser starts every
  // launch at 0: the last producer to leave (counted on counters[exit_ctr])
  // zeroes it, so it may also be moved forward past tasks that turn out to
  // be empty (expert tiles of unused slots).
  const int32_t* desc;     // [n_tasks][kDescWords]
  int n_tasks;
  int n_ctas;
  int grab;                // counter index of the task dispenser
  int exit_ctr;            // counter index of the producers' exit count
  // counter layout the top-k needs to stand in for the unused slots' tiles:
  // slot counters [L][S] from slot_ctr0, down-tile row counters [L][NR]
  // from dt_ctr0 (n_ff gate/up tiles per slot)
  int slot_ctr0, dt_ctr0, n_ff;
  uint32_t* counters;
  uint32_t epoch;
  // tensors
  const void* tmaps;       // CUtensorMap[L * kMapsPerLayer + 1]
  const uint16_t* embed;
  const uint16_t* final_norm;
  const uint16_t* const* attn_norm;   // device array [L]
  const float* const* router_bias;    // device array [L] (entries may be null)
  uint16_t* const* k_pool;            // device array [L]
  uint16_t* const* v_pool;            // device array [L]
  const double* inv_freq;             // [hd/2]
  // step inputs / output
  const int32_t* tokens;
  const int32_t* positions;
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* logits;
  // greedy steps (null otherwise): the step's token ids (read by the
  // embedding, overwritten with the greedy tokens), positions and lengths
  // (advanced by one), and this step's row of the caller's token output
  int32_t* g_tok;
  int32_t* g_pos;
  int32_t* g_len;
  int32_t* g_out;
  unsigned long long* amax;   // [B] best (logit, lowest row) keys, zero between steps
  // context buffers
  float* x;          // [L+1][B][d]
  uint8_t* actA;     // [L+1][actA_bytes]
  float* qkv;        // [L][B][qkvR]
  float* cs;         // [B][hd]  cos | sin
  float* attn_part;  // [L][B][Hkv][max_chunks][part_stride]
  float* attn_o;     // [L][B][Hq*hd]
  uint8_t* ofrag;    // [L][Hkv][ofrag_bytes]
  float* o_part;     // [L][Hkv][B][d]
  float* rlogits;    // [L][B][E]
  unsigned long long* racc;    // [2][L][B][E] router logit shares, fixed point (2^-32),
                               // by step parity (epoch & 1)
  unsigned long long* ssacc;   // [2][L][B] sums of squares of the layer's input, fixed point
  int32_t* route;    // [L][route_words]
  float* expert_a;   // [L][S][B][F]
  uint8_t* afrag;    // [L][S][afrag_bytes]
  float* moe_part;   // [L][k][B][d]
  int32_t* status;   // [16]
  uint32_t* trace;   // null, or [n_tasks][kTraceWords]
  unsigned long long timeout_cycles;   // per-wait deadline in SM clock cycles
  // shared-memory layout (byte offsets from the 1024-aligned base)
  int n_stages, nA, actA_stride;
  int off_bars, off_fifo, off_scratch, off_actA, off_actB, actB_bytes, off_ring;
  // 1: an attention chunk keeps its per-warp merge area and rotated query in
  // its own B buffer, after the chunk's inputs (when the buffer has the room);
  // 0: in the scratch area
  int attn_in_actB;
  int off_epi;       // GEMV partials [2][kConsumerWarps][16][part_cols], then the
                     // per-level 1/rms ring [kRstdRing][kMaxBatch]
  int off_ptrs;      // per-layer pointer table, copied in at launch (see PtrTable)
  int off_rcache;    // the producer's copy of one layer's routing table (route_words)
  int part_cols;     // token columns per partial row: B for B <= 2, else 8
  int smem_bytes;
};

// Counters and their targets (epoch x arrivals per step) are uint32 and wrap
// around; they are compared by signed difference, which stays right across
// the wrap as long as a counter never lags its target by 2^31 or more (a step
// adds at most a few thousand arrivals to any counter).
// reached(v, t): counter value v has reached target t.
MK_HD inline bool reached(uint32_t v, uint32_t t) { return (int32_t)(v - t) >= 0; }
// later(t1, t0): target t1 asks for more arrivals than target t0.
MK_HD inline bool later(uint32_t t1, uint32_t t0) { return (int32_t)(t1 - t0) > 0; }

// status word layout
enum StatusField : int {
  ST_CODE = 0, ST_CTA = 1, ST_TASK = 2, ST_OP = 3, ST_COUNTER = 4,
  ST_OBSERVED = 5, ST_TARGET = 6, ST_AUX = 7, ST_ABORT = 15
};

// routing table layout per layer (int32 words)
MK_HD inline int route_topk_idx(int B, int k) { (void)B; (void)k; return 1; }
MK_HD inline int route_topk_w(int B, int k) { return 1 + B * k; }
MK_HD inline int route_slot_expert(int B, int k) { return 1 + 2 * B * k; }
MK_HD inline int route_slot_ntok(int B, int k, int S) { return 1 + 2 * B * k + S; }
MK_HD inline int route_slot_tok(int B, int k, int S) { return 1 + 2 * B * k + 2 * S; }
MK_HD inline int route_slot_rank(int B, int k, int S) { return 1 + 2 * B * k + 2 * S + 8 * S; }
MK_HD inline int route_slot_w(int B, int k, int S) { return 1 + 2 * B * k + 2 * S + 16 * S; }
MK_HD inline int route_words(int B, int k, int S) {
  int w = 1 + 2 * B * k + 2 * S + 24 * S;
  return (w + 3) & ~3;
}

// ------------------------------------------------------------- planner ----
struct Shape {
  int L, d, Hq, Hkv, hd, E, k, F, V, page, max_batch, n_pages;
  float theta, eps;
};

struct Plan {
  int n_ctas = 0, B = 0, S = 0, max_chunks = 1, n_counters = 0, n_tasks = 0;
  int n_stages = 0, attn_in_actB = 0;   // from the shared-memory layout
  int n_phases = 0;
  int r_qkv = 16;
  int grab = 0;                      // dispenser counter of the fused list
  int grab_phase0 = 0;               // dispenser counters of the phase lists
  int exit_ctr = 0;                  // producers' exit count (resets the dispenser)
  int slot_ctr0 = 0, dt_ctr0 = 0, n_ff = 0;   // see Params
  int32_t* desc = nullptr;           // [n_tasks][kDescWords], fused priority order
  int32_t* targets = nullptr;        // [n_counters] arrivals per step
  // unfused launcher: the same tasks grouped by phase, phase ph being
  // phase_desc[phase_off[ph] .. phase_off[ph+1])
  int32_t* phase_desc = nullptr;
  int32_t* phase_off = nullptr;      // [n_phases + 1]
  int nc[kMaxBatch] = {0};           // attention chunks per sequence
  int ppc[kMaxBatch] = {0};          // pages per chunk per sequence
  void release();
};

// Shared-memory carve-up of one CTA for a shape and batch.
struct SmemLayout {
  int nA;             // normalized-input activation buffers (1 or 2)
  int actA_stride;    // bytes per A buffer
  int actB_bytes;     // bytes per small-activation buffer (two of them)
  int scratch_bytes;
  int attn_in_actB;   // see Params
  int n_stages;       // ring stages of kStageBytes
  int off_bars, off_fifo, off_scratch, off_actA, off_actB, off_ring, off_epi, off_ptrs;
  int off_rcache;
  int part_cols;
  int total;          // bytes from the 1024-aligned base
  int dyn_bytes;      // dynamic shared memory to request (total + alignment slack)
};
int smem_layout(const Shape& s, int B, int max_chunks, SmemLayout* out);

// Returns MK_OK or MK_ERR_INVALID / MK_ERR_CAPACITY for an unsupported shape.
int validate_shape(const Shape& s);

// Validates the shape and builds the plan; returns 0 or an mk_status code.
int plan_schedule(const Shape& s, int n_ctas, int B, const int32_t* seq_lens,
                  const int32_t* plan_len, bool with_phases, Plan* out);
void group_by_phase(const Plan& plan, int32_t* out);

// GEMV tile geometry shared by planner and host (rows per tile for a K).
int gemv_rows_for(int K, int n_mat);

}  // namespace mk
