// mk_plan.cpp -- host schedule builder: decode step -> one task list.
//
// Every operation of the step is cut into tiles, one task per tile, emitted in
// one topological order that is also a priority order.  At run time every CTA
// takes the next task of that list with an atomic add (any free SM picks up
// the next tile, so no work is rounded up to whole waves: agenticcommons.xyz,
// "Cohere North Mini Code megakernel serving engine", section "Three sources
// of speedup", item 1).  A task only ever waits on tasks that are earlier in
// the list; those were taken earlier by CTAs that are running (all CTAs are
// co-resident) and that finish their tasks in order, so the step cannot
// deadlock.
//
// Dependencies are counters, one per producer group, with per-step arrival
// counts; a task waits until counter >= epoch * arrivals (section "How the
// megakernel works": increment on completion, spin on the producer).  The
// O-proj of one KV group waits only for that group's attention, and the down
// projection of one expert only for that expert's gate/up tiles (section
// "Three sources of speedup", item 2).
//
// Priority order inside a layer: the norm tiles (which also produce the
// router logits, share by share); QKV and top-k; attention chunks (their
// cached K/V stream before the new query exists); expert gate/up (the MoE
// branch is the longer one); then the attention tail and the expert down
// projections.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <queue>
#include <vector>

#include "mk.h"
#include "mk_internal.h"

namespace mk {

void Plan::release() {
  std::free(desc);
  std::free(targets);
  std::free(phase_desc);
  std::free(phase_off);
  desc = targets = phase_desc = phase_off = nullptr;
}

static int gcd_int(int a, int b) {
  while (b) {
    int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// Rows per GEMV tile: a ring stage holds 8 units of 16 rows x 64 columns; a
// tile of n_mat matrices x R rows consumes stages of (8 / (n_mat*R/16)) column
// chunks each, which must divide the K/64 chunks of the row.
int gemv_rows_for(int K, int n_mat) {
  int kc = K / 64;
  int per_stage = 8 / n_mat;                  // units per stage per matrix
  int kcps = gcd_int(per_stage, kc);          // column chunks per stage
  int mt = per_stage / kcps;                  // 16-row tiles per matrix
  return 16 * mt;
}

int validate_shape(const Shape& s) {
  if (s.L < 1 || s.d < 128 || s.d % 64 != 0 || s.d > 16384) return MK_ERR_INVALID;
  if (s.hd != 64 && s.hd != 128) return MK_ERR_INVALID;
  if (s.Hkv < 1 || s.Hq < s.Hkv || s.Hq % s.Hkv != 0) return MK_ERR_INVALID;
  if (s.Hkv > 16) return MK_ERR_CAPACITY;
  const int G = s.Hq / s.Hkv;
  if (G > 4) return MK_ERR_CAPACITY;
  if ((G * s.hd) % 128 != 0) return MK_ERR_INVALID;
  const int r_qkv = gemv_rows_for(s.d, 1);
  if (r_qkv > s.hd || s.hd % r_qkv != 0) return MK_ERR_INVALID;
  if (s.E < 1 || s.E > 256) return MK_ERR_CAPACITY;
  if (s.E % 4 != 0) return MK_ERR_INVALID;   // router logits summed as float4 columns
  if (s.k < 1 || s.k > kMaxTopK || s.k > s.E) return MK_ERR_INVALID;
  if (s.F < 128 || s.F % 128 != 0) return MK_ERR_INVALID;
  if (s.F % gemv_rows_for(s.d, 2) != 0) return MK_ERR_INVALID;
  if (s.V < 1) return MK_ERR_INVALID;
  if (s.page != kPage) return MK_ERR_INVALID;
  if (s.max_batch < 1 || s.max_batch > kMaxBatch) return MK_ERR_INVALID;
  if (s.n_pages < 1) return MK_ERR_INVALID;
  if (!(s.eps > 0.0f) || !(s.theta > 0.0f)) return MK_ERR_INVALID;
  return MK_OK;
}

static int round_up(int x, int a) { return (x + a - 1) / a * a; }

int smem_layout(const Shape& s, int B, int max_chunks, SmemLayout* o) {
  const int G = s.Hq / s.Hkv;
  const int NR = s.d / 64;
  const int actA_bytes = 4 * (s.d + kActPad) * B + round_up(NR * B * 4, 16);
  o->actA_stride = round_up(actA_bytes, 128);
  int b_need = std::max(4 * (G * s.hd + kActPad) * B,
                        std::max(4 * (s.F + kActPad) * B, (G + 3) * s.hd * 4));
  o->actB_bytes = round_up(b_need, 128);
  // attention's working area: the 8 warps' partial outputs, the rotated query
  // and the new token's K and V; in the chunk's own B buffer, after its inputs
  // (G + 3 rows of hd floats), where that buffer has the room (batch > 2)
  const int attn_work = 8 * G * (s.hd + 4) * 4 + G * s.hd * 4 + 2 * s.hd * 4;
  o->attn_in_actB = (G + 3) * s.hd * 4 + attn_work <= o->actB_bytes ? 1 : 0;
  int sc_attn = o->attn_in_actB ? 0 : attn_work + 256;
  int sc_gemv = 8 * 512 + 1024 * 4 + 64;
  int sc_topk = (64 + 64 + kRouteMaskWords + 1) * 4;              // selections, weights, masks
  int sc_rn = (kMaxBatch * 64 + kRnStage) * 4 + 64;
  int sc_comb = 256 * 16 + kMaxAttnOut * 4 + 3 * max_chunks * G * 4 + 2 * G * 4 + 256;
  int sc = std::max(std::max(sc_attn, sc_gemv), std::max(std::max(sc_topk, sc_rn), sc_comb));
  o->scratch_bytes = round_up(sc, 1024);
  const int fifo = kFifo * kFifoEntryWords * 4;
  const int max_stages = 14;
  const int bars = round_up((2 * max_stages + 4 * kFifo + 12) * 8, 1024);
  o->part_cols = B <= 2 ? B : 8;
  const int epi = round_up(2 * kConsumerWarps * 16 * o->part_cols * 4 + kRstdRing * kMaxBatch * 4,
                           128);
  const int budget = 232448 - 1040;   // max per block, less the alignment pad and static smem
  const int ptrs = round_up(ptr_table_words(s.L) * 8, 128);
  // the routing table copy, plus the producer's own routing scratch when it
  // computes the table itself (B <= kLocalRouteMaxB)
  const int rcache = round_up((route_words(B, s.k, std::min(s.E, B * s.k)) +
                               (B <= kLocalRouteMaxB ? kRouteTmpWords : 0)) * 4, 128);
  int rest1 = bars + fifo + epi + ptrs + rcache + o->scratch_bytes + o->actA_stride +
              2 * o->actB_bytes;
  int rest2 = rest1 + o->actA_stride;
  int nA = ((budget - rest2) / kStageBytes >= 8) ? 2 : 1;
  int rest = nA == 2 ? rest2 : rest1;
  int ns = std::min(max_stages, (budget - rest) / kStageBytes);
  if (ns < 2) return MK_ERR_CAPACITY;
  o->nA = nA;
  o->n_stages = ns;
  o->off_ring = 0;
  o->off_bars = ns * kStageBytes;
  o->off_fifo = o->off_bars + bars;
  o->off_scratch = o->off_fifo + fifo;
  o->off_actA = o->off_scratch + o->scratch_bytes;
  o->off_actB = o->off_actA + nA * o->actA_stride;
  o->off_epi = o->off_actB + 2 * o->actB_bytes;
  o->off_ptrs = o->off_epi + epi;
  o->off_rcache = o->off_ptrs + ptrs;
  o->total = o->off_rcache + rcache;
  o->dyn_bytes = o->total + 1024;
  return MK_OK;
}

namespace {


struct Task {
  int32_t w[kDescWords];
};

struct Layout {
  int L, B, S, Hkv, NR;
  int norm0, qkv0, rtr0, attp0, atto0, slot0, dt0, lmarr, lmdone, total;
  void build(int L_, int B_, int S_, int Hkv_, int NR_) {
    L = L_; B = B_; S = S_; Hkv = Hkv_; NR = NR_;
    int c = 0;
    norm0 = c; c += L + 1;
    qkv0 = c; c += L * Hkv;
    rtr0 = c; c += L;
    attp0 = c; c += L * B * Hkv;
    atto0 = c; c += L * Hkv;
    slot0 = c; c += L * S;
    dt0 = c; c += L * NR;
    lmarr = c; c += 1;
    lmdone = c; c += 1;
    total = c;
  }
  int norm(int l) const { return norm0 + l; }
  int qkv(int l, int g) const { return qkv0 + l * Hkv + g; }
  int rtr(int l) const { return rtr0 + l; }
  int attp(int l, int b, int g) const { return attp0 + (l * B + b) * Hkv + g; }
  int atto(int l, int g) const { return atto0 + l * Hkv + g; }
  int slot(int l, int j) const { return slot0 + l * S + j; }
  int dt(int l, int r) const { return dt0 + l * NR + r; }
};

Task make_task(int op, int layer, int phase) {
  Task t;
  std::memset(t.w, 0, sizeof(t.w));
  t.w[D_OP] = op;
  t.w[D_LAYER] = layer;
  t.w[D_PW] = -1;
  t.w[D_PWN] = 0;
  t.w[D_W0] = -1;
  t.w[D_W1] = -1;
  t.w[D_S0] = -1;
  t.w[D_S1] = -1;
  t.w[D_MAP0] = -1;
  t.w[D_MAP1] = -1;
  t.w[D_PHASE] = phase;
  t.w[D_ACT] = ACT_NONE;
  return t;
}

void add_wait(Task& t, int ctr, int n) {
  int i = t.w[D_NWAIT]++;
  t.w[D_W0 + 2 * i] = ctr;
  t.w[D_W0N + 2 * i] = n;
}
void add_signal(Task& t, int ctr) {
  int i = t.w[D_NSIG]++;
  t.w[D_S0 + i] = ctr;
}


}  // namespace

int plan_schedule(const Shape& s, int n_ctas, int B, const int32_t* seq_lens,
                  const int32_t* plan_len, bool with_phases, Plan* out) {
  if (!out || n_ctas < 1 || B < 1 || B > s.max_batch || B > kMaxBatch) return MK_ERR_INVALID;
  if (!seq_lens) return MK_ERR_INVALID;
  const int L = s.L, d = s.d, hd = s.hd, Hq = s.Hq, Hkv = s.Hkv, E = s.E, k = s.k, F = s.F;
  const int G = Hq / Hkv;
  const int NR = d / 64;
  const int S = std::min(E, B * k);
  const int qkvR = (Hq + 2 * Hkv) * hd;
  const int r_qkv = gemv_rows_for(d, 1);
  const int r_ff = gemv_rows_for(d, 2);
  const int n_qkv = qkvR / r_qkv;
  const int n_ff = F / r_ff;
  const int n_lm = (s.V + 127) / 128;
  if (r_qkv > hd || hd % r_qkv != 0) return MK_ERR_INVALID;

  // ---- attention chunk plan: whole pages, chunks sized so that the step's
  // KV stream spreads over all CTAs.
  int cap_pages[kMaxBatch];
  long total_pages = 0;
  for (int b = 0; b < B; ++b) {
    if (seq_lens[b] < 0) return MK_ERR_INVALID;
    long pl = plan_len ? (long)plan_len[b] : (long)seq_lens[b] + kPage;
    if (pl < seq_lens[b]) return MK_ERR_INVALID;
    cap_pages[b] = (int)((pl + kPage - 1) / kPage);
    total_pages += (long)cap_pages[b] * Hkv;
  }
  long ppc_all = std::max(1L, (total_pages + n_ctas - 1) / n_ctas);
  int max_chunks = 1;
  for (int b = 0; b < B; ++b) {
    out->ppc[b] = (int)ppc_all;
    out->nc[b] = std::max(1, (int)((cap_pages[b] + ppc_all - 1) / ppc_all));
    max_chunks = std::max(max_chunks, out->nc[b]);
  }

  Layout lay;
  lay.build(L, B, S, Hkv, NR);
  std::vector<int32_t> targets(lay.total, 0);


  std::vector<Task> tasks;
  tasks.reserve((size_t)L * (NR + n_qkv + 1 + 2 * B * Hkv * max_chunks + NR * Hkv +
                             S * (n_ff + NR)) + NR + n_lm + 16);
  const int PH = 8;  // phases per layer
  auto map_of = [&](int l, int which) { return l * kMapsPerLayer + which; };

  // a task that also performs the join it completes: it arrives on
  // arrive_ctr, and the last of `arrivals` arrivals runs the joined work and
  // signals join_ctr
  auto fuse = [&](Task& t, int flag, int arrive_ctr, int arrivals, int join_ctr) {
    t.w[D_FLAGS] |= flag;
    t.w[D_X0] = arrive_ctr;
    t.w[D_X1] = arrivals;
    t.w[D_X2] = join_ctr;
    targets[arrive_ctr] += 1;
  };
  // residual add + RMSNorm tiles producing level l; a tile of a level that
  // feeds a layer also computes its 64 columns' share of that layer's router
  // logits (W_r[:, tile] . gamma x), its router columns streamed through the
  // ring like GEMV weights: one stage per 128 experts
  auto emit_norm = [&](int l) {
    for (int r = 0; r < NR; ++r) {
      Task t = make_task(OP_RN, l, l * PH + 0);
      t.w[D_A] = r;
      if (l < L) {
        t.w[D_NSTAGE] = (E + kRouterRowsPerStage - 1) / kRouterRowsPerStage;
        t.w[D_MAP0] = map_of(l, kMapRouter);
      }
      if (l > 0) add_wait(t, lay.dt(l - 1, r), Hkv + S);
      add_signal(t, lay.norm(l));
      targets[lay.norm(l)] += 1;
      tasks.push_back(t);
    }
  };
  // the producer of an expert tile needs the layer's routing: up to
  // kLocalRouteMaxB tokens it computes the table itself once the layer's norm
  // tiles are done; beyond that it waits for the layer's top-k task
  auto set_route_wait = [&](Task& t, int l) {
    if (B <= kLocalRouteMaxB) {
      t.w[D_PW] = lay.norm(l);
      t.w[D_PWN] = NR;
    } else {
      t.w[D_PW] = lay.rtr(l);
      t.w[D_PWN] = 1;
    }
  };
  emit_norm(0);
  for (int l = 0; l < L; ++l) {
    if (l > 0) emit_norm(l);
    // -- top-k over the router logits summed from the norm tiles' shares
    {
      Task t = make_task(OP_TOPK, l, l * PH + 2);
      add_wait(t, lay.norm(l), NR);
      add_signal(t, lay.rtr(l));
      tasks.push_back(t);
    }
    targets[lay.rtr(l)] += 1;   // one top-k per layer
    // -- QKV tiles (grouped by KV group so attention of a group starts early)
    for (int g = 0; g < Hkv; ++g) {
      auto emit_rows = [&](int row_begin, int rows) {
        for (int r0 = row_begin; r0 < row_begin + rows; r0 += r_qkv) {
          Task t = make_task(OP_QKV, l, l * PH + 1);
          t.w[D_A] = r0 / r_qkv;
          t.w[D_B] = g;
          t.w[D_ROW0] = r0;
          t.w[D_K0] = 0;
          t.w[D_KCH] = d / 64;
          t.w[D_R] = r_qkv;
          t.w[D_NMAT] = 1;
          t.w[D_MAP0] = map_of(l, 0);
          t.w[D_NSTAGE] = (r_qkv / 16) * (d / 64) / 8;
          add_wait(t, lay.norm(l), NR);
          add_signal(t, lay.qkv(l, g));
          targets[lay.qkv(l, g)] += 1;
          t.w[D_ACT] = ACT_A;
          tasks.push_back(t);
        }
      };
      emit_rows(g * G * hd, G * hd);            // q heads of the group
      emit_rows(Hq * hd + g * hd, hd);          // k head
      emit_rows((Hq + Hkv) * hd + g * hd, hd);  // v head
    }
    // -- attention chunks, then combines
    for (int g = 0; g < Hkv; ++g) {
      for (int b = 0; b < B; ++b) {
        int nc = out->nc[b];
        for (int c = 0; c < nc; ++c) {
          Task t = make_task(OP_ATTN, l, l * PH + 3);
          t.w[D_A] = b;
          t.w[D_B] = g;
          t.w[D_C] = c;
          t.w[D_D] = nc;
          t.w[D_PPC] = out->ppc[b];
          t.w[D_MAP0] = map_of(l, 6);
          t.w[D_MAP1] = map_of(l, 7);
          if (c == nc - 1) t.w[D_FLAGS] |= F_LAST_CHUNK;
          if (nc == 1) t.w[D_FLAGS] |= F_SINGLE;
          add_wait(t, lay.qkv(l, g), (G * hd + 2 * hd) / r_qkv);
          // the attention merge of (b, g) is done by the chunk whose arrival
          // completes the (b, g) count (an acquire-release arrival counter)
          if (nc == 1)
            add_signal(t, lay.atto(l, g));
          else
            fuse(t, F_COMBINE, lay.attp(l, b, g), nc, lay.atto(l, g));
          long p0 = (long)c * out->ppc[b];
          long pages_now = ((long)seq_lens[b] + kPage - 1) / kPage;
          long np = std::max(0L, std::min((long)out->ppc[b], pages_now - p0));
          t.w[D_ACT] = ACT_B;
          tasks.push_back(t);
        }
      }
    }
    for (int g = 0; g < Hkv; ++g) targets[lay.atto(l, g)] += B;   // one output per (b, g)
    // -- O-proj: (64-row tile, KV group)
    for (int g = 0; g < Hkv; ++g) {
      for (int r = 0; r < NR; ++r) {
        Task t = make_task(OP_OPROJ, l, l * PH + 5);
        t.w[D_A] = r;
        t.w[D_B] = g;
        t.w[D_ROW0] = r * 64;
        t.w[D_K0] = g * G * hd;
        t.w[D_KCH] = G * hd / 64;
        t.w[D_R] = 64;
        t.w[D_NMAT] = 1;
        t.w[D_MAP0] = map_of(l, 1);
        t.w[D_NSTAGE] = 4 * (G * hd / 64) / 8;
        add_wait(t, lay.atto(l, g), B);
        add_signal(t, lay.dt(l, r));
        targets[lay.dt(l, r)] += 1;
        t.w[D_ACT] = ACT_B;
        tasks.push_back(t);
      }
    }
    // -- experts: gate/up tiles per slot, then down tiles per slot
    for (int j = 0; j < S; ++j) {
      for (int f = 0; f < n_ff; ++f) {
        Task t = make_task(OP_GATEUP, l, l * PH + 6);
        t.w[D_A] = j;
        t.w[D_B] = f;
        t.w[D_ROW0] = f * r_ff;
        t.w[D_K0] = 0;
        t.w[D_KCH] = d / 64;
        t.w[D_R] = r_ff;
        t.w[D_NMAT] = 2;
        t.w[D_MAP0] = map_of(l, 3);
        t.w[D_MAP1] = map_of(l, 4);
        t.w[D_NSTAGE] = 2 * (r_ff / 16) * (d / 64) / 8;
        set_route_wait(t, l);
        add_wait(t, lay.norm(l), NR);
        add_signal(t, lay.slot(l, j));
        targets[lay.slot(l, j)] += 1;
        t.w[D_ACT] = ACT_A;
        tasks.push_back(t);
      }
    }
    for (int j = 0; j < S; ++j) {
      for (int r = 0; r < NR; ++r) {
        Task t = make_task(OP_DOWN, l, l * PH + 7);
        t.w[D_A] = j;
        t.w[D_B] = r;
        t.w[D_ROW0] = r * 64;
        t.w[D_K0] = 0;
        t.w[D_KCH] = F / 64;
        t.w[D_R] = 64;
        t.w[D_NMAT] = 1;
        t.w[D_MAP0] = map_of(l, 5);
        t.w[D_NSTAGE] = 4 * (F / 64) / 8;
        set_route_wait(t, l);
        add_wait(t, lay.slot(l, j), n_ff);
        add_signal(t, lay.dt(l, r));
        targets[lay.dt(l, r)] += 1;
        t.w[D_ACT] = ACT_B;
        tasks.push_back(t);
      }
    }
  }
  emit_norm(L);   // the final norm
  // -- LM head
  for (int t_i = 0; t_i < n_lm; ++t_i) {
    Task t = make_task(OP_LMHEAD, L, L * PH + 1);
    t.w[D_A] = t_i;
    t.w[D_ROW0] = t_i * 128;
    t.w[D_K0] = 0;
    t.w[D_KCH] = d / 64;
    t.w[D_R] = 128;
    t.w[D_NMAT] = 1;
    t.w[D_MAP0] = L * kMapsPerLayer;
    t.w[D_NSTAGE] = 8 * (d / 64) / 8;
    add_wait(t, lay.norm(L), NR);
    // the last LM-head tile to finish completes a greedy step's tokens
    fuse(t, F_ARGMAX, lay.lmarr, n_lm, lay.lmdone);
    t.w[D_ACT] = ACT_A;
    tasks.push_back(t);
  }
  targets[lay.lmdone] += 1;

  // ---- priority order: stable sort by (layer, operation rank)
  static const int kRank[OP_COUNT] = {
      /*NONE*/ 99, /*RN*/ 0, /*QKV*/ 2, /*ROUTER*/ 1, /*TOPK*/ 3, /*ATTN*/ 4,
      /*COMBINE*/ 6, /*OPROJ*/ 7, /*GATEUP*/ 5, /*DOWN*/ 8, /*LMHEAD*/ 9};
  std::stable_sort(tasks.begin(), tasks.end(), [](const Task& x, const Task& y) {
    if (x.w[D_LAYER] != y.w[D_LAYER]) return x.w[D_LAYER] < y.w[D_LAYER];
    return kRank[x.w[D_OP]] < kRank[y.w[D_OP]];
  });
  // expert tiles: D_C = the list index one past the layer's last tile of the
  // same operation.  Slots are filled in ascending order at run time and the
  // tiles are slot-major, so once a producer meets a tile of an unused slot
  // every later tile up to that index is unused too and the dispenser jumps
  // there.
  for (size_t i = 0; i < tasks.size();) {
    const int op = tasks[i].w[D_OP];
    size_t j = i + 1;
    if (op == OP_GATEUP || op == OP_DOWN) {
      while (j < tasks.size() && tasks[j].w[D_OP] == op &&
             tasks[j].w[D_LAYER] == tasks[i].w[D_LAYER])
        ++j;
      for (size_t q = i; q < j; ++q) tasks[q].w[D_C] = (int)j;
    }
    i = j;
  }
  // A-slot double buffering where two buffers fit in shared memory
  SmemLayout sl;
  int slrc = smem_layout(s, B, max_chunks, &sl);
  if (slrc != MK_OK) return slrc;

  const int n_tasks = (int)tasks.size();
  const int n_phases = L * PH + 2;
  // task dispensers: one for the fused list, one per phase list
  // (each launch starts them at 0 and its last producer out zeroes them)
  const int grab = lay.total;
  const int grab_phase0 = lay.total + 1;
  const int exit_ctr = lay.total + 1 + n_phases;
  const int n_counters = lay.total + 2 + n_phases;
  targets.resize(n_counters, 0);

  out->release();
  out->n_ctas = n_ctas;
  out->B = B;
  out->S = S;
  out->max_chunks = max_chunks;
  out->n_counters = n_counters;
  out->n_tasks = n_tasks;
  out->r_qkv = r_qkv;
  out->n_phases = n_phases;
  out->grab = grab;
  out->grab_phase0 = grab_phase0;
  out->exit_ctr = exit_ctr;
  out->slot_ctr0 = lay.slot0;
  out->dt_ctr0 = lay.dt0;
  out->n_ff = n_ff;
  out->desc = (int32_t*)std::malloc((size_t)n_tasks * kDescWords * sizeof(int32_t));
  out->targets = (int32_t*)std::calloc((size_t)n_counters, sizeof(int32_t));
  out->phase_desc = with_phases
                        ? (int32_t*)std::malloc((size_t)n_tasks * kDescWords * sizeof(int32_t))
                        : nullptr;
  out->phase_off = (int32_t*)std::calloc((size_t)n_phases + 1, sizeof(int32_t));
  if (!out->desc || !out->targets || !out->phase_off || (with_phases && !out->phase_desc)) {
    out->release();
    return MK_ERR_OOM;
  }
  for (int i = 0; i < n_tasks; ++i)
    std::memcpy(out->desc + (size_t)i * kDescWords, tasks[i].w, sizeof(int32_t) * kDescWords);
  // phase lists: the same tasks grouped by phase, each group in priority order
  std::vector<int> per_phase(n_phases, 0);
  for (const auto& t : tasks) per_phase[t.w[D_PHASE]]++;
  for (int ph = 0; ph < n_phases; ++ph) {
    out->phase_off[ph + 1] = out->phase_off[ph] + per_phase[ph];
  }
  if (with_phases) group_by_phase(*out, out->phase_desc);
  std::memcpy(out->targets, targets.data(), sizeof(int32_t) * n_counters);
  out->n_stages = sl.n_stages;
  out->attn_in_actB = sl.attn_in_actB;
  return MK_OK;
}

// The unfused launcher's lists: the plan's tasks grouped by phase (phase ph
// at [phase_off[ph], phase_off[ph + 1]) of `out`), each group in list order.
// An expert phase holds one layer's tiles of one operation, so their jump
// index (D_C) becomes the phase's own length.
void group_by_phase(const Plan& plan, int32_t* out) {
  std::vector<int> fill(plan.phase_off, plan.phase_off + plan.n_phases);
  for (int i = 0; i < plan.n_tasks; ++i) {
    const int32_t* w = plan.desc + (size_t)i * kDescWords;
    const int ph = w[D_PHASE];
    const int pos = fill[ph]++;
    int32_t* o = out + (size_t)pos * kDescWords;
    std::memcpy(o, w, sizeof(int32_t) * kDescWords);
    if (w[D_OP] == OP_GATEUP || w[D_OP] == OP_DOWN)
      o[D_C] = plan.phase_off[ph + 1] - plan.phase_off[ph];
  }
}

}  // namespace mk

extern "C" mk_status mk_plan_schedule(const mk_config* cfg, int n_ctas, int batch,
                                      const int32_t* seq_lens, const int32_t* plan_len,
                                      int32_t* meta, int32_t* desc, int32_t* targets) {
  if (!cfg || !meta) return MK_ERR_INVALID;
  mk::Shape s{cfg->n_layers, cfg->d_model, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim,
              cfg->n_experts, cfg->top_k, cfg->d_ff, cfg->vocab, cfg->page_size,
              cfg->max_batch, cfg->n_pages, cfg->rope_theta, cfg->rms_eps};
  int v = mk::validate_shape(s);
  if (v != MK_OK) return (mk_status)v;
  mk::Plan p;
  int rc = mk::plan_schedule(s, n_ctas, batch, seq_lens, plan_len, false, &p);
  if (rc != MK_OK) return (mk_status)rc;
  std::memset(meta, 0, 16 * sizeof(int32_t));
  meta[0] = p.n_tasks;
  meta[1] = p.n_counters;
  meta[2] = p.S;
  meta[3] = p.max_chunks;
  meta[4] = mk::kDescWords;
  meta[5] = p.n_phases;
  meta[6] = p.r_qkv;
  meta[7] = p.ppc[0];
  meta[8] = p.grab;
  meta[9] = p.grab_phase0;
  meta[10] = p.n_stages;
  meta[11] = p.attn_in_actB;
  if (desc) std::memcpy(desc, p.desc, sizeof(int32_t) * (size_t)p.n_tasks * mk::kDescWords);
  if (targets) std::memcpy(targets, p.targets, sizeof(int32_t) * p.n_counters);
  p.release();
  return MK_OK;
}
