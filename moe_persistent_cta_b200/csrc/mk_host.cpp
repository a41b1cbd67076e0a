// mk_host.cpp -- the C ABI: context creation (validation, TMA tensor maps,
// context-owned device memory), schedule upload, step launches, status.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "mk.h"
#include "mk_internal.h"

namespace mk {
cudaError_t launch_interp(const Params& p, int grid, cudaStream_t stream);
cudaError_t max_coresident(int smem_bytes, int* blocks_per_sm);
mk_status static_scratch_setup(int device);
}  // namespace mk

using mk::Params;
using mk::Plan;
using mk::Shape;
using mk::SmemLayout;

struct DevBuf {
  void* ptr = nullptr;
  size_t bytes = 0;
};

struct mk_ctx {
  int device = 0;
  int n_sms = 0;
  int clock_khz = 0;   // peak SM clock: converts wait deadlines to clock64 cycles
  mk_config cfg{};
  Shape shape{};
  int r_qkv = 16, r_ff = 16;
  // model pointers (device) kept from mk_create
  const void* embed = nullptr;
  const void* lm_head = nullptr;
  const void* final_norm = nullptr;
  // context-owned device memory
  void* d_tmaps = nullptr;
  void** d_attn_norm = nullptr;
  void** d_router_bias = nullptr;
  void** d_kpool = nullptr;
  void** d_vpool = nullptr;
  double* d_inv_freq = nullptr;
  int32_t* d_status = nullptr;
  uint32_t* d_counters = nullptr;
  int counters_cap = 0;
  DevBuf desc, phase_desc;
  bool phases_uploaded = false;
  DevBuf x, actA, qkv, cs, attn_part, attn_o, ofrag, o_part, rlogits, racc, ssacc, route, expert_a, afrag,
      moe_part, amax, trace;
  DevBuf selftest;   // one descriptor + two counters for mk_selftest_timeout
  bool tracing = false;
  // schedule
  bool have_schedule = false;
  Plan plan;
  SmemLayout sl{};
  int B = 0, S = 0, max_chunks = 1, max_pages = 0;

  uint32_t epoch = 0;
  unsigned long long timeout_ns = 2000ull * 1000ull * 1000ull;
  cudaStream_t last_stream = nullptr;
  bool launched = false;   // a step was launched on last_stream
  Params base{};
};

namespace {

mk_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MK_OK;
  if (e == cudaErrorMemoryAllocation) return MK_ERR_OOM;
  return MK_ERR_CUDA;
}

#define MK_TRY(expr)                        \
  do {                                      \
    mk_status _s = (expr);                  \
    if (_s != MK_OK) return _s;             \
  } while (0)
#define MK_CUDA(expr) MK_TRY(from_cuda(expr))

mk_status ensure(DevBuf& b, size_t bytes) {
  if (bytes == 0) bytes = 16;
  if (b.bytes >= bytes) return MK_OK;
  if (b.ptr) cudaFree(b.ptr);
  b.ptr = nullptr;
  b.bytes = 0;
  MK_CUDA(cudaMalloc(&b.ptr, bytes));
  b.bytes = bytes;
  return MK_OK;
}

void release(DevBuf& b) {
  if (b.ptr) cudaFree(b.ptr);
  b.ptr = nullptr;
  b.bytes = 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 3D bf16 view of a row-major [rows][K] matrix as {64 columns, rows, K/64
// column chunks} (strides K*2 and 128 bytes), box {64, box_rows, box_chunks},
// 128-byte swizzle: one copy lands box_chunks consecutive 2 KB-per-16-rows
// units ([chunk][row][128 B]), the layout the tile routines read, so a whole
// ring stage of one matrix is a single TMA instruction.
mk_status encode_3d(CUtensorMap* m, const void* ptr, uint64_t K, uint64_t rows,
                    uint32_t box_rows, uint32_t box_chunks) {
  auto fn = get_encoder();
  if (!fn) return MK_ERR_CUDA;
  cuuint64_t dims[3] = {64, rows, K / 64};
  cuuint64_t strides[2] = {K * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_chunks};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MK_OK : MK_ERR_INVALID;
}


int round_up(int x, int a) { return (x + a - 1) / a * a; }

// A wait limit in ns as SM clock cycles at the device's peak clock: at any
// lower clock the same cycle count takes longer, so the limit only grows.
unsigned long long deadline_cycles(const mk_ctx* c, unsigned long long ns) {
  return ns * (unsigned long long)c->clock_khz / 1000000ull;
}

}  // namespace

extern "C" {

const char* mk_strerror(mk_status s) {
  switch (s) {
    case MK_OK: return "ok";
    case MK_ERR_INVALID: return "invalid argument";
    case MK_ERR_CUDA: return "CUDA error";
    case MK_ERR_OOM: return "out of device memory";
    case MK_ERR_TIMEOUT: return "device wait exceeded its deadline";
    case MK_ERR_CAPACITY: return "request exceeds capacity";
    case MK_ERR_STATE: return "call out of order or schedule outgrown";
    case MK_ERR_DEVICE: return "device-side validation failed";
  }
  return "unknown status";
}

void mk_destroy(mk_ctx* c) {
  if (!c) return;
  cudaSetDevice(c->device);
  cudaDeviceSynchronize();
  cudaFree(c->d_tmaps);
  cudaFree(c->d_attn_norm);
  cudaFree(c->d_router_bias);
  cudaFree(c->d_kpool);
  cudaFree(c->d_vpool);
  cudaFree(c->d_inv_freq);
  cudaFree(c->d_status);
  cudaFree(c->d_counters);
  for (DevBuf* b : {&c->desc, &c->phase_desc, &c->x, &c->actA,
                    &c->qkv, &c->cs, &c->attn_part, &c->attn_o, &c->ofrag, &c->o_part,
                    &c->rlogits, &c->racc, &c->ssacc, &c->route, &c->expert_a, &c->afrag, &c->moe_part,
                    &c->amax, &c->trace, &c->selftest})
    release(*b);
  c->plan.release();
  delete c;
}

mk_status mk_create(const mk_config* cfg, const mk_tensors* t, int device, mk_ctx** out) {
  if (!out) return MK_ERR_INVALID;
  *out = nullptr;
  if (!cfg || !t) return MK_ERR_INVALID;
  Shape s{cfg->n_layers, cfg->d_model, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim,
          cfg->n_experts, cfg->top_k, cfg->d_ff, cfg->vocab, cfg->page_size,
          cfg->max_batch, cfg->n_pages, cfg->rope_theta, cfg->rms_eps};
  MK_TRY((mk_status)mk::validate_shape(s));
  const int L = s.L;
  if (!t->embed || !t->lm_head || !t->final_norm || !t->attn_norm || !t->w_qkv || !t->w_o ||
      !t->w_router || !t->w_gate || !t->w_up || !t->w_down || !t->k_pool || !t->v_pool)
    return MK_ERR_INVALID;
  for (int l = 0; l < L; ++l) {
    const void* ps[] = {t->attn_norm[l], t->w_qkv[l], t->w_o[l], t->w_router[l], t->w_gate[l],
                        t->w_up[l], t->w_down[l], t->k_pool[l], t->v_pool[l]};
    for (const void* p : ps)
      if (!p || !aligned16(p)) return MK_ERR_INVALID;
    if (t->router_bias && t->router_bias[l] && !aligned16(t->router_bias[l])) return MK_ERR_INVALID;
  }
  if (!aligned16(t->embed) || !aligned16(t->lm_head) || !aligned16(t->final_norm))
    return MK_ERR_INVALID;
  int ndev = 0;
  MK_CUDA(cudaGetDeviceCount(&ndev));
  if (device < 0 || device >= ndev) return MK_ERR_INVALID;
  MK_CUDA(cudaSetDevice(device));

  mk_ctx* c = new mk_ctx();
  c->device = device;
  c->cfg = *cfg;
  c->shape = s;
  c->r_qkv = mk::gemv_rows_for(s.d, 1);
  c->r_ff = mk::gemv_rows_for(s.d, 2);
  c->embed = t->embed;
  c->lm_head = t->lm_head;
  c->final_norm = t->final_norm;
  auto fail = [&](mk_status st) {
    mk_destroy(c);
    return st;
  };
  if (cudaDeviceGetAttribute(&c->n_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return fail(MK_ERR_CUDA);
  if (cudaDeviceGetAttribute(&c->clock_khz, cudaDevAttrClockRate, device) != cudaSuccess ||
      c->clock_khz <= 0)
    c->clock_khz = 2000000;   // not reported: assume 2 GHz

  // tensor maps
  const int nmaps = L * mk::kMapsPerLayer + 1;
  std::vector<CUtensorMap> maps(nmaps);
  std::memset(maps.data(), 0, sizeof(CUtensorMap) * nmaps);
  const int G = s.Hq / s.Hkv;
  const uint64_t qkvR = (uint64_t)(s.Hq + 2 * s.Hkv) * s.hd;
  for (int l = 0; l < L; ++l) {
    CUtensorMap* m = &maps[l * mk::kMapsPerLayer];
    mk_status st;
    // box chunks = the column chunks one 16 KB stage holds: 8 units of 16 rows
    // shared by the tile's matrices and row tiles
    const uint32_t ch_qkv = 128u / (uint32_t)c->r_qkv, ch_ff = 64u / (uint32_t)c->r_ff;
    if ((st = encode_3d(m + 0, t->w_qkv[l], s.d, qkvR, c->r_qkv, ch_qkv)) != MK_OK)
      return fail(st);
    if ((st = encode_3d(m + 1, t->w_o[l], (uint64_t)s.Hq * s.hd, s.d, 64, 2)) != MK_OK)
      return fail(st);
    // router: one 64-column chunk of up to 128 expert rows per copy
    if ((st = encode_3d(m + mk::kMapRouter, t->w_router[l], s.d, s.E,
                        (uint32_t)std::min(s.E, mk::kRouterRowsPerStage), 1)) != MK_OK)
      return fail(st);
    if ((st = encode_3d(m + 3, t->w_gate[l], s.d, (uint64_t)s.E * s.F, c->r_ff, ch_ff)) != MK_OK)
      return fail(st);
    if ((st = encode_3d(m + 4, t->w_up[l], s.d, (uint64_t)s.E * s.F, c->r_ff, ch_ff)) != MK_OK)
      return fail(st);
    if ((st = encode_3d(m + 5, t->w_down[l], s.F, (uint64_t)s.E * s.d, 64, 2)) != MK_OK)
      return fail(st);
    // K/V pools: one (page, head) block of 64 tokens x hd per copy
    const uint64_t kvrows = (uint64_t)s.n_pages * s.Hkv * mk::kPage;
    if ((st = encode_3d(m + 6, t->k_pool[l], s.hd, kvrows, 64, s.hd / 64)) != MK_OK)
      return fail(st);
    if ((st = encode_3d(m + 7, t->v_pool[l], s.hd, kvrows, 64, s.hd / 64)) != MK_OK)
      return fail(st);
  }
  {
    mk_status st = encode_3d(&maps[L * mk::kMapsPerLayer], t->lm_head, s.d, s.V, 128, 1);
    if (st != MK_OK) return fail(st);
  }
  (void)G;
  if (cudaMalloc(&c->d_tmaps, sizeof(CUtensorMap) * nmaps) != cudaSuccess) return fail(MK_ERR_OOM);
  if (cudaMemcpy(c->d_tmaps, maps.data(), sizeof(CUtensorMap) * nmaps, cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return fail(MK_ERR_CUDA);

  // per-layer pointer arrays
  std::vector<void*> an(L), rb(L, nullptr), kp(L), vp(L);
  for (int l = 0; l < L; ++l) {
    an[l] = const_cast<void*>(t->attn_norm[l]);
    if (t->router_bias) rb[l] = const_cast<float*>(t->router_bias[l]);
    kp[l] = t->k_pool[l];
    vp[l] = t->v_pool[l];
  }
  auto upload_ptrs = [&](void*** dst, std::vector<void*>& src) -> mk_status {
    MK_CUDA(cudaMalloc(reinterpret_cast<void**>(dst), sizeof(void*) * src.size()));
    MK_CUDA(cudaMemcpy(*dst, src.data(), sizeof(void*) * src.size(), cudaMemcpyHostToDevice));
    return MK_OK;
  };
  {
    mk_status st;
    if ((st = upload_ptrs(&c->d_attn_norm, an)) != MK_OK) return fail(st);
    if ((st = upload_ptrs(&c->d_router_bias, rb)) != MK_OK) return fail(st);
    if ((st = upload_ptrs(&c->d_kpool, kp)) != MK_OK) return fail(st);
    if ((st = upload_ptrs(&c->d_vpool, vp)) != MK_OK) return fail(st);
  }
  // RoPE inverse frequencies theta^(-2i/hd), computed in double
  std::vector<double> inv(s.hd / 2);
  for (int i = 0; i < s.hd / 2; ++i)
    inv[i] = std::pow((double)s.theta, -2.0 * (double)i / (double)s.hd);
  if (cudaMalloc(&c->d_inv_freq, sizeof(double) * inv.size()) != cudaSuccess)
    return fail(MK_ERR_OOM);
  if (cudaMemcpy(c->d_inv_freq, inv.data(), sizeof(double) * inv.size(), cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return fail(MK_ERR_CUDA);
  if (cudaMalloc(&c->d_status, sizeof(int32_t) * 16) != cudaSuccess) return fail(MK_ERR_OOM);
  if (cudaMemset(c->d_status, 0, sizeof(int32_t) * 16) != cudaSuccess) return fail(MK_ERR_CUDA);
  // The fixed scratch array of mk_decode_step_static is resolved (and so
  // loaded) here, not on that call's first use.  If it cannot be, the context
  // still serves every other entry point; mk_decode_step_static then fails.
  (void)mk::static_scratch_setup(device);
  const char* env = std::getenv("MK_TIMEOUT_MS");
  if (env) {
    long ms = std::atol(env);
    if (ms > 0) c->timeout_ns = (unsigned long long)ms * 1000000ull;
  }
  *out = c;
  return MK_OK;
}

mk_status mk_set_trace(mk_ctx* c, int32_t enable) {
  if (!c) return MK_ERR_INVALID;
  c->tracing = enable != 0;
  return MK_OK;
}

mk_status mk_set_timeout_ms(mk_ctx* c, int32_t ms) {
  if (!c || ms <= 0) return MK_ERR_INVALID;
  c->timeout_ns = (unsigned long long)ms * 1000000ull;
  return MK_OK;
}

mk_status mk_build_schedule(mk_ctx* c, int batch, const int32_t* seq_lens,
                            const int32_t* plan_len, int32_t max_pages_per_seq) {
  if (!c || !seq_lens) return MK_ERR_INVALID;
  const Shape& s = c->shape;
  if (batch < 1 || batch > s.max_batch) return MK_ERR_INVALID;
  if (max_pages_per_seq < 1) return MK_ERR_INVALID;
  for (int b = 0; b < batch; ++b) {
    if (seq_lens[b] < 0) return MK_ERR_INVALID;
    const long need = (long)seq_lens[b] / mk::kPage + 1;   // page of the new token
    if (need > max_pages_per_seq) return MK_ERR_INVALID;
    if (plan_len && plan_len[b] < seq_lens[b]) return MK_ERR_INVALID;
  }
  MK_CUDA(cudaSetDevice(c->device));
  MK_CUDA(cudaDeviceSynchronize());
  c->have_schedule = false;
  Plan plan;
  MK_TRY((mk_status)mk::plan_schedule(s, c->n_sms, batch, seq_lens, plan_len, false, &plan));
  SmemLayout sl;
  {
    int rc = mk::smem_layout(s, batch, plan.max_chunks, &sl);
    if (rc != MK_OK) {
      plan.release();
      return (mk_status)rc;
    }
  }
  int per_sm = 0;
  if (mk::max_coresident(sl.dyn_bytes, &per_sm) != cudaSuccess || per_sm < 1) {
    plan.release();
    return MK_ERR_CAPACITY;
  }
  const int B = batch, L = s.L, d = s.d, G = s.Hq / s.Hkv, NR = d / 64, S = plan.S;
  const int qkvR = (s.Hq + 2 * s.Hkv) * s.hd;
  const int part_stride = round_up(2 * G + G * s.hd, 4);
  const int actA_rows = 4 * (d + mk::kActPad) * B;
  const int actA_bytes = actA_rows + round_up(NR * B * 4, 16);
  const int ofrag_bytes = 4 * (G * s.hd + mk::kActPad) * B;
  const int afrag_bytes = 4 * (s.F + mk::kActPad) * B;
  const int rwords = mk::route_words(B, s.k, S);
  auto fail = [&](mk_status st) {
    plan.release();
    return st;
  };
  mk_status st;
#define ENSURE(buf, bytes) \
  if ((st = ensure(c->buf, (size_t)(bytes))) != MK_OK) return fail(st)
  ENSURE(x, (size_t)(L + 1) * B * d * 4);
  ENSURE(actA, (size_t)(L + 1) * actA_bytes);
  ENSURE(qkv, (size_t)L * B * qkvR * 4);
  ENSURE(cs, (size_t)B * s.hd * 4);
  ENSURE(attn_part, (size_t)L * B * s.Hkv * plan.max_chunks * part_stride * 4);
  ENSURE(attn_o, (size_t)L * B * s.Hq * s.hd * 4);
  ENSURE(ofrag, (size_t)L * s.Hkv * ofrag_bytes);
  ENSURE(o_part, (size_t)L * s.Hkv * B * d * 4);
  ENSURE(rlogits, (size_t)L * B * s.E * 4);
  ENSURE(racc, (size_t)2 * L * B * s.E * 8);
  ENSURE(ssacc, (size_t)2 * L * B * 8);
  ENSURE(route, (size_t)L * rwords * 4);
  ENSURE(expert_a, (size_t)L * S * B * s.F * 4);
  ENSURE(afrag, (size_t)L * S * afrag_bytes);
  ENSURE(moe_part, (size_t)L * s.k * B * d * 4);
  ENSURE(amax, (size_t)B * 8);
  ENSURE(desc, (size_t)plan.n_tasks * mk::kDescWords * 4);
#undef ENSURE
  if (plan.n_counters > c->counters_cap) {
    cudaFree(c->d_counters);
    c->d_counters = nullptr;
    c->counters_cap = 0;
    if (cudaMalloc(&c->d_counters, sizeof(uint32_t) * plan.n_counters) != cudaSuccess)
      return fail(MK_ERR_OOM);
    c->counters_cap = plan.n_counters;
  }
  if (cudaMemset(c->d_counters, 0, sizeof(uint32_t) * c->counters_cap) != cudaSuccess)
    return fail(MK_ERR_CUDA);
  if (cudaMemset(c->route.ptr, 0, c->route.bytes) != cudaSuccess) return fail(MK_ERR_CUDA);
  if (cudaMemset(c->amax.ptr, 0, c->amax.bytes) != cudaSuccess) return fail(MK_ERR_CUDA);
  if (cudaMemset(c->racc.ptr, 0, c->racc.bytes) != cudaSuccess) return fail(MK_ERR_CUDA);
  if (cudaMemset(c->ssacc.ptr, 0, c->ssacc.bytes) != cudaSuccess) return fail(MK_ERR_CUDA);
  if (cudaMemcpy(c->desc.ptr, plan.desc, (size_t)plan.n_tasks * mk::kDescWords * 4,
                 cudaMemcpyHostToDevice) != cudaSuccess)
    return fail(MK_ERR_CUDA);
  c->phases_uploaded = false;   // the unfused path builds its phase lists on first use

  Params& p = c->base;
  std::memset(&p, 0, sizeof(p));
  p.L = L; p.d = d; p.Hq = s.Hq; p.Hkv = s.Hkv; p.hd = s.hd; p.E = s.E; p.k = s.k; p.F = s.F;
  p.V = s.V; p.B = B; p.S = S; p.G = G; p.NR = NR; p.qkvR = qkvR;
  p.max_chunks = plan.max_chunks;
  p.max_pages = max_pages_per_seq;
  p.n_pages = s.n_pages;
  p.part_stride = part_stride;
  p.eps = s.eps;
  p.actA_bytes = actA_bytes;
  p.actA_rows_bytes = actA_rows;
  p.ofrag_bytes = ofrag_bytes;
  p.afrag_bytes = afrag_bytes;
  p.route_words = rwords;
  p.counters = c->d_counters;
  p.exit_ctr = plan.exit_ctr;
  p.slot_ctr0 = plan.slot_ctr0;
  p.dt_ctr0 = plan.dt_ctr0;
  p.n_ff = plan.n_ff;
  p.tmaps = c->d_tmaps;
  p.embed = static_cast<const uint16_t*>(c->embed);
  p.final_norm = static_cast<const uint16_t*>(c->final_norm);
  p.attn_norm = reinterpret_cast<const uint16_t* const*>(c->d_attn_norm);
  p.router_bias = reinterpret_cast<const float* const*>(c->d_router_bias);
  p.k_pool = reinterpret_cast<uint16_t* const*>(c->d_kpool);
  p.v_pool = reinterpret_cast<uint16_t* const*>(c->d_vpool);
  p.inv_freq = c->d_inv_freq;
  p.x = static_cast<float*>(c->x.ptr);
  p.actA = static_cast<uint8_t*>(c->actA.ptr);
  p.qkv = static_cast<float*>(c->qkv.ptr);
  p.cs = static_cast<float*>(c->cs.ptr);
  p.attn_part = static_cast<float*>(c->attn_part.ptr);
  p.attn_o = static_cast<float*>(c->attn_o.ptr);
  p.ofrag = static_cast<uint8_t*>(c->ofrag.ptr);
  p.o_part = static_cast<float*>(c->o_part.ptr);
  p.rlogits = static_cast<float*>(c->rlogits.ptr);
  p.racc = static_cast<unsigned long long*>(c->racc.ptr);
  p.ssacc = static_cast<unsigned long long*>(c->ssacc.ptr);
  p.route = static_cast<int32_t*>(c->route.ptr);
  p.expert_a = static_cast<float*>(c->expert_a.ptr);
  p.afrag = static_cast<uint8_t*>(c->afrag.ptr);
  p.moe_part = static_cast<float*>(c->moe_part.ptr);
  p.amax = static_cast<unsigned long long*>(c->amax.ptr);
  p.status = c->d_status;
  p.n_stages = sl.n_stages;
  p.nA = sl.nA;
  p.actA_stride = sl.actA_stride;
  p.off_bars = sl.off_bars;
  p.off_fifo = sl.off_fifo;
  p.off_scratch = sl.off_scratch;
  p.attn_in_actB = sl.attn_in_actB;
  p.off_actA = sl.off_actA;
  p.off_actB = sl.off_actB;
  p.actB_bytes = sl.actB_bytes;
  p.off_ring = sl.off_ring;
  p.off_epi = sl.off_epi;
  p.off_ptrs = sl.off_ptrs;
  p.off_rcache = sl.off_rcache;
  p.part_cols = sl.part_cols;
  p.smem_bytes = sl.dyn_bytes;

  c->plan.release();
  c->plan = plan;  // takes ownership of the host arrays
  c->sl = sl;
  c->B = B;
  c->S = S;
  c->max_chunks = plan.max_chunks;
  c->max_pages = max_pages_per_seq;
  c->epoch = 0;
  c->have_schedule = true;
  MK_CUDA(cudaDeviceSynchronize());
  return MK_OK;
}

// A greedy step's writable views of its inputs and its row of the token output.
struct Greedy {
  int32_t* tokens;
  int32_t* positions;
  int32_t* seq_lens;
  int32_t* out;
};

static mk_status launch_step(mk_ctx* c, const int32_t* tokens, const int32_t* positions,
                             const int32_t* page_table, const int32_t* seq_lens, float* logits,
                             void* stream, bool unfused, const Greedy* greedy = nullptr) {
  if (!c) return MK_ERR_INVALID;
  if (!c->have_schedule) return MK_ERR_STATE;
  if (!tokens || !positions || !page_table || !seq_lens || !logits) return MK_ERR_INVALID;
  MK_CUDA(cudaSetDevice(c->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Params p = c->base;
  p.tokens = tokens;
  p.positions = positions;
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.logits = logits;
  if (greedy) {
    p.g_tok = greedy->tokens;
    p.g_pos = greedy->positions;
    p.g_len = greedy->seq_lens;
    p.g_out = greedy->out;
  }
  p.timeout_cycles = deadline_cycles(c, c->timeout_ns);
  p.epoch = c->epoch + 1;
  cudaError_t e = cudaSuccess;
  p.n_ctas = c->plan.n_ctas;
  if (!unfused) {
    if (c->tracing) {
      const size_t tb = (size_t)c->plan.n_tasks * mk::kTraceWords * 4;
      MK_TRY(ensure(c->trace, tb));
      MK_CUDA(cudaMemsetAsync(c->trace.ptr, 0, tb, st));
      p.trace = static_cast<uint32_t*>(c->trace.ptr);
    }
    p.desc = static_cast<const int32_t*>(c->desc.ptr);
    p.n_tasks = c->plan.n_tasks;
    p.grab = c->plan.grab;
    e = mk::launch_interp(p, c->plan.n_ctas, st);
  } else {
    if (!c->phases_uploaded) {
      // the same tasks grouped by phase, each group in list order
      const size_t bytes = (size_t)c->plan.n_tasks * mk::kDescWords * 4;
      std::vector<int32_t> h((size_t)c->plan.n_tasks * mk::kDescWords);
      mk::group_by_phase(c->plan, h.data());
      MK_TRY(ensure(c->phase_desc, bytes));
      MK_CUDA(cudaMemcpy(c->phase_desc.ptr, h.data(), bytes, cudaMemcpyHostToDevice));
      c->phases_uploaded = true;
    }
    for (int ph = 0; ph < c->plan.n_phases && e == cudaSuccess; ++ph) {
      const int n = c->plan.phase_off[ph + 1] - c->plan.phase_off[ph];
      if (n == 0) continue;
      p.desc = static_cast<const int32_t*>(c->phase_desc.ptr) +
               (size_t)c->plan.phase_off[ph] * mk::kDescWords;
      p.n_tasks = n;
      p.grab = c->plan.grab_phase0 + ph;
      e = mk::launch_interp(p, c->plan.n_ctas, st);
    }
  }
  if (e != cudaSuccess) return from_cuda(e);
  c->epoch += 1;
  c->last_stream = st;
  c->launched = true;
  return MK_OK;
}

mk_status mk_decode_step(mk_ctx* c, const int32_t* tokens, const int32_t* positions,
                         const int32_t* page_table, const int32_t* seq_lens, float* logits,
                         void* stream) {
  return launch_step(c, tokens, positions, page_table, seq_lens, logits, stream, false);
}

mk_status mk_decode_step_unfused(mk_ctx* c, const int32_t* tokens, const int32_t* positions,
                                 const int32_t* page_table, const int32_t* seq_lens, float* logits,
                                 void* stream) {
  return launch_step(c, tokens, positions, page_table, seq_lens, logits, stream, true);
}

mk_status mk_decode_greedy(mk_ctx* c, int32_t n_steps, int32_t* tokens, int32_t* positions,
                           const int32_t* page_table, int32_t* seq_lens, float* logits,
                           int32_t* out_tokens, void* stream) {
  if (!c) return MK_ERR_INVALID;
  if (n_steps < 0 || (n_steps > 0 && !out_tokens)) return MK_ERR_INVALID;
  for (int32_t i = 0; i < n_steps; ++i) {
    const Greedy g{tokens, positions, seq_lens, out_tokens + (size_t)i * c->B};
    MK_TRY(launch_step(c, tokens, positions, page_table, seq_lens, logits, stream, false, &g));
  }
  return MK_OK;
}

mk_status mk_check(mk_ctx* c, int32_t* device_status, int32_t* detail) {
  if (!c) return MK_ERR_INVALID;
  MK_CUDA(cudaSetDevice(c->device));
  if (c->launched)
    MK_CUDA(cudaStreamSynchronize(c->last_stream));
  else
    MK_CUDA(cudaDeviceSynchronize());
  int32_t st[16];
  MK_CUDA(cudaMemcpy(st, c->d_status, sizeof(st), cudaMemcpyDeviceToHost));
  if (device_status) *device_status = st[mk::ST_CODE];
  if (detail)
    for (int i = 0; i < 8; ++i) detail[i] = st[i];
  if (st[mk::ST_CODE] != 0 || st[mk::ST_ABORT] != 0) {
    // a step that stopped part-way leaves counters short of their targets:
    // restart the epochs so the next step begins from a clean state
    MK_CUDA(cudaMemset(c->d_status, 0, sizeof(st)));
    if (c->d_counters)
      MK_CUDA(cudaMemset(c->d_counters, 0, sizeof(uint32_t) * c->counters_cap));
    if (c->amax.ptr) MK_CUDA(cudaMemset(c->amax.ptr, 0, c->amax.bytes));
    if (c->racc.ptr) MK_CUDA(cudaMemset(c->racc.ptr, 0, c->racc.bytes));
    if (c->ssacc.ptr) MK_CUDA(cudaMemset(c->ssacc.ptr, 0, c->ssacc.bytes));
    c->epoch = 0;
    return st[mk::ST_CODE] != 0 ? (mk_status)st[mk::ST_CODE] : MK_ERR_DEVICE;
  }
  return MK_OK;
}

size_t mk_debug_size(mk_ctx* c, int which) {
  if (!c || !c->have_schedule) return 0;
  const Shape& s = c->shape;
  const size_t L = s.L, B = c->B, S = c->S;
  switch (which) {
    case MK_BUF_X: return (L + 1) * B * s.d * 4;
    case MK_BUF_QKV: return L * B * (s.Hq + 2 * s.Hkv) * s.hd * 4;
    case MK_BUF_ATTN_O: return L * B * s.Hq * s.hd * 4;
    case MK_BUF_RLOGITS: return L * B * s.E * 4;
    case MK_BUF_TOPK: return 2 * L * B * s.k * 4;
    case MK_BUF_NSLOTS: return L * 4;
    case MK_BUF_EXPERT_A: return L * S * B * s.F * 4;
    case MK_BUF_MOE: return L * s.k * B * s.d * 4;
    case MK_BUF_OPART: return L * s.Hkv * B * s.d * 4;
    case MK_BUF_TRACE: return (size_t)c->plan.n_tasks * mk::kTraceWords * 4;
    case MK_BUF_PLAN: return (size_t)c->plan.n_tasks * mk::kDescWords * 4;
  }
  return 0;
}

mk_status mk_debug_read(mk_ctx* c, int which, void* dst, size_t bytes) {
  if (!c || !dst) return MK_ERR_INVALID;
  if (!c->have_schedule) return MK_ERR_STATE;
  const size_t need = mk_debug_size(c, which);
  if (need == 0 || bytes != need) return MK_ERR_INVALID;
  MK_CUDA(cudaSetDevice(c->device));
  MK_CUDA(cudaDeviceSynchronize());
  const Shape& s = c->shape;
  const int L = s.L, B = c->B, K = s.k, S = c->S;
  const void* src = nullptr;
  switch (which) {
    case MK_BUF_X: src = c->x.ptr; break;
    case MK_BUF_QKV: src = c->qkv.ptr; break;
    case MK_BUF_ATTN_O: src = c->attn_o.ptr; break;
    case MK_BUF_RLOGITS: src = c->rlogits.ptr; break;
    case MK_BUF_EXPERT_A: src = c->expert_a.ptr; break;
    case MK_BUF_MOE: src = c->moe_part.ptr; break;
    case MK_BUF_OPART: src = c->o_part.ptr; break;
    default: break;
  }
  if (which == MK_BUF_TRACE) {
    if (!c->trace.ptr) return MK_ERR_STATE;
    src = c->trace.ptr;
  }
  if (which == MK_BUF_PLAN) {
    std::memcpy(dst, c->plan.desc, sizeof(int32_t) * (size_t)c->plan.n_tasks * mk::kDescWords);
    return MK_OK;
  }
  if (src) {
    MK_CUDA(cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost));
    return MK_OK;
  }
  const int rw = mk::route_words(B, K, S);
  std::vector<int32_t> rt((size_t)L * rw);
  MK_CUDA(cudaMemcpy(rt.data(), c->route.ptr, rt.size() * 4, cudaMemcpyDeviceToHost));
  int32_t* o = static_cast<int32_t*>(dst);
  if (which == MK_BUF_NSLOTS) {
    for (int l = 0; l < L; ++l) o[l] = rt[(size_t)l * rw];
    return MK_OK;
  }
  // MK_BUF_TOPK: ids [L][B][k] then weights [L][B][k]
  for (int l = 0; l < L; ++l)
    for (int i = 0; i < B * K; ++i) {
      o[(size_t)l * B * K + i] = rt[(size_t)l * rw + mk::route_topk_idx(B, K) + i];
      o[(size_t)L * B * K + (size_t)l * B * K + i] = rt[(size_t)l * rw + mk::route_topk_w(B, K) + i];
    }
  return MK_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Step with caller-supplied scratch (used by the fixed-array entry point).
namespace mk {

int ctx_device(const mk_ctx* c) { return c ? c->device : -1; }

namespace {
// Carves the per-step buffers of the current schedule out of one region, in
// a fixed order, each start rounded up to 256 bytes.  Returns the bytes used.
size_t carve_scratch(const Params& b, int n_counters, uint8_t* base, Params* p) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* q = base ? base + off : nullptr;
    off += (bytes + 255) & ~size_t(255);
    return q;
  };
  const size_t L = b.L, B = b.B, d = b.d;
  uint8_t* counters = take(sizeof(uint32_t) * (size_t)n_counters);
  uint8_t* route = take((size_t)L * b.route_words * 4);
  uint8_t* racc = take((size_t)2 * L * B * b.E * 8);
  uint8_t* ssacc = take((size_t)2 * L * B * 8);
  uint8_t* x = take((L + 1) * B * d * 4);
  uint8_t* actA = take((L + 1) * (size_t)b.actA_bytes);
  uint8_t* qkv = take(L * B * b.qkvR * 4);
  uint8_t* cs = take(B * b.hd * 4);
  uint8_t* attn_part = take(L * B * b.Hkv * b.max_chunks * b.part_stride * 4);
  uint8_t* attn_o = take(L * B * b.Hq * b.hd * 4);
  uint8_t* ofrag = take(L * b.Hkv * (size_t)b.ofrag_bytes);
  uint8_t* o_part = take(L * b.Hkv * B * d * 4);
  uint8_t* rlogits = take(L * B * b.E * 4);
  uint8_t* expert_a = take(L * b.S * B * b.F * 4);
  uint8_t* afrag = take(L * b.S * (size_t)b.afrag_bytes);
  uint8_t* moe_part = take(L * b.k * B * d * 4);
  if (p) {
    p->counters = reinterpret_cast<uint32_t*>(counters);
    p->route = reinterpret_cast<int32_t*>(route);
    p->x = reinterpret_cast<float*>(x);
    p->actA = actA;
    p->qkv = reinterpret_cast<float*>(qkv);
    p->cs = reinterpret_cast<float*>(cs);
    p->attn_part = reinterpret_cast<float*>(attn_part);
    p->attn_o = reinterpret_cast<float*>(attn_o);
    p->ofrag = ofrag;
    p->o_part = reinterpret_cast<float*>(o_part);
    p->rlogits = reinterpret_cast<float*>(rlogits);
    p->racc = reinterpret_cast<unsigned long long*>(racc);
    p->ssacc = reinterpret_cast<unsigned long long*>(ssacc);
    p->expert_a = reinterpret_cast<float*>(expert_a);
    p->afrag = afrag;
    p->moe_part = reinterpret_cast<float*>(moe_part);
  }
  return off;
}
}  // namespace

// One fused step whose per-step buffers and counters live in `scratch`
// (device memory of `cap` bytes) instead of the context's own.  Clears the
// counters and routing words on the stream first, then runs at epoch 1.
// The context's buffers, epoch and trace are left untouched.
mk_status launch_step_in(mk_ctx* c, const int32_t* tokens, const int32_t* positions,
                         const int32_t* page_table, const int32_t* seq_lens, float* logits,
                         void* stream, void* scratch, size_t cap) {
  if (!c) return MK_ERR_INVALID;
  if (!c->have_schedule) return MK_ERR_STATE;
  if (!tokens || !positions || !page_table || !seq_lens || !logits || !scratch)
    return MK_ERR_INVALID;
  const size_t need = carve_scratch(c->base, c->plan.n_counters, nullptr, nullptr);
  if (need > cap) return MK_ERR_CAPACITY;
  MK_CUDA(cudaSetDevice(c->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Params p = c->base;
  carve_scratch(c->base, c->plan.n_counters, static_cast<uint8_t*>(scratch), &p);
  const size_t zero_bytes = reinterpret_cast<uint8_t*>(p.x) - static_cast<uint8_t*>(scratch);
  // counters, routing words and the router accumulators start at zero
  MK_CUDA(cudaMemsetAsync(scratch, 0, zero_bytes, st));
  c->last_stream = st;
  c->launched = true;
  p.tokens = tokens;
  p.positions = positions;
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.logits = logits;
  p.timeout_cycles = deadline_cycles(c, c->timeout_ns);
  p.epoch = 1;
  p.trace = nullptr;
  p.g_tok = p.g_pos = p.g_len = p.g_out = nullptr;
  p.n_ctas = c->plan.n_ctas;
  p.desc = static_cast<const int32_t*>(c->desc.ptr);
  p.n_tasks = c->plan.n_tasks;
  p.grab = c->plan.grab;
  return from_cuda(mk::launch_interp(p, c->plan.n_ctas, st));
}

}  // namespace mk

// ---------------------------------------------------------------------------
// Failure-detection self-test: a one-task list whose only wait is on a
// counter nothing signals, run with a short deadline.  The bounded wait runs
// out by design; the kernel latches MK_ERR_TIMEOUT, every CTA leaves its task
// loop, and the status is read back and cleared here.  The step's own
// counters and epoch are not touched.
mk_status mk_selftest_timeout(mk_ctx* c, int32_t timeout_ms, int32_t* device_status,
                              int32_t* detail) {
  if (!c || timeout_ms <= 0) return MK_ERR_INVALID;
  if (!c->have_schedule) return MK_ERR_STATE;
  MK_CUDA(cudaSetDevice(c->device));
  const size_t bytes = sizeof(int32_t) * (mk::kDescWords + 4);
  MK_TRY(ensure(c->selftest, bytes));
  int32_t h[mk::kDescWords + 4];
  std::memset(h, 0, sizeof(h));
  h[mk::D_OP] = mk::OP_RN;       // never runs: its wait cannot be met
  h[mk::D_LAYER] = 0;
  h[mk::D_NWAIT] = 1;
  h[mk::D_W0] = 0;               // self-test counter 0: nothing signals it
  h[mk::D_W0N] = 1;
  h[mk::D_W1] = -1;
  h[mk::D_PW] = -1;
  h[mk::D_S0] = -1;
  h[mk::D_S1] = -1;
  h[mk::D_MAP0] = -1;
  h[mk::D_MAP1] = -1;
  h[mk::D_ACT] = mk::ACT_NONE;
  // words kDescWords.. : counter 0 (never signalled), counter 1 (dispenser),
  // counter 2 (producers' exit count)
  MK_CUDA(cudaMemcpy(c->selftest.ptr, h, bytes, cudaMemcpyHostToDevice));
  MK_CUDA(cudaMemset(c->d_status, 0, sizeof(int32_t) * 16));
  Params p = c->base;
  p.desc = static_cast<const int32_t*>(c->selftest.ptr);
  p.counters = reinterpret_cast<uint32_t*>(static_cast<int32_t*>(c->selftest.ptr) + mk::kDescWords);
  p.n_tasks = 1;
  p.grab = 1;
  p.exit_ctr = 2;
  p.n_ctas = c->plan.n_ctas;
  p.epoch = 1;
  p.trace = nullptr;
  p.timeout_cycles = deadline_cycles(c, (unsigned long long)timeout_ms * 1000000ull);
  // step inputs are never read (the task does not run); any device address
  int32_t* d0 = static_cast<int32_t*>(c->selftest.ptr);
  p.tokens = d0;
  p.positions = d0;
  p.page_table = d0;
  p.seq_lens = d0;
  p.logits = reinterpret_cast<float*>(c->x.ptr);
  MK_CUDA(mk::launch_interp(p, c->plan.n_ctas, nullptr));
  MK_CUDA(cudaDeviceSynchronize());
  int32_t st[16];
  MK_CUDA(cudaMemcpy(st, c->d_status, sizeof(st), cudaMemcpyDeviceToHost));
  MK_CUDA(cudaMemset(c->d_status, 0, sizeof(st)));
  if (device_status) *device_status = st[mk::ST_CODE];
  if (detail)
    for (int i = 0; i < 8; ++i) detail[i] = st[i];
  return st[mk::ST_CODE] != 0 ? (mk_status)st[mk::ST_CODE] : MK_OK;
}
