// mk_kernel.cu -- the persistent decode interpreter for sm_100a.
//
// One CTA per SM stays resident for the whole decode step and walks its own
// list of task descriptors (agenticcommons.xyz, "Cohere North Mini Code
// megakernel serving engine", section "How the megakernel works").  Warp roles
// inside a CTA:
//   warp 0 (producer)  resolves each task (routing table for expert tiles,
//                      page table for attention chunks) and streams its
//                      immutable weight / KV tiles into a ring of 16 KB shared
//                      memory stages with TMA, BEFORE the task's activation
//                      dependency is known to be satisfied (section "Three
//                      sources of speedup", item 3).  The ring's stage/phase
//                      runs on across task boundaries, so consecutive tiles
//                      never drain and refill the pipeline (section "Building
//                      on Hazy Research": phase continuation across tiles and
//                      weight loads issued before the cross-SM wait).
//   warp 1 (loader)    spins on the task's global counters (bounded by a
//                      deadline) and then bulk-copies the task's activation
//                      vector into shared memory.
//   warp 2 (signaler)  after the consumers finish a task, publishes it with a
//                      release add on each of the task's counters.
//   warp 3 (epilogue)  reduces the consumer warps' GEMV partial sums and
//                      writes the tile's outputs.
//   warps 4..11        compute: exact fp32 FMAs for one or two token columns,
//                      else mma.sync bf16 tiles (weights as the 16-row A
//                      operand read from the swizzled TMA tile with ldmatrix,
//                      fp32 activations as the 8-column B operand split into
//                      three bf16 terms, so the product keeps ~24 bits),
//                      attention with an online softmax, norm and top-k.
// Warpgroup 0 (warps 0..3) gives registers to the two consumer warpgroups
// (setmaxnreg: 80 and 208 per thread, from the 168 the launch holds).  Every
// routine is inlined into the kernel so that ptxas budgets each warpgroup's
// code on its own: an out-of-line function is compiled for the launch's 168
// and holds every caller to it.
// Every wait is bounded by a deadline counted in SM clock cycles (clock64; the
// host converts the millisecond limit at the device's peak SM clock); on expiry
// the CTA latches an error in the status word, raises the abort flag and
// unwinds, waiting for its own copies in flight before it exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "mk.h"
#include "mk_internal.h"

namespace mk {
namespace {

constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------- PTX -----
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// %globaltimer is slow to read: used for trace stamps only.  Deadlines of
// the wait loops count SM clock cycles (clock64), which is cheap.
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// L2 policy for streamed tensors (weights, cached K/V): evict first, so the
// once-per-step stream does not push code, activations and counters out of L2.
// 3D tiled copy {x, y, z} (the weight and KV views are {64 columns, rows,
// 64-column chunks}).
__device__ __forceinline__ void tma_3d(uint32_t dst, const void* map, int x, int y, int z,
                                       uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// Same test, but a thread whose phase is not complete is suspended (up to
// the hint, in ns) until it completes instead of returning at once, so
// waiting warps do not take issue slots from the math warps.
__device__ __forceinline__ bool mbar_wait_hint(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* a, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "l"(a), "r"(v)
               : "memory");
  return old;
}
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// The router's logit shares and the sums of squares are accumulated across
// the norm tiles as 64-bit fixed-point integers in units of 2^-32: integer
// addition is associative, so a sum does not depend on the order in which
// the tiles arrive (the step stays bit-reproducible), and one load of the
// accumulator replaces a load per tile.
__device__ __forceinline__ unsigned long long to_fixed(float x) {
  return (unsigned long long)__float2ll_rn(x * 4294967296.0f);
}
__device__ __forceinline__ float from_fixed(unsigned long long v) {
  return (float)((double)(long long)v * 2.3283064365386963e-10);
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma1688(float* c, uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
// Named barriers among the 8 consumer warps only: barrier 1 inside tile
// routines, barrier 2 for the consumers' agreement on leaving the task loop
// (every exit and every task with internal barriers passes through it, so
// all consumer warps execute the same sequence of barrier-1 waits).
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ int cbar_or(int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 2, 256, p;\n\tselp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred)
      : "memory");
  return r;
}

// Approximate PTX math (each within ~2^-22 relative): short instruction
// sequences keep the interpreter's code, and so its instruction-cache
// footprint, small.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fexp(float x) { return ex2(x * 1.4426950408889634f); }
__device__ __forceinline__ float frcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float frsqrt(float x) {
  float y;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16 helpers
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16r(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
// Split a pair of fp32 values into three bf16x2 terms hi + mid + lo that sum
// to the pair within 2^-27 relative (each difference is exact in fp32).
__device__ __forceinline__ void split3(float a, float b, uint32_t& h, uint32_t& m, uint32_t& l) {
  __nv_bfloat162 hh = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(hh);
  const float ra = a - hf.x, rb = b - hf.y;
  __nv_bfloat162 mm = __floats2bfloat162_rn(ra, rb);
  const float2 mf = __bfloat1622float2(mm);
  __nv_bfloat162 ll = __floats2bfloat162_rn(ra - mf.x, rb - mf.y);
  h = *reinterpret_cast<uint32_t*>(&hh);
  m = *reinterpret_cast<uint32_t*>(&mm);
  l = *reinterpret_cast<uint32_t*>(&ll);
}

// Two fp32 FMAs in one instruction (sm_100 packed fp32): (c0, c1) +=
// (a0 * b0, a1 * b1), each rounded as fma.rn.f32.
__device__ __forceinline__ void ffma2(float& c0, float& c1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 pa, pb, pc;\n\t"
      "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\tmov.b64 pc, {%0, %1};\n\t"
      "fma.rn.f32x2 pc, pa, pb, pc;\n\tmov.b64 {%0, %1}, pc;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// -------------------------------------------------------------- state -----
extern __shared__ uint8_t g_smem[];
__shared__ int g_abort;   // this CTA's abort flag

// View of the CTA's shared-memory carve-out, rebuilt from the launch
// parameters inside each role function so that it lives in registers.
struct Smem {
  uint8_t* ring;
  uint8_t* scratch;
  uint8_t* actA;
  uint8_t* actB;
  uint8_t* epi;
  const void* const* ptrs;   // per-layer pointer table
  int32_t* fifo;
  int32_t* rcache;           // the producer's copy of one layer's routing table
  uint32_t bars;  // shared-window address of barrier 0
  int NS;
  __device__ uint32_t bar(int i) const { return bars + 8u * (uint32_t)i; }
  __device__ uint32_t full(int s) const { return bar(s); }
  __device__ uint32_t empty(int s) const { return bar(NS + s); }
  __device__ uint32_t ready(int e) const { return bar(2 * NS + e); }
  __device__ uint32_t done(int e) const { return bar(2 * NS + kFifo + e); }
  __device__ uint32_t fempty(int e) const { return bar(2 * NS + 2 * kFifo + e); }
  __device__ uint32_t posted(int e) const { return bar(2 * NS + 3 * kFifo + e); }
  __device__ uint32_t afullA(int i) const { return bar(2 * NS + 4 * kFifo + i); }
  __device__ uint32_t aemptyA(int i) const { return bar(2 * NS + 4 * kFifo + 2 + i); }
  __device__ uint32_t afullB(int i) const { return bar(2 * NS + 4 * kFifo + 4 + i); }
  __device__ uint32_t aemptyB(int i) const { return bar(2 * NS + 4 * kFifo + 6 + i); }
  __device__ uint32_t pfull(int i) const { return bar(2 * NS + 4 * kFifo + 8 + i); }
  __device__ uint32_t pempty(int i) const { return bar(2 * NS + 4 * kFifo + 10 + i); }
};

// Entries of the shared-memory pointer table.
__device__ __forceinline__ const uint16_t* norm_w(const Smem& sm, int lv) {
  return static_cast<const uint16_t*>(sm.ptrs[lv]);   // lv == L: the final norm
}
__device__ __forceinline__ const float* router_b(const Params& p, const Smem& sm, int l) {
  return static_cast<const float*>(sm.ptrs[p.L + 1 + l]);
}
__device__ __forceinline__ uint16_t* kpool_of(const Params& p, const Smem& sm, int l) {
  return static_cast<uint16_t*>(const_cast<void*>(sm.ptrs[2 * p.L + 1 + l]));
}
__device__ __forceinline__ uint16_t* vpool_of(const Params& p, const Smem& sm, int l) {
  return static_cast<uint16_t*>(const_cast<void*>(sm.ptrs[3 * p.L + 1 + l]));
}

__device__ __forceinline__ Smem smem_view(const Params& p) {
  Smem s;
  const uint32_t raw = saddr(g_smem);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* base = g_smem + pad;
  s.ring = base + p.off_ring;
  s.scratch = base + p.off_scratch;
  s.actA = base + p.off_actA;
  s.actB = base + p.off_actB;
  s.epi = base + p.off_epi;
  s.ptrs = reinterpret_cast<const void* const*>(base + p.off_ptrs);
  s.fifo = reinterpret_cast<int32_t*>(base + p.off_fifo);
  s.rcache = reinterpret_cast<int32_t*>(base + p.off_rcache);
  s.bars = raw + pad + (uint32_t)p.off_bars;
  s.NS = p.n_stages;
  return s;
}

__device__ __forceinline__ bool aborted() { return *(volatile int*)&g_abort != 0; }
__device__ __forceinline__ void set_abort() { *(volatile int*)&g_abort = 1; }

__device__ __forceinline__ void raise_error(const Params& p, int code, int task, int op, int ctr, uint32_t obs,
                            uint32_t tgt, int aux) {
  if (atomicCAS(&p.status[ST_CODE], 0, code) == 0) {
    p.status[ST_CTA] = blockIdx.x;
    p.status[ST_TASK] = task;
    p.status[ST_OP] = op;
    p.status[ST_COUNTER] = ctr;
    p.status[ST_OBSERVED] = (int)obs;
    p.status[ST_TARGET] = (int)tgt;
    p.status[ST_AUX] = aux;
  }
  __threadfence();
  atomicExch(&p.status[ST_ABORT], 1);
}

// Bounded spin on a global counter (one lane).
__device__ __forceinline__ bool wait_counter_slow(const Params& p, int ctr, uint32_t target,
                                               int task, int op) {
  const uint32_t* c = p.counters + ctr;
  uint32_t v;
  const uint64_t t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    v = ld_acquire(c);
    if (reached(v, target)) return true;
    if ((it & 7u) == 0) {
      if (aborted()) return false;
      if (*(volatile int*)(p.status + ST_ABORT)) {
        set_abort();
        return false;
      }
      if ((uint64_t)clock64() - t0 > p.timeout_cycles) {
        raise_error(p, MK_ERR_TIMEOUT, task, op, ctr, v, target, 0);
        set_abort();
        return false;
      }
    }
  }
}

// Bounded wait on a shared-memory mbarrier phase (every calling lane): the
// common already-complete case first, then the bounded spin.
__device__ __forceinline__ bool wait_bar_slow(const Params& p, uint32_t bar, uint32_t parity,
                                           int aux) {
  const uint64_t t0 = clock64();
  for (;;) {
    if (mbar_wait_hint(bar, parity)) return true;
    if (aborted()) return false;
    if ((uint64_t)clock64() - t0 > p.timeout_cycles) {
      raise_error(p, MK_ERR_TIMEOUT, -1, -1, -1, 0, 0, aux);
      set_abort();
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_bar(const Params& p, uint32_t bar, uint32_t parity, int aux) {
  if (mbar_test(bar, parity)) return true;
  return wait_bar_slow(p, bar, parity, aux);
}

// Warp-uniform bounded wait: lane 0 waits, the outcome is broadcast.
__device__ __forceinline__ bool warp_wait(const Params& p, uint32_t bar, uint32_t parity,
                                          int aux) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(p, bar, parity, aux) ? 1 : 0;
  ok = __shfl_sync(FULL, ok, 0);
  return ok != 0;
}

// Wait for a phase that is known to complete (copies in flight), bounded.
__device__ __forceinline__ void drain_bar(const Params& p, uint32_t bar, uint32_t parity) {
  const uint64_t t0 = clock64();
  while (!mbar_wait_hint(bar, parity)) {
    if ((uint64_t)clock64() - t0 > p.timeout_cycles) break;
  }
}

__device__ __forceinline__ void stamp(const Params& p, int task, int field) {
  if (p.trace) p.trace[(size_t)task * kTraceWords + field] = (uint32_t)gtimer();
}


__device__ __forceinline__ void trace_put(const Params& p, int task, int field, uint32_t v) {
  if (p.trace) p.trace[(size_t)task * kTraceWords + field] = v;
}
__device__ __forceinline__ void cstamp(const Params& p, int task, int field) {
  if (p.trace) p.trace[(size_t)task * kTraceWords + field] = (uint32_t)clock64();
}

// ================================================================ routing ==
// Order-preserving key of a float: a larger float gives a larger unsigned key.
__device__ __forceinline__ uint32_t ordered_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// One warp: token b's router logits in layer l from the fixed-point
// accumulators of step parity par, logit_e = share_e * rstd + bias_e with
// rstd = 1/sqrt(sum of squares / d + eps); its top-k (logit descending,
// expert id ascending on ties) into sel[0..k) and the softmax over the k
// selected logits into w[0..k) (shared memory).  logits (may be null)
// receives the token's E logits.  Lane-parallel over experts (E <= 256).
__device__ __forceinline__ void token_route(const Params& p, const float* bias, int l, uint32_t par,
                                         int b, int32_t* sel, float* w, float* logits) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, K = p.k;
  const size_t lb = (size_t)par * p.L + l;
  const float ss = from_fixed(__ldcg(p.ssacc + lb * p.B + b));
  const float rstd = frsqrt(ss / (float)p.d + p.eps);
  const unsigned long long* acc = p.racc + (lb * p.B + b) * E;
  uint32_t key[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int e = lane + 32 * t;
    uint32_t k = 0u;   // 0: taken or absent (no finite logit has key 0)
    if (e < E) {
      const float v = from_fixed(__ldcg(acc + e)) * rstd + (bias ? __ldg(bias + e) : 0.f);
      if (logits) logits[e] = v;
      k = ordered_key(v);
    }
    key[t] = k;
  }
#pragma unroll 1
  for (int j = 0; j < K; ++j) {
    uint32_t bk = 0u;
    int bi = 0x7fffffff;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (key[t] > bk) {   // ascending e within a lane: the first max has the smallest e
        bk = key[t];
        bi = lane + 32 * t;
      }
    }
    const uint32_t mk = __reduce_max_sync(FULL, bk);
    const int wi = __reduce_min_sync(FULL, bk == mk ? bi : 0x7fffffff);
#pragma unroll
    for (int t = 0; t < 8; ++t)
      if (lane + 32 * t == wi) key[t] = 0u;
    if (lane == 0) {
      sel[j] = wi;
      w[j] = key_value(mk);
    }
  }
  __syncwarp();
  // softmax over the selected logits: lane j < K takes rank j
  const float v0 = w[0];
  float x = lane < K ? fexp(w[lane & 7] - v0) : 0.f;
  float sum = x;
  for (int o = 4; o > 0; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
  __syncwarp();
  if (lane < K) w[lane] = x * frcp(sum);
  __syncwarp();
}

// One warp: the layer's routing words (see route_*) from every token's
// selection sel[b * 8 + j] and weight w[b * 8 + j] (shared memory): the
// union of selected experts in ascending id becomes slots 0 .. n_used - 1,
// each with its tokens in ascending order, their ranks and weights; slots
// past n_used hold expert -1.  rt may be shared or global memory; mask is
// kRouteMaskWords words of shared scratch: the union's bitmask, then each
// token's own expert bitmask (a token's position in a slot is the number of
// earlier tokens whose bitmask holds the expert).  Returns n_used.
__device__ __forceinline__ int compact_routes(const Params& p, const int32_t* sel, const float* w,
                                           uint32_t* mask, int32_t* rt) {
  const int lane = threadIdx.x & 31;
  const int B = p.B, K = p.k, S = p.S, BK = B * K;
  uint32_t* tokmask = mask + 8;   // [B][8]
  for (int i = lane; i < 8 + 8 * B; i += 32) mask[i] = 0u;
  __syncwarp();
  for (int q = lane; q < BK; q += 32) {
    const int b = q / K;
    const int e = sel[b * 8 + q - b * K];
    atomicOr(&mask[e >> 5], 1u << (e & 31));
    atomicOr(&tokmask[b * 8 + (e >> 5)], 1u << (e & 31));
  }
  __syncwarp();
  uint32_t m[8];
  int n_used = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m[i] = mask[i];
    n_used += __popc(m[i]);
  }
  if (lane == 0) rt[0] = n_used;
  for (int s = n_used + lane; s < S; s += 32) {
    rt[route_slot_expert(B, K) + s] = -1;
    rt[route_slot_ntok(B, K, S) + s] = 0;
  }
  for (int q = lane; q < BK; q += 32) {
    const int b = q / K, j = q - b * K;
    const int e = sel[b * 8 + j];
    const float wt = w[b * 8 + j];
    rt[route_topk_idx(B, K) + q] = e;
    reinterpret_cast<float*>(rt)[route_topk_w(B, K) + q] = wt;
    // slot of e = the number of used experts below it
    int s = __popc(m[e >> 5] & ((1u << (e & 31)) - 1u));
#pragma unroll
    for (int i = 0; i < 8; ++i) s += (i < (e >> 5)) ? __popc(m[i]) : 0;
    // position among the slot's tokens (earlier tokens that selected e) and,
    // for the first of them, the slot's token count
    const uint32_t bit = 1u << (e & 31);
    int pos = 0, cnt = 0;
#pragma unroll
    for (int b2 = 0; b2 < kMaxBatch; ++b2) {
      if (b2 < B) {
        const int hit = (tokmask[b2 * 8 + (e >> 5)] & bit) ? 1 : 0;
        if (b2 < b) pos += hit;
        else cnt += hit;
      }
    }
    rt[route_slot_tok(B, K, S) + s * 8 + pos] = b;
    rt[route_slot_rank(B, K, S) + s * 8 + pos] = j;
    reinterpret_cast<float*>(rt)[route_slot_w(B, K, S) + s * 8 + pos] = wt;
    if (pos == 0) {
      rt[route_slot_expert(B, K) + s] = e;
      rt[route_slot_ntok(B, K, S) + s] = cnt;
    }
  }
  __syncwarp();
  return n_used;
}

// ============================================================== producer ==
// The producer takes tasks of the step's list from the dispenser (an atomic
// add on a counter that every launch starts at 0), posts each in the CTA's
// task FIFO, and streams its tiles.  A taken index past the end
// posts a stop entry.  The next task is taken as soon as the current one is
// posted (after a long attention chunk: once its stages are issued), so the
// dispenser's round trip overlaps the current task's stage issue.
__device__ __forceinline__ void prefetch_tmap(const void* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}

// A launch parameter moved into a register through an opaque move: a loop
// that uses it keeps it there instead of re-reading the constant bank at
// every use (after switching to other code those reads can miss).
template <typename T>
__device__ __forceinline__ T in_reg(T v) {
  static_assert(sizeof(T) == 4 || sizeof(T) == 8, "32- or 64-bit value");
  if constexpr (sizeof(T) == 8) {
    unsigned long long u = reinterpret_cast<const unsigned long long&>(v), r;
    asm("mov.b64 %0, %1;" : "=l"(r) : "l"(u));
    return reinterpret_cast<const T&>(r);
  } else {
    unsigned u = reinterpret_cast<const unsigned&>(v), r;
    asm("mov.b32 %0, %1;" : "=r"(r) : "r"(u));
    return reinterpret_cast<const T&>(r);
  }
}

__device__ __forceinline__ void producer_loop(const Params& p) {
  const Smem sm = smem_view(p);
  // the values the dispense/resolve/issue path reads, in registers for the
  // whole loop
  struct {
    uint32_t* counters;
    const int32_t *desc, *route, *seq_lens, *page_table;
    const uint8_t* tmaps;
    uint32_t epoch;
    int grab, n_tasks, n_ctas, route_words, B, k, S, E, F, d, max_pages, n_pages, Hkv, hd;
  } const pp = {in_reg(p.counters), in_reg(p.desc), in_reg(p.route), in_reg(p.seq_lens),
                in_reg(p.page_table), in_reg(static_cast<const uint8_t*>(p.tmaps)),
                in_reg(p.epoch), in_reg(p.grab), in_reg(p.n_tasks), in_reg(p.n_ctas),
                in_reg(p.route_words), in_reg(p.B), in_reg(p.k), in_reg(p.S), in_reg(p.E),
                in_reg(p.F), in_reg(p.d), in_reg(p.max_pages), in_reg(p.n_pages), in_reg(p.Hkv),
                in_reg(p.hd)};
  auto tmap_at = [&](int idx) { return static_cast<const void*>(pp.tmaps + (size_t)idx * 128); };
  const int lane = threadIdx.x & 31;
  const int NS = sm.NS;
  uint32_t slot = 0, phase = 0;   // ring position of the next stage
  const uint64_t pol = l2_evict_first();
  auto valid = [&](int t) { return t >= 0 && t < pp.n_tasks; };
  int t_next = 0;
  int32_t dw_next = 0;
  auto take = [&]() {   // next task index and its descriptor (word `lane`)
    uint32_t raw = 0;
    if (lane == 0) raw = atomicAdd(pp.counters + pp.grab, 1u);
    t_next = __shfl_sync(FULL, (int)raw, 0);
    dw_next = valid(t_next) ? __ldg(pp.desc + (size_t)t_next * kDescWords + lane) : 0;
  };
  // an expert tile of an unused slot: the rest of its layer's tiles of that
  // operation are unused too (slots fill in ascending order, tiles are
  // slot-major); move the dispenser past them and take the next task
  auto skip_unused = [&](int32_t dw) {
    const int end = __shfl_sync(FULL, dw, D_C);
    if (lane == 0) atomicMax(pp.counters + pp.grab, (uint32_t)end);
    take();
  };
  int pw_done_ctr = -1;          // producer wait already seen satisfied (this step)
  uint32_t pw_done_tgt = 0;
  int nu_layer = -1, n_used = 0;  // slots used in layer nu_layer (known after its top-k)
  int rc_layer = -1;              // layer whose routing table sm.rcache holds
  auto ring_next = [&]() {
    if (++slot == (uint32_t)NS) {
      slot = 0;
      phase ^= 1u;
    }
  };
  take();
  for (int i = 0;; ++i) {
    const int e = i % kFifo;
    if (!warp_wait(p, sm.fempty(e), ((i / kFifo) & 1) ^ 1, 100)) break;
    const int t = t_next;
    const int32_t dw = dw_next;
    int32_t* ent = sm.fifo + e * kFifoEntryWords;
    if (!valid(t)) {
      ent[D_OP] = OP_NONE;
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.posted(e));
      break;
    }
    const int op = __shfl_sync(FULL, dw, D_OP);
    const int layer = __shfl_sync(FULL, dw, D_LAYER);
    if ((op == OP_GATEUP || op == OP_DOWN) && layer == nu_layer &&
        __shfl_sync(FULL, dw, D_A) >= n_used) {
      skip_unused(dw);   // this FIFO entry stays free for the next task
      --i;
      continue;
    }
    int nstage = __shfl_sync(FULL, dw, D_NSTAGE);
    const int map0 = __shfl_sync(FULL, dw, D_MAP0), map1 = __shfl_sync(FULL, dw, D_MAP1);
    if (lane == 0 && (nstage > 0 || op == OP_ATTN)) {
      prefetch_tmap(tmap_at(map0));
      if (op == OP_GATEUP || op == OP_ATTN) prefetch_tmap(tmap_at(map1));
    }
    int32_t rw = 0;  // resolved word `lane`
    uint32_t pwait = 0;
    int expert = -1, ntok = 0, p0 = 0, seqlen = 0, phys_new = -1, pos = 0;
    bool fail = false;
    if (op == OP_GATEUP || op == OP_DOWN) {
      const int ctr = __shfl_sync(FULL, dw, D_PW);
      const uint32_t tgt = pp.epoch * (uint32_t)__shfl_sync(FULL, dw, D_PWN);
      if (ctr != pw_done_ctr || later(tgt, pw_done_tgt)) {
        int ok = 1;
        if (lane == 0)
          ok = (reached(ld_acquire(pp.counters + ctr), tgt) || wait_counter_slow(p, ctr, tgt, t, op)) ? 1 : 0;
        ok = __shfl_sync(FULL, ok, 0);
        if (!ok) break;
        pw_done_ctr = ctr;
        pw_done_tgt = tgt;
      }
      // The layer's routing table is set up in shared memory once, so the
      // layer's other expert tiles on this CTA resolve without a global round
      // trip: up to kLocalRouteMaxB tokens the producer computes it from the
      // norm tiles' accumulators (final once the norm tiles have signalled,
      // which is what this task's producer wait covered), else it copies the
      // top-k task's table (final once the top-k has signalled).
      __syncwarp();   // the wait's acquire (lane 0) orders every lane's loads
      if (rc_layer != layer && pp.B <= kLocalRouteMaxB) {
        int32_t* tsel = sm.rcache + pp.route_words;
        float* tw = reinterpret_cast<float*>(tsel + 64);
        uint32_t* tmask = reinterpret_cast<uint32_t*>(tw + 64);
        const float* bias = router_b(p, sm, layer);
        for (int b = 0; b < pp.B; ++b)
          token_route(p, bias, layer, pp.epoch & 1u, b, tsel + b * 8, tw + b * 8, nullptr);
        compact_routes(p, tsel, tw, tmask, sm.rcache);
        rc_layer = layer;
      } else if (rc_layer != layer) {
        const int32_t* rt = pp.route + (size_t)layer * pp.route_words;
        for (int w0 = 0; w0 < pp.route_words; w0 += 32 * 16) {
          int32_t v[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int w = w0 + u * 32 + lane;
            v[u] = w < pp.route_words ? __ldcg(rt + w) : 0;
          }
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int w = w0 + u * 32 + lane;
            if (w < pp.route_words) sm.rcache[w] = v[u];
          }
        }
        __syncwarp();
        rc_layer = layer;
      }
      // every routing word of the slot: lane R_EXPERT the expert, R_NTOK the
      // token count, R_TOK/R_RANK/R_W + n token n's id, rank and weight
      // (words past the count are read and then dropped)
      const int j = __shfl_sync(FULL, dw, D_A);
      const int32_t* rt = sm.rcache;
      const int B = pp.B, K = pp.k, S = pp.S;
      int idx = -1;
      if (lane == R_EXPERT) idx = route_slot_expert(B, K) + j;
      else if (lane == R_NTOK) idx = route_slot_ntok(B, K, S) + j;
      else if (lane >= R_TOK && lane < R_TOK + 8) idx = route_slot_tok(B, K, S) + j * 8 + lane - R_TOK;
      else if (lane >= R_RANK && lane < R_RANK + 8)
        idx = route_slot_rank(B, K, S) + j * 8 + lane - R_RANK;
      else if (lane >= R_W && lane < R_W + 8) idx = route_slot_w(B, K, S) + j * 8 + lane - R_W;
      else if (lane == 3) idx = 0;   // slots in use
      const int32_t v = idx >= 0 ? rt[idx] : 0;
      expert = __shfl_sync(FULL, v, R_EXPERT);
      ntok = __shfl_sync(FULL, v, R_NTOK);
      const int used = __shfl_sync(FULL, v, 3);
      if (expert >= pp.E || ntok < 0 || ntok > B || used < 0 || used > S) {
        if (lane == 0) raise_error(p, MK_ERR_DEVICE, t, op, -1, expert, ntok, 1);
        set_abort();
        break;
      }
      nu_layer = layer;
      n_used = used;
      if (expert < 0) {   // an unused slot: its tiles are dropped (the top-k
        skip_unused(dw);  // stood in for their signals)
        --i;
        continue;
      }
      if (lane >= R_TOK && lane < R_W + 8) rw = ((lane - R_TOK) & 7) < ntok ? v : 0;
    } else if (op == OP_ATTN) {
      const int b = __shfl_sync(FULL, dw, D_A);
      const int c = __shfl_sync(FULL, dw, D_C);
      const int nc = __shfl_sync(FULL, dw, D_D);
      const int ppc = __shfl_sync(FULL, dw, D_PPC);
      seqlen = __ldg(pp.seq_lens + b);
      // a prefill group: entries b - grp .. b - 1 hold the tokens before this
      // one, so the chunks read the cached prefix only
      pos = __ldg(p.positions + b);
      const int grp = pos - seqlen;
      const int pages_now = (seqlen + kPage - 1) / kPage;
      p0 = c * ppc;
      int np = min(ppc, pages_now - p0);
      if (np < 0) np = 0;
      const bool last = (c == nc - 1);
      if (seqlen < 0 || grp < 0 || grp > b || (last && p0 + ppc < pages_now) ||
          (pos / kPage) >= pp.max_pages) {
        if (lane == 0) raise_error(p, MK_ERR_STATE, t, op, -1, seqlen, pos, b);
        set_abort();
        fail = true;
      }
      if (!fail && last) {
        phys_new = __ldg(pp.page_table + (size_t)b * pp.max_pages + pos / kPage);
        if (phys_new < 0 || phys_new >= pp.n_pages) {
          if (lane == 0) raise_error(p, MK_ERR_DEVICE, t, op, -1, phys_new, pp.n_pages, 2);
          set_abort();
          fail = true;
        }
      }
      if (fail) break;
      nstage = 2 * np;
      ntok = np;
    }
    if (lane == R_NSTAGE) rw = nstage;
    if (lane == R_EXPERT) rw = expert;
    if (lane == R_NTOK) rw = ntok;
    if (lane == R_P0) rw = p0;
    if (lane == R_SEQLEN) rw = seqlen;
    if (lane == R_PHYS_NEW) rw = phys_new;
    if (lane == R_POS) rw = pos;
    if (lane == R_TASK) rw = t;
    ent[lane] = dw;
    ent[32 + lane] = rw;
    __syncwarp();
    if (lane == 0) {
      stamp(p, t, T_P_RESOLVED);
      if (p.trace) p.trace[(size_t)t * kTraceWords + T_CTA] = blockIdx.x + 1;
      mbar_arrive(sm.posted(e));
    }
    // take the next task now, so its dispenser round trip overlaps this
    // task's stage issue -- except after a long attention chunk (at long
    // contexts one chunk per CTA, hundreds of stages), where a task taken now
    // would wait behind the chunk while other CTAs could run it
    const bool early = op != OP_ATTN || __shfl_sync(FULL, dw, D_PPC) <= kEarlyTakeMaxPages;
    if (early) take();

    // ---- stream the task's tiles
    if (op == OP_ATTN) {
      const int b = __shfl_sync(FULL, dw, D_A);
      const int g = __shfl_sync(FULL, dw, D_B);
      const void* mk_ = tmap_at(map0);
      const void* mv_ = tmap_at(map1);
      const int np = ntok;
      int pg = -1;
      const int* pt = pp.page_table + (size_t)b * pp.max_pages;
      for (int s = 0; s < nstage; ++s) {
        const int pi = s >> 1;
        if ((pi & 31) == 0 && (s & 1) == 0) {
          int idx = p0 + pi + lane;
          pg = (pi + lane < np) ? __ldg(pt + idx) : 0;
          int bad = (pi + lane < np) && (pg < 0 || pg >= pp.n_pages);
          if (__any_sync(FULL, bad)) {
            if (lane == 0) raise_error(p, MK_ERR_DEVICE, t, op, -1, 0, 0, 3);
            set_abort();
            fail = true;
          }
        }
        if (fail) break;
        const int phys = __shfl_sync(FULL, pg, pi & 31);
        if (!warp_wait(p, sm.empty(slot), phase ^ 1, 101)) {
          fail = true;
          break;
        }
        if (lane == 0) {
          const uint32_t bytes = (uint32_t)pp.hd * kPage * 2;
          const uint32_t fb = sm.full(slot);
          mbar_expect_tx(fb, bytes);
          const uint32_t dst = saddr(sm.ring + (size_t)slot * kStageBytes);
          const int y = (phys * pp.Hkv + g) * kPage;
          const void* m = (s & 1) ? mv_ : mk_;
          tma_3d(dst, m, 0, y, 0, fb, pol);   // [hd/64 chunks][64 tokens][128 B]
        }
        __syncwarp();
        ring_next();
      }
      if (fail) break;
    } else if (op == OP_RN && nstage > 0) {
      // the tile's router weights: rows [128 s, 128 s + 128) of its 64-column
      // chunk; rows past E land as zeros
      const int r = __shfl_sync(FULL, dw, D_A);
      const void* m0 = tmap_at(map0);
      const uint32_t box_bytes = (uint32_t)min(pp.E, kRouterRowsPerStage) * 128u;
      for (int s = 0; s < nstage; ++s) {
        if (!warp_wait(p, sm.empty(slot), phase ^ 1, 103)) {
          fail = true;
          break;
        }
        if (lane == 0) {
          const uint32_t fb = sm.full(slot);
          mbar_expect_tx(fb, box_bytes);
          const uint32_t dst = saddr(sm.ring + (size_t)slot * kStageBytes);
          tma_3d(dst, m0, 0, kRouterRowsPerStage * s, r, fb, pol);
        }
        __syncwarp();
        ring_next();
      }
      if (fail) break;
    } else if (nstage > 0) {
      const int nm = __shfl_sync(FULL, dw, D_NMAT);
      const int R = __shfl_sync(FULL, dw, D_R);
      const int MT = R / 16, kcps = 8 / (nm * MT);
      const int k0 = __shfl_sync(FULL, dw, D_K0);
      int row0 = __shfl_sync(FULL, dw, D_ROW0);
      if (op == OP_GATEUP) row0 += expert * pp.F;
      if (op == OP_DOWN) row0 += expert * pp.d;
      const void* m0 = tmap_at(map0);
      const void* m1 = nm > 1 ? tmap_at(map1) : m0;
      for (int s = 0; s < nstage; ++s) {
        const uint64_t w0 = clock64();
        if (!warp_wait(p, sm.empty(slot), phase ^ 1, 102)) {
          fail = true;
          break;
        }
        pwait += (uint32_t)(clock64() - w0);
        if (lane == 0) {
          // one copy per matrix: kcps chunks x R rows, landing as units
          // [matrix][chunk][row tile] of 16 rows x 64 columns
          const uint32_t fb = sm.full(slot);
          mbar_expect_tx(fb, kStageBytes);
          const uint32_t dst = saddr(sm.ring + (size_t)slot * kStageBytes);
          const int z = k0 / 64 + s * kcps;
          tma_3d(dst, m0, 0, row0, z, fb, pol);
          if (nm > 1) tma_3d(dst + kcps * MT * kUnitBytes, m1, 0, row0, z, fb, pol);
        }
        __syncwarp();
        ring_next();
      }
      if (fail) break;
    }
    if (!early) take();
    if (lane == 0) {
      stamp(p, t, T_P_ISSUED);
      trace_put(p, t, T_P_WAITCYC, pwait);
    }
  }
  // drain: every fill issued must land before the CTA may exit.  A slot
  // already filled in the current lap of the ring completes phase `phase`
  // with its last fill, the others phase `phase ^ 1` (for a slot never
  // filled that wait passes at once)
  for (int s2 = 0; s2 < NS; ++s2) {
    const uint32_t st2 = (uint32_t)s2 < slot ? phase : (phase ^ 1u);
    drain_bar(p, sm.full(s2), st2);
  }
  // every producer has taken its last task once all have counted out: the
  // last one starts the next launch's dispenser at 0
  if (lane == 0) {
    const uint32_t old = atomicAdd(pp.counters + p.exit_ctr, 1u);
    if (old + 1u == (uint32_t)pp.n_ctas) {
      atomicExch(pp.counters + pp.grab, 0u);
      atomicExch(pp.counters + p.exit_ctr, 0u);
    }
  }
}

// ================================================================ loader ==
// The loader follows the FIFO: it waits for the producer to post a task,
// spins on the task's counters, and bulk-copies the task's activation into
// shared memory: the normalized input of a level into slot A (reused while
// consecutive A-tasks read the same level; two buffers when they fit), a
// small activation into the next of the two B buffers.
__device__ __forceinline__ void loader_loop(const Params& p) {
  const Smem sm = smem_view(p);
  // the activation sources and sizes, in registers for the whole loop
  struct {
    const uint8_t* actA;
    const float *qkv, *cs;
    const uint8_t *ofrag, *afrag;
    int actA_bytes, actA_stride, actB_bytes, ofrag_bytes, afrag_bytes, S, Hkv, Hq, qkvR, B, hd,
        G;
  } const lp = {in_reg(p.actA), in_reg(p.qkv), in_reg(p.cs), in_reg(p.ofrag), in_reg(p.afrag),
                in_reg(p.actA_bytes), in_reg(p.actA_stride), in_reg(p.actB_bytes),
                in_reg(p.ofrag_bytes), in_reg(p.afrag_bytes), in_reg(p.S), in_reg(p.Hkv),
                in_reg(p.Hq), in_reg(p.qkvR), in_reg(p.B), in_reg(p.hd), in_reg(p.G)};
  const int lane = threadIdx.x & 31;
  int curA = -1, nloadA = 0, nloadB = 0;
  const int nA = p.nA;
  // lane w: the last counter its wait slot saw reach a target this step (the
  // counters only grow within a step, so a later wait on the same counter
  // for no more arrivals needs no load)
  int seen_ctr = -1;
  uint32_t seen_tgt = 0;
  const uint32_t* const ctrs = in_reg(p.counters);
  const uint32_t epoch = in_reg(p.epoch);
  for (int i = 0;; ++i) {
    const int e = i % kFifo;
    if (!warp_wait(p, sm.posted(e), (i / kFifo) & 1, 200)) break;
    const int32_t* ent = sm.fifo + e * kFifoEntryWords;
    const int32_t dw = ent[lane];
    const int op = __shfl_sync(FULL, dw, D_OP);
    if (op == OP_NONE) {
      if (lane == 0) mbar_arrive(sm.ready(e));
      break;
    }
    const int t = ent[32 + R_TASK];
    const int layer = __shfl_sync(FULL, dw, D_LAYER);
    const int act = __shfl_sync(FULL, dw, D_ACT);
    const int nwait = __shfl_sync(FULL, dw, D_NWAIT);
    int ok = 1;
    // lane w polls the task's w-th counter: all counters in one round trip
    if (lane < nwait) {
      const int ctr = ent[D_W0 + 2 * lane];
      const uint32_t tgt = epoch * (uint32_t)ent[D_W0N + 2 * lane];
      if (ctr != seen_ctr || later(tgt, seen_tgt)) {
        ok = (reached(ld_acquire(ctrs + ctr), tgt) || wait_counter_slow(p, ctr, tgt, t, op)) ? 1 : 0;
        seen_ctr = ctr;
        seen_tgt = tgt;
      }
    }
    ok = __all_sync(FULL, ok);
    if (!ok) break;
    if (lane == 0) stamp(p, t, T_L_DEPS);
    bool is_ready = false;
    if (act == ACT_A && layer != curA) {
      // The consumer frees the previous level's buffer when it picks up the
      // first task of the new level, so that task is marked ready before the
      // buffer is waited for (with a single buffer the two would otherwise
      // wait on each other); the consumer then waits for afullA.
      if (lane == 0) {
        stamp(p, t, T_L_ACT);
        mbar_arrive(sm.ready(e));
      }
      is_ready = true;
      const int buf = nloadA % nA;
      if (!warp_wait(p, sm.aemptyA(buf), (uint32_t)(((nloadA / nA) & 1) ^ 1), 201)) break;
      ++nloadA;
      curA = layer;
      if (lane == 0) {
        fence_proxy_async_global();
        const uint32_t fb = sm.afullA(buf);
        mbar_expect_tx(fb, (uint32_t)lp.actA_bytes);
        bulk_g2s(saddr(sm.actA + (size_t)buf * lp.actA_stride),
                 lp.actA + (size_t)layer * lp.actA_bytes, (uint32_t)lp.actA_bytes, fb);
      }
      __syncwarp();
    }
    if (act == ACT_B) {
      const int buf = nloadB & 1;
      if (!warp_wait(p, sm.aemptyB(buf), (uint32_t)(((nloadB >> 1) & 1) ^ 1), 202)) break;
      ++nloadB;
      if (lane == 0) {
        fence_proxy_async_global();
        const uint32_t fb = sm.afullB(buf);
        const uint32_t dst = saddr(sm.actB + (size_t)buf * lp.actB_bytes);
        const int a = ent[D_A];
        const int bb = ent[D_B];
        if (op == OP_ATTN) {
          const int b = a, g = bb, G = lp.G, hd = lp.hd;
          const float* row = lp.qkv + ((size_t)layer * lp.B + b) * lp.qkvR;
          const uint32_t qb = (uint32_t)(G * hd * 4), hb = (uint32_t)(hd * 4);
          mbar_expect_tx(fb, qb + 3 * hb);
          bulk_g2s(dst, row + (size_t)g * G * hd, qb, fb);
          bulk_g2s(dst + qb, row + (size_t)lp.Hq * hd + g * hd, hb, fb);
          bulk_g2s(dst + qb + hb, row + (size_t)(lp.Hq + lp.Hkv) * hd + g * hd, hb, fb);
          bulk_g2s(dst + qb + 2 * hb, lp.cs + (size_t)b * hd, hb, fb);
        } else if (op == OP_OPROJ) {
          const int g = bb;
          mbar_expect_tx(fb, (uint32_t)lp.ofrag_bytes);
          bulk_g2s(dst, lp.ofrag + ((size_t)layer * lp.Hkv + g) * lp.ofrag_bytes,
                   (uint32_t)lp.ofrag_bytes, fb);
        } else {  // OP_DOWN
          const int j = a;
          mbar_expect_tx(fb, (uint32_t)lp.afrag_bytes);
          bulk_g2s(dst, lp.afrag + ((size_t)layer * lp.S + j) * lp.afrag_bytes,
                   (uint32_t)lp.afrag_bytes, fb);
        }
      }
      __syncwarp();
    }
    if (lane == 0 && !is_ready) {
      stamp(p, t, T_L_ACT);
      mbar_arrive(sm.ready(e));
    }
    __syncwarp();
  }
  // drain activation copies in flight (the last load of each buffer)
  for (int b = 0; b < nA; ++b)
    if (nloadA > b) drain_bar(p, sm.afullA(b), (uint32_t)((((nloadA - 1 - b) / nA)) & 1));
  for (int b = 0; b < 2; ++b)
    if (nloadB > b) drain_bar(p, sm.afullB(b), (uint32_t)(((nloadB - 1 - b) / 2) & 1));
}

// ============================================================== signaler ==
__device__ __forceinline__ void signal_loop(const Params& p) {
  const Smem sm = smem_view(p);
  const int lane = threadIdx.x & 31;
  uint32_t* const ctrs = in_reg(p.counters);
  for (int i = 0;; ++i) {
    const int e = i % kFifo;
    if (!warp_wait(p, sm.done(e), (i / kFifo) & 1, 300)) break;
    const int32_t* ent = sm.fifo + e * kFifoEntryWords;
    if (ent[D_OP] == OP_NONE) break;
    if (lane == 0) {
      const int nsig = ent[D_NSIG];
      for (int s = 0; s < nsig; ++s) red_release_add(ctrs + ent[D_S0 + s], 1u);
      mbar_arrive(sm.fempty(e));
    }
    __syncwarp();
  }
}

// ============================================================= consumers ==
// consumer thread / warp / lane indices
#define MK_CONSUMER_IDS                                        \
  const int ct = (int)threadIdx.x - kFirstConsumerWarp * 32;   \
  const int cw = ct >> 5;                                      \
  const int lane = (int)threadIdx.x & 31;                      \
  (void)ct;                                                    \
  (void)cw;                                                    \
  (void)lane

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts16(uint32_t addr, unsigned short v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ float2 lds64f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Stage ring position: slot and phase advance together (no division in
// the stage loops).
struct Ring {
  uint32_t slot, phase;
  int NS;
  __device__ void init(uint32_t stage_ctr, int ns) {
    NS = ns;
    slot = stage_ctr % (uint32_t)ns;
    phase = (stage_ctr / (uint32_t)ns) & 1u;
  }
  __device__ void next() {
    if (++slot == (uint32_t)NS) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// CUDA-core stage loop for 1 or 2 activation columns (partial rows of pc
// floats): exact fp32 FMAs of bf16 weights (widened by a shift/mask) with fp32
// activations, two per instruction (ffma2): each row keeps the sums of its even
// and odd columns, added at the end.  Lane l reads
// 16-byte chunk (l & 7) of rows (l >> 3) + 4i of its warp's 16-row unit, so a
// warp's 32 lanes cover the unit's 512 bytes per row group without bank
// conflicts; partial sums are reduced over the 8 lanes of a row at the end.
template <int NB>
__device__ __forceinline__ void gemv_stages_ffma(const Params& p, const Smem& sm, int nstage,
                                                 int kcps, int kl, uint32_t xaddr0,
                                                 uint32_t xaddr1, Ring& ring, float* part_w,
                                                 uint32_t pe_bar, uint32_t pe_par,
                                                 uint32_t& waitcyc, int pc) {
  MK_CONSUMER_IDS;
  const int c = lane & 7, rg = lane >> 3;
  float acc[4][NB], acc_odd[4][NB];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[i][b] = acc_odd[i][b] = 0.f;
  uint32_t woff[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = rg + 4 * i;
    woff[i] = r * 128 + ((c ^ (r & 7)) << 4);
  }
  const uint32_t ring0 = saddr(sm.ring) + cw * kUnitBytes;
  for (int s = 0; s < nstage; ++s) {
    const uint64_t w0 = clock64();
    wait_bar(p, sm.full(ring.slot), ring.phase, 400);
    waitcyc += (uint32_t)(clock64() - w0);
    __syncwarp();
    const uint32_t ub = ring0 + ring.slot * kStageBytes;
    const uint32_t koff = (uint32_t)((s * kcps + kl) * 64 + 8 * c) * 4u;
    uint4 w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = lds128(ub + woff[i]);
    float4 xa[NB], xb[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const uint32_t xo = (b == 0 ? xaddr0 : xaddr1) + koff;
      const uint4 u0 = lds128(xo), u1 = lds128(xo + 16);
      xa[b] = make_float4(__uint_as_float(u0.x), __uint_as_float(u0.y), __uint_as_float(u0.z),
                          __uint_as_float(u0.w));
      xb[b] = make_float4(__uint_as_float(u1.x), __uint_as_float(u1.y), __uint_as_float(u1.z),
                          __uint_as_float(u1.w));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.empty(ring.slot));
    ring.next();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        float e = acc[i][b], o = acc_odd[i][b];
        ffma2(e, o, lo_bf16(w[i].x), hi_bf16(w[i].x), xa[b].x, xa[b].y);
        ffma2(e, o, lo_bf16(w[i].y), hi_bf16(w[i].y), xa[b].z, xa[b].w);
        ffma2(e, o, lo_bf16(w[i].z), hi_bf16(w[i].z), xb[b].x, xb[b].y);
        ffma2(e, o, lo_bf16(w[i].w), hi_bf16(w[i].w), xb[b].z, xb[b].w);
        acc[i][b] = e;
        acc_odd[i][b] = o;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float a = acc[i][b] + acc_odd[i][b];
      a += __shfl_xor_sync(FULL, a, 1);
      a += __shfl_xor_sync(FULL, a, 2);
      a += __shfl_xor_sync(FULL, a, 4);
      acc[i][b] = a;
    }
  wait_bar(p, pe_bar, pe_par, 403);   // the epilogue warp has read this buffer's last use
  if (c == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int b = 0; b < NB; ++b) part_w[(rg + 4 * i) * pc + b] = acc[i][b];
  }
}

// Tensor-core stage loop for 3..8 activation columns: weights as the 16-row
// A operand (ldmatrix from the swizzled tile), the fp32 activation columns
// as the B operand split into three bf16 terms (hi + mid + lo, exact
// differences, ~24 bits), accumulated into three independent fp32 chains.
__device__ __forceinline__ void gemv_stages_mma(const Params& p, const Smem& sm, int nstage,
                                                int kcps, int kl, uint32_t xaddr, Ring& ring,
                                                float* part_w, uint32_t pe_bar, uint32_t pe_par,
                                                uint32_t& waitcyc) {
  MK_CONSUMER_IDS;
  const int g8 = lane >> 2, q = lane & 3;
  float ah[4] = {0.f, 0.f, 0.f, 0.f}, am[4] = {0.f, 0.f, 0.f, 0.f},
        al[4] = {0.f, 0.f, 0.f, 0.f};
  const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int achunk_hi = lane >> 4;
  const uint32_t ring0 = saddr(sm.ring) + cw * kUnitBytes + arow * 128;
  for (int s = 0; s < nstage; ++s) {
    const uint64_t w0 = clock64();
    wait_bar(p, sm.full(ring.slot), ring.phase, 400);
    waitcyc += (uint32_t)(clock64() - w0);
    __syncwarp();
    const uint32_t ub = ring0 + ring.slot * kStageBytes;
    const uint32_t kbase = xaddr + (uint32_t)((s * kcps + kl) * 64 + 2 * q) * 4u;
    uint32_t a[4][4];
    float2 b0[4], b1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int chunk = 2 * i + achunk_hi;
      ldsm_x4(ub + ((chunk ^ (arow & 7)) << 4), a[i][0], a[i][1], a[i][2], a[i][3]);
      b0[i] = lds64f(kbase + i * 64);
      b1[i] = lds64f(kbase + i * 64 + 32);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.empty(ring.slot));
    ring.next();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t h0, m0, l0, h1, m1, l1;
      split3(b0[i].x, b0[i].y, h0, m0, l0);
      split3(b1[i].x, b1[i].y, h1, m1, l1);
      mma16816(ah, a[i][0], a[i][1], a[i][2], a[i][3], h0, h1);
      mma16816(am, a[i][0], a[i][1], a[i][2], a[i][3], m0, m1);
      mma16816(al, a[i][0], a[i][1], a[i][2], a[i][3], l0, l1);
    }
  }
  wait_bar(p, pe_bar, pe_par, 403);   // the epilogue warp has read this buffer's last use
  part_w[g8 * 8 + 2 * q] = ah[0] + (am[0] + al[0]);
  part_w[g8 * 8 + 2 * q + 1] = ah[1] + (am[1] + al[1]);
  part_w[(g8 + 8) * 8 + 2 * q] = ah[2] + (am[2] + al[2]);
  part_w[(g8 + 8) * 8 + 2 * q + 1] = ah[3] + (am[3] + al[3]);
}

// Generic skinny GEMV tile, consumer side: n_mat matrices x R rows x
// (KCH*64) columns against up to 8 activation columns.  `act` holds the
// activation as fp32 rows of `stride` floats; output column n reads row
// colrow(n) (the slot's token list for expert gate/up, else n); columns >=
// ncols read row 0 and are ignored by the epilogue.  Each warp streams its
// own 16-row unit of every stage and leaves its partial sums in `pw`
// ([16][part_cols]); the epilogue warp reduces the warps' partials.
template <int NBK>
__device__ __forceinline__ uint32_t gemv_consume(const Params& p, const int32_t* ent,
                                                 const float* act, int stride,
                                                 const int32_t* tokmap, int ncols, float* pw,
                                                 uint32_t pe_bar, uint32_t pe_par,
                                                 uint32_t stage_ctr) {
  const Smem sm = smem_view(p);
  MK_CONSUMER_IDS;
  const int nstage = ent[32 + R_NSTAGE];
  const int nm = ent[D_NMAT], R = ent[D_R];
  const int MT = R / 16, kcps = 8 / (nm * MT);
  const int kl = (cw / MT) % kcps;   // unit cw = (matrix * kcps + chunk) * MT + row tile
  Ring ring;
  ring.init(stage_ctr, sm.NS);
  const uint32_t xbase = saddr(act);
  auto row_of = [&](int n) { return n < ncols ? (tokmap ? tokmap[n] : n) : 0; };
  uint32_t waitcyc = 0;
  if (ct == 0) cstamp(p, ent[32 + R_TASK], T_K2);
  const uint64_t l0 = clock64();
  if constexpr (NBK == 1) {
    gemv_stages_ffma<1>(p, sm, nstage, kcps, kl, xbase + row_of(0) * stride * 4, 0, ring, pw,
                        pe_bar, pe_par, waitcyc, 1);
  } else if constexpr (NBK == 2) {
    gemv_stages_ffma<2>(p, sm, nstage, kcps, kl, xbase + row_of(0) * stride * 4,
                        xbase + row_of(1) * stride * 4, ring, pw, pe_bar, pe_par, waitcyc, 2);
  } else if (ncols == 1) {
    // an expert tile of one or two tokens in a larger batch: the exact FFMA
    // path costs fewer instructions per stage than eight mma columns
    gemv_stages_ffma<1>(p, sm, nstage, kcps, kl, xbase + row_of(0) * stride * 4, 0, ring, pw,
                        pe_bar, pe_par, waitcyc, 8);
  } else if (ncols == 2) {
    gemv_stages_ffma<2>(p, sm, nstage, kcps, kl, xbase + row_of(0) * stride * 4,
                        xbase + row_of(1) * stride * 4, ring, pw, pe_bar, pe_par, waitcyc, 8);
  } else {
    gemv_stages_mma(p, sm, nstage, kcps, kl, xbase + row_of(lane >> 2) * stride * 4, ring, pw,
                    pe_bar, pe_par, waitcyc);
  }
  if (ct == 0) {
    trace_put(p, ent[32 + R_TASK], T_C_LOOPCYC, (uint32_t)(clock64() - l0));
    trace_put(p, ent[32 + R_TASK], T_C_WAITCYC, waitcyc);
    cstamp(p, ent[32 + R_TASK], T_K3);
    stamp(p, ent[32 + R_TASK], T_C_MATH);
  }
  return stage_ctr + (uint32_t)nstage;
}

// GEMV tile, epilogue side (one warp): sums the consumer warps' partials
// over the column chunks that shared a row tile, in chunk order, and writes
// the operation's outputs.  `rs` is the level's 1/rms per token (A-input
// operations).
// The launch parameters the epilogue writes through, held in registers for the
// whole loop (see in_reg).
struct EpiParams {
  float *qkv, *logits, *o_part, *expert_a, *moe_part;
  uint8_t* afrag;
  int qkvR, V, Hkv, d, S, F, afrag_bytes, k, B, PC;
  __device__ explicit EpiParams(const Params& p)
      : qkv(in_reg(p.qkv)), logits(in_reg(p.logits)), o_part(in_reg(p.o_part)),
        expert_a(in_reg(p.expert_a)), moe_part(in_reg(p.moe_part)), afrag(in_reg(p.afrag)),
        qkvR(in_reg(p.qkvR)), V(in_reg(p.V)), Hkv(in_reg(p.Hkv)), d(in_reg(p.d)), S(in_reg(p.S)),
        F(in_reg(p.F)), afrag_bytes(in_reg(p.afrag_bytes)), k(in_reg(p.k)), B(in_reg(p.B)),
        PC(in_reg(p.part_cols)) {}
};

// LM-head tile epilogue: the logits of the tile's rows for every token, and in
// a greedy step each token's best logit of the tile with its lowest row,
// folded into amax[n] as the 64-bit key (ordered logit << 32 | ~row), whose
// maximum over all tiles is the largest logit at the lowest row.
__device__ __forceinline__ void lm_epilogue(const EpiParams& p, const Params& pr,
                                            const int32_t* ent, const float* part,
                                            const float* rs) {
  const int lane = threadIdx.x & 31;
  const int R = ent[D_R], row0 = ent[D_ROW0];
  const int MT = R / 16, kcps = 8 / MT;
  const int PC = p.PC;
  unsigned long long* const amax = pr.g_tok ? pr.amax : nullptr;
  for (int n = 0; n < p.B; ++n) {
    uint32_t bk = 0u;
    int brow = 0x7fffffff;
    for (int r = lane; r < R; r += 32) {   // rows ascend per lane: the first max is kept
      const int mt = r >> 4, r16 = r & 15;
      float s0 = 0.f;
      for (int kc = 0; kc < kcps; ++kc) s0 += part[((kc * MT + mt) * 16 + r16) * PC + n];
      const int row = row0 + r;
      if (row < p.V) {
        const float v = s0 * rs[n];
        p.logits[(size_t)n * p.V + row] = v;
        const uint32_t key = ordered_key(v);
        if (key > bk) {
          bk = key;
          brow = row;
        }
      }
    }
    if (amax) {
      const uint32_t mk_ = __reduce_max_sync(FULL, bk);
      const int mrow = __reduce_min_sync(FULL, bk == mk_ ? brow : 0x7fffffff);
      if (lane == 0 && mrow != 0x7fffffff)
        atomicMax(amax + n, ((unsigned long long)mk_ << 32) | (unsigned long long)(~(uint32_t)mrow));
    }
  }
}

// After an LM-head tile: its arrival; the tile that completes the step's
// count (it has acquired every tile's keys) takes each token's key (resetting
// it to zero for the next step) and, in a greedy step, writes the token, feeds
// it to the next step and advances the position and length by one.
__device__ __forceinline__ void lm_finish(const Params& p, const int32_t* ent) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  int last = 0;
  if (lane == 0) {
    const uint32_t old = atom_add_acq_rel(p.counters + ent[D_X0], 1u);
    last = old + 1u == p.epoch * (uint32_t)ent[D_X1];
  }
  if (!__shfl_sync(FULL, last, 0)) return;
  if (p.g_tok && lane < p.B) {
    const unsigned long long key = atomicExch(p.amax + lane, 0ull);
    const int tok = (int)~(uint32_t)key;
    p.g_out[lane] = tok;
    p.g_tok[lane] = tok;
    p.g_pos[lane] += 1;
    if (p.g_len != p.g_pos) p.g_len[lane] += 1;   // one buffer may serve as both
  }
  __syncwarp();
  if (lane == 0) red_release_add(p.counters + ent[D_X2], 1u);
}

__device__ __forceinline__ void gemv_epilogue(const EpiParams& p, const int32_t* ent,
                                              const float* part, const float* rs) {
  const int lane = threadIdx.x & 31;
  const int op = ent[D_OP], layer = ent[D_LAYER];
  const int nm = ent[D_NMAT], R = ent[D_R], row0 = ent[D_ROW0];
  const int MT = R / 16, MTn = nm * MT, kcps = 8 / MTn;
  const int PC = p.PC;
  const bool expert = (op == OP_GATEUP || op == OP_DOWN);
  const int ncols = expert ? ent[32 + R_NTOK] : p.B;
  const int n_out = R * ncols;
  for (int idx = lane; idx < n_out; idx += 32) {
    const int n = idx / R, r = idx - n * R;   // r fastest: coalesced output rows
    const int mt = r >> 4, r16 = r & 15;
    float s0 = 0.f, s1 = 0.f;
    for (int kc = 0; kc < kcps; ++kc) {
      s0 += part[((kc * MT + mt) * 16 + r16) * PC + n];
      if (nm > 1) s1 += part[(((kcps + kc) * MT + mt) * 16 + r16) * PC + n];
    }
    const int row = row0 + r;
    switch (op) {
      case OP_QKV:
        p.qkv[((size_t)layer * p.B + n) * p.qkvR + row] = s0 * rs[n];
        break;
      case OP_OPROJ: {
        const int g = ent[D_B];
        p.o_part[(((size_t)layer * p.Hkv + g) * p.B + n) * p.d + row] = s0;
        break;
      }
      case OP_GATEUP: {
        const int f = ent[D_B], j = ent[D_A];
        const float rt = rs[ent[32 + R_TOK + n]];
        const float gt = s0 * rt, ut = s1 * rt;
        const float a = gt * frcp(1.0f + fexp(-gt)) * ut;
        p.expert_a[(((size_t)layer * p.S + j) * p.B + n) * p.F + f * R + r] = a;
        float* arow =
            reinterpret_cast<float*>(p.afrag + ((size_t)layer * p.S + j) * p.afrag_bytes);
        arow[(size_t)n * (p.F + kActPad) + f * R + r] = a;
        break;
      }
      default: {  // OP_DOWN
        const int tok = ent[32 + R_TOK + n];
        const int rank = ent[32 + R_RANK + n];
        const float w = __int_as_float(ent[32 + R_W + n]);
        p.moe_part[(((size_t)layer * p.k + rank) * p.B + tok) * p.d + row] = w * s0;
        break;
      }
    }
  }
}

__device__ __forceinline__ bool is_gemv(int op) {
  return op == OP_QKV || op == OP_OPROJ || op == OP_GATEUP ||
         op == OP_DOWN || op == OP_LMHEAD;
}

// Write the normalized attention output o[G][hd] (smem) of token b, group g:
// fp32 copy and the O-proj B-operand fragments.
__device__ __forceinline__ void write_attn_out(const Params& p, int layer, int b, int g,
                                           const float* o) {
  MK_CONSUMER_IDS;
  const int G = p.G, hd = p.hd, B = p.B;
  float* dst = p.attn_o + ((size_t)layer * B + b) * (size_t)p.Hq * hd + (size_t)g * G * hd;
  for (int idx = ct; idx < G * hd; idx += 256) dst[idx] = o[idx];
  float* row = reinterpret_cast<float*>(p.ofrag + ((size_t)layer * p.Hkv + g) * p.ofrag_bytes) +
               (size_t)b * (G * hd + kActPad);
  for (int idx = ct; idx < G * hd; idx += 256) row[idx] = o[idx];
}

template <int HD>
__device__ __forceinline__ uint32_t attn_task(const Params& p, const int32_t* ent, const uint8_t* act,
                                           uint32_t stage_ctr) {
  const Smem sm = smem_view(p);
  MK_CONSUMER_IDS;
  const int layer = ent[D_LAYER], b = ent[D_A], g = ent[D_B], chunk = ent[D_C];
  const int flags = ent[D_FLAGS];
  const int np = ent[32 + R_NTOK], p0 = ent[32 + R_P0], seqlen = ent[32 + R_SEQLEN];
  const int phys_new = ent[32 + R_PHYS_NEW], pos = ent[32 + R_POS];
  const int G = p.G;
  const int g8 = lane >> 2, q = lane & 3;
  constexpr int HALF = HD / 2;
  const float* q_raw = reinterpret_cast<const float*>(act);
  const float* k_raw = q_raw + G * HD;
  const float* v_raw = k_raw + HD;
  const float* csv = v_raw + HD;
  float* mrg = p.attn_in_actB                              // [8][G][HD+4]
                   ? reinterpret_cast<float*>(const_cast<uint8_t*>(act) + (G + 3) * HD * 4)
                   : reinterpret_cast<float*>(sm.scratch);
  float* qs = mrg + 8 * G * (HD + 4);                      // [G][HD]
  float* kn = qs + G * HD;                                 // [HD]
  float* vn = kn + HD;                                     // [HD]
  // The rotated, scaled query as the A operand of the score MMAs: a bf16
  // tile of 8 rows x HD, rows [0, G) the hi halves and rows [G, 2G) the lo
  // halves (the rest zero), its 16-byte chunks swizzled by row so that the
  // page loop's ldmatrix reads are conflict-free.  It sits in the merge
  // area, which is idle until the page loop ends.
  const uint32_t qt = saddr(mrg);
  auto qt_off = [](int row, int i) {
    const int c = i >> 3;
    return (uint32_t)(row * HD * 2 + (((c & ~7) | ((c ^ row) & 7)) << 4) + (i & 7) * 2);
  };
  const float qscale = 1.4426950408889634f / sqrtf((float)HD);
  for (int idx = ct; idx < G * HD; idx += 256) {
    const int h = idx / HD, i = idx % HD, i1 = i % HALF;
    const float co = csv[i1], si = csv[HALF + i1];
    const float x = q_raw[h * HD + i];
    const float y = (i < HALF) ? q_raw[h * HD + i + HALF] : q_raw[h * HD + i - HALF];
    const float r = (i < HALF) ? (x * co - y * si) : (x * co + y * si);
    const float v = r * qscale;
    qs[idx] = v;
    const __nv_bfloat16 hb = __float2bfloat16_rn(v);
    const __nv_bfloat16 lb = __float2bfloat16_rn(v - __bfloat162float(hb));
    sts16(qt + qt_off(h, i), __bfloat16_as_ushort(hb));
    sts16(qt + qt_off(G + h, i), __bfloat16_as_ushort(lb));
  }
  for (int idx = 2 * G * HD + ct; idx < 8 * HD; idx += 256)
    sts16(qt + qt_off(idx / HD, idx % HD), 0);
  for (int i = ct; i < HD; i += 256) {
    const int i1 = i % HALF;
    const float co = csv[i1], si = csv[HALF + i1];
    const float x = k_raw[i];
    const float y = (i < HALF) ? k_raw[i + HALF] : k_raw[i - HALF];
    const float r = (i < HALF) ? (x * co - y * si) : (x * co + y * si);
    const __nv_bfloat16 kb = __float2bfloat16_rn(r);
    const __nv_bfloat16 vb = __float2bfloat16_rn(v_raw[i]);
    kn[i] = __bfloat162float(kb);
    vn[i] = __bfloat162float(vb);
    if (flags & F_LAST_CHUNK) {
      const size_t off = (((size_t)phys_new * p.Hkv + g) * kPage + (pos % kPage)) * HD + i;
      reinterpret_cast<__nv_bfloat16*>(kpool_of(p, sm, layer))[off] = kb;
      reinterpret_cast<__nv_bfloat16*>(vpool_of(p, sm, layer))[off] = vb;
    }
  }
  cbar();
  // this lane's ldmatrix rows of the query tile: row lane % 8, chunk
  // 4 k2 + lane / 8 for the k2-th 32 columns (two 16-wide k steps)
  uint32_t qaddr[HD / 32];
#pragma unroll
  for (int k2 = 0; k2 < HD / 32; ++k2) qaddr[k2] = qt + qt_off(lane & 7, 32 * k2 + 8 * (lane >> 3));
  float m_run = -1e30f, l_run = 0.f;
  float acc[HD / 8][4];
#pragma unroll
  for (int j = 0; j < HD / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  // The new token joins the softmax of the chunk that owns it (warp 0).  In
  // a prefill group so do the group's earlier tokens, which are not in the
  // pool yet: their K (rotated at their own positions) and V come from this
  // step's QKV output, rounded to bf16 as the pool stores them.
  if ((flags & F_LAST_CHUNK) && cw == 0) {
    float sn[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = lane; i < HD; i += 32)
      for (int h = 0; h < G; ++h) sn[h] += qs[h * HD + i] * kn[i];
#pragma unroll
    for (int h = 0; h < 4; ++h)
      for (int o = 16; o > 0; o >>= 1) sn[h] += __shfl_xor_sync(FULL, sn[h], o);
    if (g8 < G) {
      m_run = sn[g8];
      l_run = 1.f;
#pragma unroll
      for (int j = 0; j < HD / 8; ++j) {
        acc[j][0] = vn[8 * j + 2 * q];
        acc[j][1] = vn[8 * j + 2 * q + 1];
      }
    }
    const int grp = pos - seqlen;
#pragma unroll 1
    for (int j = 0; j < grp; ++j) {
      const int bj = b - grp + j;
      const float* kr = p.qkv + ((size_t)layer * p.B + bj) * p.qkvR + (size_t)p.Hq * HD + g * HD;
      const float* vr = kr + (size_t)p.Hkv * HD;
      const float* cs = p.cs + (size_t)bj * HD;
      float sj[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = lane; i < HD; i += 32) {
        const int i1 = i % HALF;
        const float co = __ldcg(cs + i1), si = __ldcg(cs + HALF + i1);
        const float x = __ldcg(kr + i);
        const float y = __ldcg(kr + (i < HALF ? i + HALF : i - HALF));
        const float kv = bf16r(i < HALF ? (x * co - y * si) : (x * co + y * si));
#pragma unroll
        for (int h = 0; h < 4; ++h)
          if (h < G) sj[h] += qs[h * HD + i] * kv;
      }
#pragma unroll
      for (int h = 0; h < 4; ++h)
        for (int o = 16; o > 0; o >>= 1) sj[h] += __shfl_xor_sync(FULL, sj[h], o);
      if (g8 < G) {
        const float sc = g8 == 0 ? sj[0] : g8 == 1 ? sj[1] : g8 == 2 ? sj[2] : sj[3];
        const float m_new = fmaxf(m_run, sc);
        const float alpha = ex2(m_run - m_new), e = ex2(sc - m_new);
        l_run = l_run * alpha + e;
        m_run = m_new;
#pragma unroll
        for (int jj = 0; jj < HD / 8; ++jj) {
          const float2 t2 = __ldcg(reinterpret_cast<const float2*>(vr + 8 * jj + 2 * q));
          acc[jj][0] = acc[jj][0] * alpha + e * bf16r(t2.x);
          acc[jj][1] = acc[jj][1] * alpha + e * bf16r(t2.y);
        }
      }
    }
  }
  const int key8 = 8 * cw;
  const int krow = key8 + (lane & 7);
  Ring ring;   // K and V stages alternate; the position advances without a division
  ring.init(stage_ctr, sm.NS);
  for (int pi = 0; pi < np; ++pi) {
    // ---- K page: scores of this warp's 8 keys for the G heads
    uint32_t qa[HD / 32][4];
#pragma unroll
    for (int k2 = 0; k2 < HD / 32; ++k2)
      ldsm_x4(qaddr[k2], qa[k2][0], qa[k2][1], qa[k2][2], qa[k2][3]);
    wait_bar(p, sm.full(ring.slot), ring.phase, 401);
    __syncwarp();
    const uint32_t kb = saddr(sm.ring + (size_t)ring.slot * kStageBytes);
    float sc[4] = {0.f, 0.f, 0.f, 0.f}, sd[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t kr[HD / 32][4];
#pragma unroll
    for (int k2 = 0; k2 < HD / 32; ++k2) {
      const int hd0 = k2 * 32;
      const int box = hd0 / 64;
      const int chunk = ((hd0 % 64) >> 3) + (lane >> 3);
      ldsm_x4(kb + box * 8192 + krow * 128 + ((chunk ^ (krow & 7)) << 4), kr[k2][0], kr[k2][1],
              kr[k2][2], kr[k2][3]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.empty(ring.slot));
    ring.next();
    ++stage_ctr;
#pragma unroll
    for (int k2 = 0; k2 < HD / 32; ++k2) {
      mma16816(sc, qa[k2][0], 0u, qa[k2][1], 0u, kr[k2][0], kr[k2][1]);
      mma16816(sd, qa[k2][2], 0u, qa[k2][3], 0u, kr[k2][2], kr[k2][3]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) sc[j] += sd[j];
    float s0 = sc[0] + __shfl_down_sync(FULL, sc[0], 4 * G);
    float s1 = sc[1] + __shfl_down_sync(FULL, sc[1], 4 * G);
    const int kidx = (p0 + pi) * kPage + key8 + 2 * q;
    if (kidx >= seqlen) s0 = -INFINITY;
    if (kidx + 1 >= seqlen) s1 = -INFINITY;
    float mx = fmaxf(s0, s1);
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = ex2(m_run - m_new);
    const float e0 = ex2(s0 - m_new), e1 = ex2(s1 - m_new);
    float ps = e0 + e1;
    ps += __shfl_xor_sync(FULL, ps, 1);
    ps += __shfl_xor_sync(FULL, ps, 2);
    l_run = l_run * alpha + ps;
    m_run = m_new;
    // lanes holding the lo rows take their head's scale and probabilities
    const float alpha_lo = __shfl_up_sync(FULL, alpha, 4 * G);
    const float e0_lo = __shfl_up_sync(FULL, e0, 4 * G);
    const float e1_lo = __shfl_up_sync(FULL, e1, 4 * G);
    float my_alpha = 1.f;
    uint32_t pa = 0u;
    if (g8 < G) {
      my_alpha = alpha;
      pa = pack_bf16(e0, e1);
    } else if (g8 < 2 * G) {
      my_alpha = alpha_lo;
      pa = pack_bf16(e0_lo - bf16r(e0_lo), e1_lo - bf16r(e1_lo));
    }
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
      acc[j][0] *= my_alpha;
      acc[j][1] *= my_alpha;
    }
    // ---- V page: acc += P V
    wait_bar(p, sm.full(ring.slot), ring.phase, 402);
    __syncwarp();
    const uint32_t vb = saddr(sm.ring + (size_t)ring.slot * kStageBytes);
#pragma unroll
    for (int j4 = 0; j4 < HD / 32; ++j4) {
      const int hd0 = j4 * 32;
      const int box = hd0 / 64;
      const int chunk = ((hd0 % 64) >> 3) + (lane >> 3);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vb + box * 8192 + krow * 128 + ((chunk ^ (krow & 7)) << 4), b0, b1, b2, b3);
      mma1688(acc[4 * j4 + 0], pa, 0u, b0);
      mma1688(acc[4 * j4 + 1], pa, 0u, b1);
      mma1688(acc[4 * j4 + 2], pa, 0u, b2);
      mma1688(acc[4 * j4 + 3], pa, 0u, b3);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.empty(ring.slot));
    ring.next();
    ++stage_ctr;
  }
  if (ct == 0) stamp(p, ent[32 + R_TASK], T_C_MATH);
  cbar();   // every warp is done with the query tile in the merge area
  // ---- per-warp state -> shared memory: O = hi rows + lo rows
  float* mw = mrg + cw * G * (HD + 4);
#pragma unroll
  for (int j = 0; j < HD / 8; ++j) {
    const float o0 = acc[j][0] + __shfl_down_sync(FULL, acc[j][0], 4 * G);
    const float o1 = acc[j][1] + __shfl_down_sync(FULL, acc[j][1], 4 * G);
    if (g8 < G) {
      mw[g8 * (HD + 4) + 8 * j + 2 * q] = o0;
      mw[g8 * (HD + 4) + 8 * j + 2 * q + 1] = o1;
    }
  }
  if (g8 < G && q == 0) {
    mw[g8 * (HD + 4) + HD] = m_run;
    mw[g8 * (HD + 4) + HD + 1] = l_run;
  }
  cbar();
  // ---- merge the 8 warps
  float* osm = qs;  // reuse: [G][HD]
  const bool single = (flags & F_SINGLE) != 0;
  float* part = p.attn_part +
                ((((size_t)layer * p.B + b) * p.Hkv + g) * p.max_chunks + chunk) * p.part_stride;
  for (int idx = ct; idx < G * HD; idx += 256) {
    const int h = idx / HD, i = idx % HD;
    float M = -1e30f;
    for (int w = 0; w < 8; ++w) M = fmaxf(M, mrg[(w * G + h) * (HD + 4) + HD]);
    float Lsum = 0.f, O = 0.f;
    for (int w = 0; w < 8; ++w) {
      const float* mwp = mrg + (w * G + h) * (HD + 4);
      const float sc = ex2(mwp[HD] - M);
      Lsum += sc * mwp[HD + 1];
      O += sc * mwp[i];
    }
    if (single) {
      osm[idx] = O * frcp(Lsum);
    } else {
      part[idx] = O;   // chunk record: [O (G x hd)][m (G)][l (G)]
      if (i == 0) {
        part[G * HD + h] = M;
        part[G * HD + G + h] = Lsum;
      }
    }
  }
  if (single) {
    cbar();
    write_attn_out(p, layer, b, g, osm);
  }
  return stage_ctr;
}

// Log-sum-exp merge of the chunk partials of (token b, KV group g).  Every
// load is issued in parallel across the CTA (no per-chunk dependency chain).
__device__ __forceinline__ void combine_task(const Params& p, const int32_t* ent) {
  const Smem sm = smem_view(p);
  MK_CONSUMER_IDS;
  const int layer = ent[D_LAYER], b = ent[D_A], g = ent[D_B], nc = ent[D_D];
  const int G = p.G, hd = p.hd, PS = p.part_stride, GH = G * hd;
  // chunk records [O (G x hd)][m (G)][l (G)], PS floats apart
  const float* parts =
      p.attn_part + (((size_t)layer * p.B + b) * p.Hkv + g) * p.max_chunks * (size_t)PS;
  float4* gsum = reinterpret_cast<float4*>(sm.scratch);   // [nCG][GH / 4] group sums
  float* osm = reinterpret_cast<float*>(gsum + 256);      // [G][hd]
  float* msm = osm + kMaxAttnOut;                         // [nc][G] chunk maxima
  float* lsm = msm + p.max_chunks * G;                    // [nc][G] chunk sums
  float* wsm = lsm + p.max_chunks * G;                    // [nc][G] merge weights
  float* ML = wsm + p.max_chunks * G;                     // [2][G]
  for (int t = ct; t < nc * G; t += 256) {
    const float* pp = parts + (size_t)(t / G) * PS + GH;
    msm[t] = __ldcg(pp + t % G);
    lsm[t] = __ldcg(pp + G + t % G);
  }
  cbar();
  if (cw < G) {
    const int h = cw;
    float M = -1e30f;
    for (int ch = lane; ch < nc; ch += 32) M = fmaxf(M, msm[ch * G + h]);
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, o));
    float Ls = 0.f;
    for (int ch = lane; ch < nc; ch += 32) Ls += ex2(msm[ch * G + h] - M) * lsm[ch * G + h];
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(FULL, Ls, o);
    if (lane == 0) {
      ML[h] = M;
      ML[G + h] = frcp(Ls);
    }
  }
  cbar();
  for (int t = ct; t < nc * G; t += 256) wsm[t] = ex2(msm[t] - ML[t % G]) * ML[G + t % G];
  cbar();
  // thread (group cg, float4 column c4) sums chunks cg, cg + nCG, ... of its
  // four outputs with eight loads in flight; the groups are added in cg order
  const int C4 = GH / 4, nCG = 256 / C4;
  if (ct < nCG * C4) {
    const int cg = ct / C4, c4 = ct - cg * C4, h = (4 * c4) / hd;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int ch0 = cg; ch0 < nc; ch0 += 8 * nCG) {
      float4 v[8];
      float w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int ch = ch0 + j * nCG;
        const bool on = ch < nc;
        v[j] = on ? __ldcg(reinterpret_cast<const float4*>(parts + (size_t)ch * PS) + c4)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
        w[j] = on ? wsm[ch * G + h] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        acc.x = fmaf(w[j], v[j].x, acc.x);
        acc.y = fmaf(w[j], v[j].y, acc.y);
        acc.z = fmaf(w[j], v[j].z, acc.z);
        acc.w = fmaf(w[j], v[j].w, acc.w);
      }
    }
    gsum[cg * C4 + c4] = acc;
  }
  cbar();
#pragma unroll 1
  for (int c4 = ct; c4 < C4; c4 += 256) {
    float4 o = gsum[c4];
#pragma unroll 1
    for (int cg = 1; cg < nCG; ++cg) {
      const float4 v = gsum[cg * C4 + c4];
      o.x += v.x;
      o.y += v.y;
      o.z += v.z;
      o.w += v.w;
    }
    reinterpret_cast<float4*>(osm)[c4] = o;
  }
  cbar();
  write_attn_out(p, layer, b, g, osm);
}

// RoPE cos/sin of this step's positions (angle in double: a 262144-token
// position loses ~0.03 rad in fp32), plus the position check.  Runs once per
// step.
__device__ __forceinline__ void rope_table(const Params& p, int task) {
  MK_CONSUMER_IDS;
  const int half = p.hd / 2;
  for (int t = ct; t < p.B * half; t += 256) {
    const int bb = t / half, i = t % half;
    const int pos = __ldg(p.positions + bb);
    const int sl = __ldg(p.seq_lens + bb);
    if (i == 0) {
      // positions == seq_lens, except in a prefill group: entry bb's
      // position may exceed its length by g when entries bb - g .. bb - 1
      // carry the sequence's previous tokens (same length, consecutive
      // positions); greedy steps advance every entry alone, so none there
      const int g = pos - sl;
      const bool ok = g == 0 || (g > 0 && g <= bb && p.g_pos == nullptr &&
                                 __ldg(p.seq_lens + bb - 1) == sl &&
                                 __ldg(p.positions + bb - 1) == pos - 1);
      if (!ok) raise_error(p, MK_ERR_DEVICE, task, OP_RN, -1, pos, sl, 5);
    }
    double sv, cv;
    sincos((double)pos * p.inv_freq[i], &sv, &cv);
    p.cs[(size_t)bb * p.hd + i] = (float)cv;
    p.cs[(size_t)bb * p.hd + half + i] = (float)sv;
  }
}

// Fused residual add + RMSNorm statistics for one 64-column tile of level l:
// x_l = x_{l-1} + sum_g o_part[g] + sum_j moe_part[j] (fixed order), the
// gamma-scaled rows the next projections read, and the tile's sum of squares
// per token (1/rms is applied by the readers).  The partials are staged
// through shared memory in rounds so that all loads of a round are in flight
// at once.
//
// A level that feeds a layer also adds the tile's share of that layer's
// router logits, sum over the tile's 64 columns c of W_r[e][c] (gamma x)[b][c],
// and the tile's sum of squares into the layer's fixed-point accumulators
// (racc, ssacc).  The producer streams the tile's router columns into the
// ring when it hands the task out (128 expert rows of 128 bytes per stage,
// 128-byte swizzled), so they are resident before the inputs are.  Returns
// the advanced ring counter.
__device__ __forceinline__ uint32_t rn_task(const Params& p, const int32_t* ent, uint32_t stage_ctr) {
  const Smem sm = smem_view(p);
  MK_CONSUMER_IDS;
  const int l = ent[D_LAYER], r = ent[D_A];
  const int B = p.B, d = p.d, per = B * 64;
  float* xs = reinterpret_cast<float*>(sm.scratch);  // [B][64]
  float* stage = xs + kMaxBatch * 64;                 // [kRnStage] staged partials
  const int nparts = (l == 0) ? 1 : 1 + p.Hkv + p.k;
  const int nst = ent[32 + R_NSTAGE];   // router stages (0 for the final norm)
  // this thread's gamma column (every element it owns is column ct % 64)
  const float gam =
      __uint_as_float((uint32_t)__ldg(norm_w(sm, l) + r * 64 + (ct & 63)) << 16);
  if (l == 0) {
    // the embedding rows of this step's tokens
#pragma unroll 1
    for (int e = ct; e < per; e += 256) {
      const int b = e >> 6;
      int tok = __ldg(p.tokens + b);
      if (tok < 0 || tok >= p.V) {
        if ((e & 63) == 0) raise_error(p, MK_ERR_DEVICE, ent[32 + R_TASK], OP_RN, -1, tok, p.V, 4);
        tok = 0;
      }
      xs[e] = __uint_as_float((uint32_t)__ldg(p.embed + (size_t)tok * d + r * 64 + (e & 63)) << 16);
    }
  } else {
    // part j of the sum (x_{l-1}, then the O-proj partial of each KV group,
    // then the expert partial of each rank), at this tile's first column
    const float** pp = reinterpret_cast<const float**>(stage + kRnStage) - kMaxParts;
    if (ct < nparts) {
      const int j = ct;
      const size_t lb = (size_t)(l - 1);
      const float* src = j == 0 ? p.x + lb * B * d
                         : j <= p.Hkv ? p.o_part + (lb * p.Hkv + (j - 1)) * B * d
                                      : p.moe_part + (lb * p.k + (j - 1 - p.Hkv)) * B * d;
      pp[j] = src + r * 64;
    }
    cbar();
    // thread (group jg, float4 column e4) sums parts jg, jg + nJ, ... with
    // eight loads in flight; the groups' sums are then added in jg order
    const int per4 = B * 16, nJ = 256 / per4;
    float4* grp = reinterpret_cast<float4*>(stage);   // [nJ][per4]
    if (ct < nJ * per4) {
      const int jg = ct / per4, e4 = ct - jg * per4;
      const size_t off = (size_t)(e4 >> 4) * d + 4 * (e4 & 15);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
      for (int j0 = jg; j0 < nparts; j0 += 8 * nJ) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = j0 + i * nJ;
          v[i] = j < nparts ? __ldcg(reinterpret_cast<const float4*>(pp[j] + off))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acc.x += v[i].x;
          acc.y += v[i].y;
          acc.z += v[i].z;
          acc.w += v[i].w;
        }
      }
      grp[jg * per4 + e4] = acc;
    }
    cbar();
#pragma unroll 1
    for (int e4 = ct; e4 < per4; e4 += 256) {
      float4 x = grp[e4];
#pragma unroll 1
      for (int g = 1; g < nJ; ++g) {
        const float4 v = grp[g * per4 + e4];
        x.x += v.x;
        x.y += v.y;
        x.z += v.z;
        x.w += v.w;
      }
      reinterpret_cast<float4*>(xs)[e4] = x;
    }
  }
  cbar();
  if (ct == 0) cstamp(p, ent[32 + R_TASK], T_K2);   // residual rows summed
  float* rows = reinterpret_cast<float*>(p.actA + (size_t)l * p.actA_bytes);
  float* gxs = stage;   // [B][64] gamma x of the tile (the staging area is free)
#pragma unroll 1
  for (int e = ct; e < per; e += 256) {
    const int b = e >> 6, col = r * 64 + (e & 63);
    const float x = xs[e];
    const float gx = x * gam;
    p.x[((size_t)l * B + b) * d + col] = x;
    rows[(size_t)b * (d + kActPad) + col] = gx;
    gxs[e] = gx;
  }
  if (cw < B) {
    const float x0 = xs[cw * 64 + lane], x1 = xs[cw * 64 + 32 + lane];
    float ss = x0 * x0 + x1 * x1;
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
    if (lane == 0) {
      reinterpret_cast<float*>(p.actA + (size_t)l * p.actA_bytes + p.actA_rows_bytes)[r * B + cw] = ss;
      if (l < p.L) red_add_u64(p.ssacc + ((size_t)(p.epoch & 1u) * p.L + l) * B + cw, to_fixed(ss));
    }
  }
  if (l == 0 && r == 0) rope_table(p, ent[32 + R_TASK]);
  if (nst == 0) return stage_ctr;
  cbar();
  if (ct == 0) cstamp(p, ent[32 + R_TASK], T_K3);   // outputs written
  unsigned long long* out = p.racc + ((size_t)(p.epoch & 1u) * p.L + l) * B * p.E;
  // thread pair per expert row: half hf takes columns 32 hf .. 32 hf + 31
  // (four 16-byte units, four independent FMA chains); the pair adds its two
  // sums by one shuffle and half hf adds the tokens b with b % 2 == hf into
  // the layer's fixed-point logit accumulators
#pragma unroll 1
  for (int s = 0; s < nst; ++s) {
    const uint32_t slot = stage_ctr % (uint32_t)sm.NS, ph = (stage_ctr / (uint32_t)sm.NS) & 1u;
    wait_bar(p, sm.full(slot), ph, 404);
    const uint8_t* wt = sm.ring + (size_t)slot * kStageBytes;
    const int e0 = kRouterRowsPerStage * s;
    const int rows = min(kRouterRowsPerStage, p.E - e0);   // expert rows in this stage
    const int el = ct >> 1, hf = ct & 1;
    const bool valid = el < rows;                          // warp-uniform when rows % 16 == 0
    float wf[32];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 w = valid ? *reinterpret_cast<const uint4*>(
                                  wt + el * 128 + (((4 * hf + k) ^ (el & 7)) << 4))
                            : make_uint4(0u, 0u, 0u, 0u);
      wf[8 * k + 0] = lo_bf16(w.x);
      wf[8 * k + 1] = hi_bf16(w.x);
      wf[8 * k + 2] = lo_bf16(w.y);
      wf[8 * k + 3] = hi_bf16(w.y);
      wf[8 * k + 4] = lo_bf16(w.z);
      wf[8 * k + 5] = hi_bf16(w.z);
      wf[8 * k + 6] = lo_bf16(w.w);
      wf[8 * k + 7] = hi_bf16(w.w);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.empty(slot));
    ++stage_ctr;
#pragma unroll 1
    for (int b = 0; b < B; ++b) {   // uniform: every lane takes part in the shuffle
      const float4* g = reinterpret_cast<const float4*>(gxs + b * 64 + 32 * hf);
      float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 v = g[k];
        a[k & 3] = fmaf(wf[4 * k + 0], v.x, a[k & 3]);
        a[k & 3] = fmaf(wf[4 * k + 1], v.y, a[k & 3]);
        a[k & 3] = fmaf(wf[4 * k + 2], v.z, a[k & 3]);
        a[k & 3] = fmaf(wf[4 * k + 3], v.w, a[k & 3]);
      }
      float sum = (a[0] + a[1]) + (a[2] + a[3]);
      sum += __shfl_xor_sync(FULL, sum, 1);
      if (valid && (b & 1) == hf) red_add_u64(out + (size_t)b * p.E + e0 + el, to_fixed(sum));
    }
  }
  if (ct == 0) cstamp(p, ent[32 + R_TASK], T_K4);   // router shares written
  return stage_ctr;
}

// The top-k task of layer l: every token's router logits, top-k and softmax
// (warp b takes token b) and the layer's routing table in global memory,
// read by the expert tiles' producers (at batch sizes where they do not
// route locally) and by the debug reads.  It also stands in for the signals
// of the unused slots' tiles and zeroes the other step parity's accumulators
// of the layer for the next step.
__device__ __forceinline__ void topk_task(const Params& p, int l) {
  const Smem sm = smem_view(p);
  MK_CONSUMER_IDS;
  const int B = p.B, E = p.E, S = p.S, NR = p.NR;
  const uint32_t par = p.epoch & 1u;
  int32_t* sel = reinterpret_cast<int32_t*>(sm.scratch);   // [8][8]
  float* wsel = reinterpret_cast<float*>(sel + 64);          // [8][8]
  uint32_t* mask = reinterpret_cast<uint32_t*>(wsel + 64);   // [kRouteMaskWords]
  int* n_used_s = reinterpret_cast<int*>(mask + kRouteMaskWords);
  if (cw < B)
    token_route(p, router_b(p, sm, l), l, par, cw, sel + cw * 8, wsel + cw * 8,
                p.rlogits + ((size_t)l * B + cw) * E);
  cbar();
  if (cw == 0) {
    const int nu = compact_routes(p, sel, wsel, mask, p.route + (size_t)l * p.route_words);
    if (lane == 0) *n_used_s = nu;
  }
  cbar();
  const int n_used = *n_used_s;
  // The producers drop the tiles of unused slots; stand in for the signals
  // those tiles would have sent: each down-tile row counter gets one per
  // unused slot, each unused slot's counter its n_ff gate/up tiles (so every
  // counter still gets its per-step arrival count).
  if (n_used < S) {
    for (int r = ct; r < NR; r += 256)
      atomicAdd(p.counters + p.dt_ctr0 + l * NR + r, (uint32_t)(S - n_used));
    for (int j = n_used + ct; j < S; j += 256)
      atomicAdd(p.counters + p.slot_ctr0 + l * S + j, (uint32_t)p.n_ff);
  }
  // the next step accumulates into the other parity: start it at zero (this
  // step's norm tiles only touch parity par)
  const size_t lo = ((size_t)(par ^ 1u) * p.L + l) * B;
  for (int i = ct; i < B * E; i += 256) p.racc[lo * E + i] = 0ull;
  if (ct < B) p.ssacc[lo + ct] = 0ull;
}

// NBK: the GEMV path (1 and 2: FFMA for 1 or 2 tokens; 3: mma.sync for 3..8);
// HD: the head dimension.  Each launch runs the instantiation of its batch and
// shape, so its consumer code holds one GEMV path and one attention routine.
template <int NBK, int HD>
__device__ __forceinline__ void consumer_loop(const Params& p) {
  const Smem sm = smem_view(p);
  MK_CONSUMER_IDS;
  uint32_t stage_ctr = 0, ngemv = 0;
  int curA = -1, nloadA = 0, nloadB = 0, bufA = 0;
  const int nA = p.nA;
  const int PC = p.part_cols;
  float* part0 = reinterpret_cast<float*>(sm.epi);
  float* rstd_ring = part0 + 2 * kConsumerWarps * 16 * PC;
  for (int i = 0;; ++i) {
    const int e = i % kFifo;
    // Each warp runs the FIFO on its own through GEMV tiles (no barrier);
    // leaving the loop, and entering a task with internal barriers, goes
    // through one agreement among all consumer warps.
    const bool ok = __all_sync(FULL, wait_bar(p, sm.ready(e), (i / kFifo) & 1, 500));
    if (!ok) {
      cbar_or(1);
      break;
    }
    const int32_t* ent = sm.fifo + e * kFifoEntryWords;
    const int op = ent[D_OP];
    if (op == OP_NONE) {
      if (ct == 0) mbar_arrive(sm.done(e));
      cbar_or(1);
      break;
    }
    const bool gemv = is_gemv(op);
    if (!gemv && cbar_or(aborted())) break;
    const int t = ent[32 + R_TASK];
    if (ct == 0) {
      stamp(p, t, T_C_READY);
      cstamp(p, t, T_K0);
    }
    const int act = ent[D_ACT];
    const int layer = ent[D_LAYER];
    if (act == ACT_A && layer != curA) {
      // a new level: this warp is done with the previous level's buffer
      if (curA >= 0 && lane == 0) mbar_arrive(sm.aemptyA(bufA));
      bufA = nloadA % nA;
      wait_bar(p, sm.afullA(bufA), (uint32_t)((nloadA / nA) & 1), 501);
      ++nloadA;
      curA = layer;
      if (cw < p.B) {
        // 1/rms of token cw from the level's sum-of-squares partials, once
        // per level; the epilogue warp reads it after this warp's pfull
        const float* ss = reinterpret_cast<const float*>(sm.actA + (size_t)bufA * p.actA_stride +
                                                         p.actA_rows_bytes);
        float acc = 0.f;
        for (int r = lane; r < p.NR; r += 32) acc += ss[r * p.B + cw];
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
        if (lane == 0) rstd_ring[(layer & (kRstdRing - 1)) * kMaxBatch + cw] =
            frsqrt(acc / (float)p.d + p.eps);
      }
    }
    const int bufB = nloadB & 1;
    if (act == ACT_B) {
      wait_bar(p, sm.afullB(bufB), (uint32_t)((nloadB >> 1) & 1), 502);
      ++nloadB;
    }
    if (ct == 0) {
      stamp(p, t, T_C_ACT);
      cstamp(p, t, T_K1);
    }
    const uint8_t* actA = sm.actA + (size_t)bufA * p.actA_stride;
    const uint8_t* actB = sm.actB + (size_t)bufB * p.actB_bytes;

    if (gemv) {
      const int pb = (int)(ngemv & 1u);
      const uint32_t pe_par = ((ngemv >> 1) & 1u) ^ 1u;
      float* pw = part0 + (pb * kConsumerWarps + cw) * 16 * PC;
      const float* a;
      int stride, ncols = p.B;
      const int32_t* tokmap = nullptr;
      if (op == OP_GATEUP || op == OP_DOWN) ncols = ent[32 + R_NTOK];
      if (op == OP_OPROJ) {
        a = reinterpret_cast<const float*>(actB);
        stride = p.G * p.hd + kActPad;
      } else if (op == OP_DOWN) {
        a = reinterpret_cast<const float*>(actB);
        stride = p.F + kActPad;
      } else {
        a = reinterpret_cast<const float*>(actA);
        stride = p.d + kActPad;
        if (op == OP_GATEUP) tokmap = ent + 32 + R_TOK;
      }
      stage_ctr = gemv_consume<NBK>(p, ent, a, stride, tokmap, ncols, pw, sm.pempty(pb), pe_par,
                               stage_ctr);
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.pfull(pb));
      ++ngemv;
      continue;   // the epilogue warp completes the task
    }

    switch (op) {
      case OP_RN:
        stage_ctr = rn_task(p, ent, stage_ctr);
        break;
      case OP_TOPK:
        topk_task(p, layer);
        break;
      default:  // OP_ATTN
        stage_ctr = attn_task<HD>(p, ent, actB, stage_ctr);
        if (ent[D_FLAGS] & F_COMBINE) {
          // the chunk that completes (b, g) merges all its chunks' partials
          cbar();
          int last = 0;
          if (ct == 0) {
            const uint32_t old = atom_add_acq_rel(p.counters + ent[D_X0], 1u);
            last = old + 1u == p.epoch * (uint32_t)ent[D_X1];
          }
          if (cbar_or(last)) {
            combine_task(p, ent);
            cbar();
            if (ct == 0) red_release_add(p.counters + ent[D_X2], 1u);
          }
        }
        break;
    }
    cbar();
    if (ct == 0) {
      stamp(p, t, T_C_END);
      cstamp(p, t, T_K5);
      if (act == ACT_B) mbar_arrive(sm.aemptyB(bufB));
      mbar_arrive(sm.done(e));
    }
  }
}

// ============================================================== epilogue ==
// One warp follows the FIFO behind the consumers.  For a GEMV tile it waits
// for the consumer warps' partials, reduces them, writes the outputs and
// completes the task (partials buffer, B activation buffer, done); every
// entry it passes is released to the producer together with the signaler.
__device__ __forceinline__ void epilogue_loop(const Params& p) {
  const Smem sm = smem_view(p);
  const int lane = threadIdx.x & 31;
  const int PC = p.part_cols;
  const float* part0 = reinterpret_cast<const float*>(sm.epi);
  const float* rstd_ring = part0 + 2 * kConsumerWarps * 16 * PC;
  const EpiParams ep(p);
  uint32_t ngemv = 0;
  int nloadB = 0;
  for (int i = 0;; ++i) {
    const int e = i % kFifo;
    if (!warp_wait(p, sm.ready(e), (i / kFifo) & 1, 600)) break;
    const int32_t* ent = sm.fifo + e * kFifoEntryWords;
    const int op = ent[D_OP];
    if (op == OP_NONE) break;
    const int act = ent[D_ACT];
    if (!is_gemv(op)) {
      if (act == ACT_B) ++nloadB;
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.fempty(e));
      continue;
    }
    const int pb = (int)(ngemv & 1u);
    if (!warp_wait(p, sm.pfull(pb), (ngemv >> 1) & 1u, 601)) break;
    const int t = ent[32 + R_TASK];
    if (lane == 0) cstamp(p, t, T_K4);
    const float* part = part0 + pb * kConsumerWarps * 16 * PC;
    const float* rs = rstd_ring + (ent[D_LAYER] & (kRstdRing - 1)) * kMaxBatch;
    if (op == OP_LMHEAD) {
      lm_epilogue(ep, p, ent, part, rs);
      if (ent[D_FLAGS] & F_ARGMAX) lm_finish(p, ent);
    } else {
      gemv_epilogue(ep, ent, part, rs);
    }
    __syncwarp();
    if (lane == 0) {
      stamp(p, t, T_C_END);
      cstamp(p, t, T_K5);
      mbar_arrive(sm.pempty(pb));
      if (act == ACT_B) mbar_arrive(sm.aemptyB(nloadB & 1));
      mbar_arrive(sm.done(e));
      mbar_arrive(sm.fempty(e));
    }
    __syncwarp();
    if (act == ACT_B) ++nloadB;
    ++ngemv;
  }
}

template <int NBK, int HD>
__global__ void __launch_bounds__(kThreads, 1) mk_interp(const __grid_constant__ Params p) {
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    const Smem sm = smem_view(p);
    g_abort = 0;
    for (int s = 0; s < sm.NS; ++s) {
      mbar_init(sm.full(s), 1);
      mbar_init(sm.empty(s), kConsumerWarps);
    }
    for (int e = 0; e < kFifo; ++e) {
      mbar_init(sm.posted(e), 1);
      mbar_init(sm.ready(e), 1);
      mbar_init(sm.done(e), 1);
      mbar_init(sm.fempty(e), 2);   // signaler + epilogue warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sm.afullA(b), 1);
      mbar_init(sm.aemptyA(b), kConsumerWarps);
      mbar_init(sm.afullB(b), 1);
      mbar_init(sm.aemptyB(b), 1);
      mbar_init(sm.pfull(b), kConsumerWarps);
      mbar_init(sm.pempty(b), 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  {
    const Smem sm = smem_view(p);
    const void** tab = const_cast<const void**>(sm.ptrs);
    const int L = p.L;
    for (int i = threadIdx.x; i < ptr_table_words(L); i += kThreads) {
      const void* v;
      if (i < L) v = p.attn_norm[i];
      else if (i == L) v = p.final_norm;
      else if (i < 2 * L + 1) v = p.router_bias ? p.router_bias[i - L - 1] : nullptr;
      else if (i < 3 * L + 1) v = p.k_pool[i - 2 * L - 1];
      else v = p.v_pool[i - 3 * L - 1];
      tab[i] = v;
    }
  }
  __syncthreads();
  if (warp < kFirstConsumerWarp) {
    // warpgroup 0 releases registers first; each consumer warpgroup's
    // increase waits until the CTA's pool holds them
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRoleRegs));
    if (warp == kProducerWarp) {
      producer_loop(p);
    } else if (warp == kLoaderWarp) {
      loader_loop(p);
    } else if (warp == kSignalWarp) {
      signal_loop(p);
    } else {
      epilogue_loop(p);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsumerRegs));
    consumer_loop<NBK, HD>(p);
  }
  __syncthreads();
}

}  // namespace

// Launch one step (or one phase) of the interpreter: cooperative, so that all
// CTAs are guaranteed co-resident (the counter waits and the dispenser rely
// on it).
namespace {
// the kernel instantiation for a batch size and head dimension, and the
// dynamic shared memory it was last configured for
// (the attribute is per device: the cache holds one entry per device ordinal)
constexpr int kMaxDevices = 64;
struct KernelSlot {
  const void* fn;
  int configured_bytes[kMaxDevices];   // 0: not configured on that device yet
};
KernelSlot g_kernels[3][2] = {
    {{reinterpret_cast<const void*>(mk_interp<1, 64>), {}},
     {reinterpret_cast<const void*>(mk_interp<1, 128>), {}}},
    {{reinterpret_cast<const void*>(mk_interp<2, 64>), {}},
     {reinterpret_cast<const void*>(mk_interp<2, 128>), {}}},
    {{reinterpret_cast<const void*>(mk_interp<3, 64>), {}},
     {reinterpret_cast<const void*>(mk_interp<3, 128>), {}}}};
// the cache entry of the current device, or null past kMaxDevices
int* configured_entry(KernelSlot& k) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  return &k.configured_bytes[dev];
}
KernelSlot& kernel_for(int B, int hd) {
  return g_kernels[B <= 1 ? 0 : (B == 2 ? 1 : 2)][hd == 128 ? 1 : 0];
}
}  // namespace

cudaError_t launch_interp(const Params& p, int grid, cudaStream_t stream) {
  KernelSlot& k = kernel_for(p.B, p.hd);
  int* conf = configured_entry(k);
  if (!conf || *conf != p.smem_bytes) {
    // the register split needs the registers it hands out: a build whose
    // launch holds fewer would leave the consumers' increase waiting forever,
    // so it is refused here instead of launched
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, k.fn);
    if (e != cudaSuccess) return e;
    if (attr.numRegs * kThreads < 128 * kRoleRegs + 256 * kConsumerRegs)
      return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
    if (e != cudaSuccess) return e;
    if (conf) *conf = p.smem_bytes;
  }
  void* args[] = {const_cast<Params*>(&p)};
  return cudaLaunchCooperativeKernel(k.fn, dim3(grid), dim3(kThreads), args, (size_t)p.smem_bytes,
                                     stream);
}

// Co-resident CTAs per SM at this shared-memory size; every instantiation is
// checked, as each carries its own register count.
cudaError_t max_coresident(int smem_bytes, int* blocks_per_sm) {
  int best = 1 << 30;
  for (auto& row : g_kernels) {
    for (KernelSlot& k : row) {
      cudaError_t e =
          cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
      if (e != cudaSuccess) return e;
      if (int* conf = configured_entry(k)) *conf = smem_bytes;
      int n = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k.fn, kThreads, (size_t)smem_bytes);
      if (e != cudaSuccess) return e;
      best = n < best ? n : best;
    }
  }
  *blocks_per_sm = best;
  return cudaSuccess;
}

}  // namespace mk
