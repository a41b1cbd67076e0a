// mk_static.cu -- the decode step with its per-step scratch in a fixed,
// file-scope device array, for callers that must not allocate device memory.
//
// The step's scratch (counters, routing words, residual rows, projection
// outputs, attention partials, expert activations and partial outputs) is
// normally allocated by mk_build_schedule.  Here it is carved out of one
// statically sized __device__ array instead, so a call allocates nothing.
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so the array's device address is looked up once
// per device with cudaGetSymbolAddress and then passed to the kernel.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "mk.h"
#include "mk_internal.h"

namespace mk {
int ctx_device(const mk_ctx* c);
mk_status launch_step_in(mk_ctx* c, const int32_t* tokens, const int32_t* positions,
                         const int32_t* page_table, const int32_t* seq_lens, float* logits,
                         void* stream, void* scratch, size_t cap);
}  // namespace mk

namespace {

// 32 MiB: enough for the 30B-MoE shape (48 layers, d_model 2048, 128 experts
// top-8) at batch 1 with any context length, and for small models at batch 8.
// Every device that loads this library reserves it until the process exits.
constexpr size_t kStaticScratchBytes = size_t(MK_STATIC_SCRATCH_MAX_BYTES);

static __device__ __align__(256) unsigned char g_step_scratch[kStaticScratchBytes];

std::mutex g_addr_mu;
std::unordered_map<int, void*> g_addr;   // device ordinal -> g_step_scratch on it

// Device address of g_step_scratch on `device`, which must be current.
mk_status scratch_address(int device, void** out) {
  std::lock_guard<std::mutex> lock(g_addr_mu);
  auto it = g_addr.find(device);
  if (it != g_addr.end()) {
    *out = it->second;
    return MK_OK;
  }
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_step_scratch) != cudaSuccess || ptr == nullptr)
    return MK_ERR_CUDA;
  g_addr.emplace(device, ptr);
  *out = ptr;
  return MK_OK;
}

}  // namespace

extern "C" mk_status mk_decode_step_static(mk_ctx* ctx, const int32_t* tokens,
                                           const int32_t* positions, const int32_t* page_table,
                                           const int32_t* seq_lens, float* logits, void* stream) {
  if (!ctx) return MK_ERR_INVALID;
  const int device = mk::ctx_device(ctx);
  if (cudaSetDevice(device) != cudaSuccess) return MK_ERR_CUDA;
  void* scratch = nullptr;
  const mk_status st = scratch_address(device, &scratch);
  if (st != MK_OK) return st;
  return mk::launch_step_in(ctx, tokens, positions, page_table, seq_lens, logits, stream,
                            scratch, kStaticScratchBytes);
}
