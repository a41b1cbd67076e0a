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
//
// The lookup is what loads this file's device module, and with it the array,
// when modules load lazily.  mk_create therefore does the lookup (it
// allocates anyway), so the array is reserved when a context is created on
// the device, and mk_decode_step_static itself loads and allocates nothing.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "mk.h"
#include "mk_internal.h"

namespace mk {
int ctx_device(const mk_ctx* c);
mk_status static_scratch_setup(int device);
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

// The device address of g_step_scratch on `device` if it was looked up.
bool scratch_address(int device, void** out) {
  std::lock_guard<std::mutex> lock(g_addr_mu);
  auto it = g_addr.find(device);
  if (it == g_addr.end()) return false;
  *out = it->second;
  return true;
}

}  // namespace

// Looks up g_step_scratch's address on `device` (which must be current) once
// and caches it.  Called by mk_create.  A failed lookup (for example no room
// left for the array) is cleared from the runtime's error state and reported.
mk_status mk::static_scratch_setup(int device) {
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (g_addr.count(device)) return MK_OK;
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_step_scratch);
  if (e != cudaSuccess || ptr == nullptr) {
    (void)cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? MK_ERR_OOM : MK_ERR_CUDA;
  }
  g_addr.emplace(device, ptr);
  return MK_OK;
}

extern "C" mk_status mk_decode_step_static(mk_ctx* ctx, const int32_t* tokens,
                                           const int32_t* positions, const int32_t* page_table,
                                           const int32_t* seq_lens, float* logits, void* stream) {
  if (!ctx) return MK_ERR_INVALID;
  const int device = mk::ctx_device(ctx);
  void* scratch = nullptr;
  // looked up by mk_create on this device; absent only if that lookup failed
  if (!scratch_address(device, &scratch)) return MK_ERR_CUDA;
  if (cudaSetDevice(device) != cudaSuccess) return MK_ERR_CUDA;
  return mk::launch_step_in(ctx, tokens, positions, page_table, seq_lens, logits, stream,
                            scratch, kStaticScratchBytes);
}
