// lg_lora_linear_noalloc: the merged-LoRA linear layer for callers that have
// no way to allocate device memory at the point of the call -- for example a
// plugin inside an inference engine whose device memory is planned before the
// run and which may not allocate when it is enqueued, or a serving loop that
// must never call cudaMalloc because it synchronizes the device and stalls
// every other stream.  Such a caller cannot provide lg_lora_linear's
// workspace, so this entry point keeps the bf16 copies of the merged factors
// in a fixed array that is part of the library's device image instead.
//
// The array is a file-scope static __device__ variable: every GPU on which
// the library's kernels are loaded holds LG_NOALLOC_SCRATCH_BYTES of it until
// the process exits.  In host code its name is only a host-side stand-in, so
// its device address is looked up with cudaGetSymbolAddress (with the device
// current) on the first call made on a device, and that address is what the
// kernels receive.  The address belongs to the CUDA context the lookup ran
// in: the cache is keyed on the device and the context's id, so a call made
// after the context was destroyed and recreated (cudaDeviceReset), or under a
// different context, looks the address up again.
#include <mutex>

#include "../../include/lora_gemm.h"
#include "lg_internal.h"

// Receives the bf16 copies of A_cat and B_cat.  Each call overwrites the part
// it uses before reading it, so nothing in it has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LG_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr size_t kScratchBytes = LG_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

struct Slot {
  bool valid = false;
  unsigned long long context = 0;
  void* addr = nullptr;
};

// Device address of the scratch array in the current context.
lg_status scratch_address(void** out) {
  static std::mutex mu;
  static Slot slots[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LG_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return LG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  Slot& slot = slots[dev];
  unsigned long long ctx = 0;
  if (lg::current_context_id(&ctx) && slot.valid && slot.context == ctx) {
    *out = slot.addr;
    return LG_OK;
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return LG_ERR_CUDA;
  }
  // The lookup made the runtime's context current if none was: ask again.
  slot.valid = lg::current_context_id(&ctx);
  slot.context = ctx;
  slot.addr = p;
  *out = p;
  return LG_OK;
}

}  // namespace

extern "C" lg_status lg_lora_linear_noalloc(const void* x, const void* W, const float* A_cat, const float* B_cat,
                                            void* y, int64_t M, int K, int N, int R, void* stream) {
  // lg_lora_linear's own checks first, so that both entry points give the
  // same status for the same bad argument; only then the scratch limit.
  const lg_status st = (lg_status)lg::check_lora_linear(x, W, A_cat, B_cat, y, M, K, N, R);
  if (st != LG_OK) return st;
  const size_t need = lg_lora_linear_workspace_size(M, K, N, R);
  if (need > kScratchBytes) return LG_ERR_WORKSPACE;
  if (M == 0) return LG_OK;
  void* scratch = nullptr;
  if (need > 0) {
    const lg_status sa = scratch_address(&scratch);
    if (sa != LG_OK) return sa;
  }
  // Same kernels and launch configuration as lg_lora_linear; only the
  // workspace is the built-in array.
  return lg_lora_linear(x, W, A_cat, B_cat, y, M, K, N, R, scratch, need > 0 ? kScratchBytes : 0, stream);
}
