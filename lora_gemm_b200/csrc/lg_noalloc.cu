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
// the device address is looked up once per device with cudaGetSymbolAddress
// (with that device current) on the first call made on the device, and that
// address is what the kernels receive.
#include <mutex>

#include "../../include/lora_gemm.h"

// Receives the bf16 copies of A_cat and B_cat.  Each call overwrites the part
// it uses before reading it, so nothing in it has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LG_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr size_t kScratchBytes = LG_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Device address of the scratch array on the current device (cached per device).
lg_status scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LG_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return LG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return LG_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return LG_OK;
}

}  // namespace

extern "C" lg_status lg_lora_linear_noalloc(const void* x, const void* W, const float* A_cat, const float* B_cat,
                                            void* y, int64_t M, int K, int N, int R, void* stream) {
  const size_t need = lg_lora_linear_workspace_size(M, K, N, R);
  if (need > kScratchBytes) return LG_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const lg_status st = scratch_address(&scratch);
    if (st != LG_OK) return st;
  }
  // Same validation, kernels and launch configuration as lg_lora_linear; only
  // the workspace is the built-in array.
  return lg_lora_linear(x, W, A_cat, B_cat, y, M, K, N, R, scratch, need > 0 ? kScratchBytes : 0, stream);
}
