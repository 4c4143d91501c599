// Internal host-side interface between the C ABI layer (lg_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lg {

constexpr int kMaxAdapters = 8;

struct MergeAParams {
  const float* A[kMaxAdapters];
  float scale[kMaxAdapters];
  int row_off[kMaxAdapters + 1];  // prefix sums of the ranks
  int n_adapters;
  int d_in;
};

struct MergeBParams {
  const float* B[kMaxAdapters];
  int col_off[kMaxAdapters + 1];
  int n_adapters;
  int d_out;
};

// Grid size for a grid-stride elementwise kernel over `work` items.
int elementwise_grid(int64_t work, int sm_count);

cudaError_t launch_philox_u32(uint32_t* out, int64_t n_blocks, uint64_t seed, uint64_t block_offset, int sm_count,
                              cudaStream_t s);
cudaError_t launch_philox_normal(float* eps, int64_t n, uint64_t seed, uint64_t offset, int sm_count,
                                 cudaStream_t s);
cudaError_t launch_renoise(const float* up, float* x, int64_t n, float sigma, uint64_t seed, uint64_t offset,
                           int sm_count, cudaStream_t s);
cudaError_t launch_euler(float* x, const float* v, int64_t n, float dt, int sm_count, cudaStream_t s);
cudaError_t launch_merge(const MergeAParams& pa, const MergeBParams& pb, float* A_cat, float* B_cat, int sm_count,
                         cudaStream_t s);
// FP32 -> bf16 (RNE) of A_cat [R, K] and B_cat [N, R] into dstA / dstB.
cudaError_t launch_prep_bf16(const float* A_cat, const float* B_cat, uint16_t* dstA, uint16_t* dstB,
                             int64_t nA, int64_t nB, int sm_count, cudaStream_t s);

// MXFP8 quantization of bf16 rows [rows, K] along K (K % 128 == 0): E4M3
// codes [rows, K] and E8M0 scales in the 128 x 128 blocked layout.
cudaError_t launch_mx_quantize(const uint16_t* in, int64_t rows, int K, uint8_t* codes, uint8_t* scales,
                               int sm_count, cudaStream_t s);

// Merged-LoRA linear (tcgen05 kernel).  Factors already in bf16.
struct LinearLaunch {
  const void* x;
  const void* W;
  const uint16_t* A_bf16;  // [R, K]
  const uint16_t* B_bf16;  // [N, R]
  void* y;
  int64_t M;
  int K, N, R;
  int sm_count;
  uint64_t wait_limit_ns;
  // MXFP8 base term (lg_lora_linear_mxfp8): E4M3 codes and blocked E8M0
  // scales of x [M, K] and W [N, K]; x above stays the bf16 activations (the
  // LoRA path reads them), W is unused.
  bool mx = false;
  const void* xq = nullptr;
  const void* xsf = nullptr;
  const void* wq = nullptr;
  const void* wsf = nullptr;
  // Fused SwiGLU (MXFP8 only): N = 2 ffn (gate rows, then up rows); the
  // MXFP8 codes [M, ffn] and blocked scales of silu(gate) * up replace y.
  int ffn = 0;
  void* q_codes = nullptr;
  void* q_scales = nullptr;
  // Fused Euler update (bf16 layer only): y is not
  // written; z [M / eu_frame, N, eu_frame] += eu_dt v, bf16 copy to eu_zb.
  float* eu_z = nullptr;
  void* eu_zb = nullptr;
  int64_t eu_frame = 0;
  float eu_dt = 0.f;
};
// Returns cudaSuccess or the failing CUDA error; *driver_failed is set when
// the tensor-map encoder (driver API) is missing or rejects a map.
cudaError_t launch_lora_linear(const LinearLaunch& p, cudaStream_t s, bool* driver_failed);

// CTAs per cluster sharing one panel in lg_lora_linear (0: chosen per shape).
void set_cluster_override(int g);
// MMA variant of lg_lora_linear: 1 single-SM, 2 SM pair (0: chosen per shape).
void set_variant_override(int v);

// Device error word of the current device: read and clear (synchronous on s).
cudaError_t read_and_clear_device_error(cudaStream_t s, int* value);

// The driver's process-unique id of the calling thread's current CUDA
// context.  False when no context is current or the driver cannot say; a
// per-device cache keyed on this id notices a context that was destroyed
// and recreated (cudaDeviceReset) or a different context made current.
bool current_context_id(unsigned long long* id);

// Every check lg_lora_linear makes on its arguments except those on the
// workspace, then (for M > 0) the current device's compute capability, in
// the same order and with the same status codes; launches nothing.  Returns
// an lg_status value.
int check_lora_linear(const void* x, const void* W, const float* A_cat, const float* B_cat, const void* y,
                      int64_t M, int K, int N, int R);

}  // namespace lg
