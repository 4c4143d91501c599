// MXFP8 quantization of bf16 rows along K ("Open-H3-Regenerate-2K:
// High-Resolution Video Refinement with Few-Step Diffusion", section "Where
// the 3.9x speedup comes from": MXFP8 linear layers, activations re-quantized
// at every stage).  The pages name the format only; the block rule is the
// OCP Microscaling (MX) one: 32 consecutive values along K share the scale
// 2^e, e = floor(log2 max|v|) - 8 clamped to [-127, 127] (-127 for an
// all-zero block), stored as the E8M0 byte e + 127; each value becomes the
// E4M3 code of v 2^-e, rounded to nearest even and saturated at +-448.
//
// Scale layout (what the block-scaled MMAs take through tcgen05.cp): rows in
// groups of 128 and K in groups of 128 (four blocks); group (g, kg) is 512
// contiguous bytes at ((g * (K / 128)) + kg) * 512, with the byte of row r
// (0..127 within the group) and block kb (0..3 within the K group) at
// 16 (r mod 32) + 4 (r / 32) + kb.  Rows past the end of the matrix, up to
// the next multiple of 128, get scale byte 0.
#include <cuda_fp8.h>

#include "lg_device.cuh"
#include "lg_internal.h"

namespace lg {

namespace {

constexpr int kQThreads = 256;

__device__ __forceinline__ int64_t sf_offset(int64_t row, int k_block, int k_groups) {
  const int64_t g = row >> 7;
  const int r = (int)(row & 127);
  const int kg = k_block >> 2;
  const int kb = k_block & 3;
  return ((g * k_groups + kg) << 9) + 16 * (r & 31) + 4 * (r >> 5) + kb;
}

// One thread per 32-value block: rows [0, rows_pad) x blocks [0, K / 32).
__global__ void __launch_bounds__(kQThreads) k_mx_quantize(const uint16_t* __restrict__ in, int64_t rows,
                                                           int64_t rows_pad, int K, uint8_t* __restrict__ codes,
                                                           uint8_t* __restrict__ scales) {
  const int kblocks = K / 32;
  const int k_groups = K / 128;
  const int64_t total = rows_pad * kblocks;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = t / kblocks;
    const int kb = (int)(t - row * kblocks);
    uint8_t* sf = scales + sf_offset(row, kb, k_groups);
    if (row >= rows) {
      *sf = 0;
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(in + row * (int64_t)K + 32 * kb);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 q = src[i];
      w[4 * i] = q.x;
      w[4 * i + 1] = q.y;
      w[4 * i + 2] = q.z;
      w[4 * i + 3] = q.w;
    }
    // bf16 -> FP32 is exact: the high half of the FP32 word.
    float v[32];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      amax = fmaxf(amax, fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1])));
    }
    int e = -127;
    if (amax > 0.f) {
      int ex;
      frexpf(amax, &ex);  // amax = m 2^ex, m in [0.5, 1): floor(log2 amax) = ex - 1
      e = min(max(ex - 1 - 8, -127), 127);
    }
    // 2^-e as an FP32 number (2^127 at most; 2^-127 is the subnormal 2^-127).
    const float inv = e == 127 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - e) << 23);
    uint32_t out[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_fp8x2_storage_t lo =
          __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i] * inv, v[4 * i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi =
          __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2] * inv, v[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
      out[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + row * (int64_t)K + 32 * kb);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    *sf = (uint8_t)(e + 127);
  }
}

}  // namespace

cudaError_t launch_mx_quantize(const uint16_t* in, int64_t rows, int K, uint8_t* codes, uint8_t* scales,
                               int sm_count, cudaStream_t s) {
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  const int64_t work = rows_pad * (K / 32);
  k_mx_quantize<<<elementwise_grid(work, sm_count), kQThreads, 0, s>>>(in, rows, rows_pad, K, codes, scales);
  return cudaGetLastError();
}

}  // namespace lg
