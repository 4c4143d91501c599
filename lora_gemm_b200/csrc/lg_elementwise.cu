// HBM-bound kernels of the refiner hot path: Philox stream, Gaussian noise,
// partial re-noise, the Euler update, the rank-axis LoRA merge and the bf16
// copies of the merged factors.  All are grid-stride loops over 16-byte
// vectors (one float4 = one Philox block of 4 elements), sized to a few waves
// of the SMs, with a scalar tail.
//
// Re-noise and Euler follow "Open-H3-Regenerate-2K: High-Resolution Video
// Refinement with Few-Step Diffusion", section "Three steps instead of
// dozens"; the merge follows "Open-H3-Regenerate-2K：MiniMax H3 的开源 4K
// 精修方案", section "三个步如何完成工作".
#include <algorithm>
#include <mutex>

#include "lg_bm_tables.inc"
#include "lg_device.cuh"
#include "lg_internal.h"

namespace lg {

namespace {

constexpr int kThreads = 256;
// The FP64 Box-Muller kernels are bound by their mix of instructions and
// shared-memory table gathers, not by HBM.  Each thread works on three Philox
// blocks at once (kBmUnroll) so that their FP64 chains interleave; the 100 KB
// of tables staged per block allow one 512-thread block per SM.
#ifndef LG_BM_THREADS
#define LG_BM_THREADS 512
#endif
#ifndef LG_BM_BLOCKS_PER_SM
#define LG_BM_BLOCKS_PER_SM 1
#endif
constexpr int kBmThreads = LG_BM_THREADS;
constexpr int kBmBlocksPerSm = LG_BM_BLOCKS_PER_SM;

static_assert(LG_BM_LOG_SWITCH == kBmLogSwitch, "log table built for another switch point");
static_assert(LG_BM_TRIG_COARSE_ENTRIES == 1 << kBmCoarseBits && LG_BM_TRIG_FINE_ENTRIES == (1 << (23 - kBmCoarseBits)) + 1,
              "angle tables built for another split");

// The three tables in one image, copied to shared memory as 16-byte chunks.
struct alignas(16) BmTableImage {
  BmLogEntry log[LG_BM_LOG_ENTRIES];
  BmTrigEntry coarse[LG_BM_TRIG_COARSE_ENTRIES];
  BmTrigEntry fine[LG_BM_TRIG_FINE_ENTRIES];
};
static_assert(sizeof(BmTableImage) % 16 == 0, "table image is copied in 16-byte chunks");
constexpr int kBmSmemBytes = (int)sizeof(BmTableImage);
__device__ const BmTableImage g_bm_tables = {LG_BM_LOG_TABLE, LG_BM_TRIG_COARSE_TABLE, LG_BM_TRIG_FINE_TABLE};

// Copies the Box-Muller tables into the block's (dynamic) shared memory with
// asynchronous 16-byte copies, where the data-dependent lookups cost one
// shared load each.  The copies are issued first and waited for later, so
// the caller can issue its first global loads in between.
__device__ __forceinline__ void stage_bm_tables_issue(uint8_t* smem) {
  const uint64_t src = (uint64_t)__cvta_generic_to_global(&g_bm_tables);
  const uint32_t dst = smem_u32(smem);
  for (int i = threadIdx.x; i < kBmSmemBytes / 16; i += blockDim.x)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * i), "l"(src + 16 * i) : "memory");
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ BmTables stage_bm_tables_wait(const uint8_t* smem) {
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  const BmTableImage* t = reinterpret_cast<const BmTableImage*>(smem);
  return BmTables{t->log, t->coarse, t->fine};
}

__device__ __forceinline__ int64_t gtid() { return (int64_t)blockIdx.x * blockDim.x + threadIdx.x; }
__device__ __forceinline__ int64_t gstride() { return (int64_t)gridDim.x * blockDim.x; }

__global__ void __launch_bounds__(kThreads) k_philox_u32(uint4* __restrict__ out, int64_t n_blocks, uint32_t k0,
                                                         uint32_t k1, uint64_t block0) {
  for (int64_t b = gtid(); b < n_blocks; b += gstride()) {
    const Words4 r = philox4x32_10(block0 + (uint64_t)b, k0, k1);
    out[b] = make_uint4(r.w0, r.w1, r.w2, r.w3);
  }
}

// The four normals of Philox block `block`.
__device__ __forceinline__ void normals4(uint64_t block, uint32_t k0, uint32_t k1, const BmTables& tab,
                                         double (&e)[4]) {
  const Words4 r = philox4x32_10(block, k0, k1);
  box_muller(r.w0, r.w1, tab, e[0], e[1]);
  box_muller(r.w2, r.w3, tab, e[2], e[3]);
}

// The normal stream (RENOISE = false: eps = the FP32 roundings) or the
// re-noise x = (1 - sigma) up + sigma eps (blended in double from the
// unrounded eps and rounded once to FP32) over the elements [0, 4 nb + tail)
// of one launch, whose element 0 is global element 4 block0.  Threads stride
// over the nb full Philox blocks (one float4 each) with 32-bit indices, U
// blocks at a time; each loads its next U blocks of up before the FP64 work
// on the current ones, so the loads' DRAM latency hides behind that work.
// The last, partial round computes only the blocks that exist, so the
// threads that hold one block of it do a third of a round's work.  The
// `tail` < 4 elements past the full blocks go to thread 0 of block 0.  x may
// alias up (each element is read before it is written by the same thread),
// so neither pointer is restrict.
#ifndef LG_BM_UNROLL
#define LG_BM_UNROLL 3
#endif
constexpr int kBmUnroll = LG_BM_UNROLL;  // Philox blocks a thread works on at once

// One Philox block of the stream: 4 normals, or 4 re-noised elements of u.
template <bool RENOISE>
__device__ __forceinline__ float4 stream_block(uint64_t block, uint32_t k0, uint32_t k1, const BmTables& tab,
                                               double sigma, double keep, const float4& u) {
  const Words4 r = philox4x32_10(block, k0, k1);
  float4 o;
  if constexpr (RENOISE) {
    // sigma eps = (sigma rho) cos / sin: sigma scales the radius once per
    // pair, each element then takes one fused multiply-add.
    double rho, c, s;
    box_muller_polar(r.w0, r.w1, tab, rho, c, s);
    rho *= sigma;
    o.x = (float)fma(rho, c, keep * (double)u.x);
    o.y = (float)fma(rho, s, keep * (double)u.y);
    box_muller_polar(r.w2, r.w3, tab, rho, c, s);
    rho *= sigma;
    o.z = (float)fma(rho, c, keep * (double)u.z);
    o.w = (float)fma(rho, s, keep * (double)u.w);
  } else {
    double e[4];
    box_muller(r.w0, r.w1, tab, e[0], e[1]);
    box_muller(r.w2, r.w3, tab, e[2], e[3]);
    o = make_float4((float)e[0], (float)e[1], (float)e[2], (float)e[3]);
  }
  return o;
}

template <bool RENOISE>
__device__ __forceinline__ void normal_stream(const float* up, float* out, uint32_t nb, uint32_t tail, double sigma,
                                              uint32_t k0, uint32_t k1, uint64_t block0, uint8_t* smem) {
  stage_bm_tables_issue(smem);
  const double keep = 1.0 - sigma;
  const uint32_t stride = gridDim.x * blockDim.x;
  const uint32_t first = blockIdx.x * blockDim.x + threadIdx.x;
  const float4* up4 = reinterpret_cast<const float4*>(up);
  float4* out4 = reinterpret_cast<float4*>(out);
  constexpr int U = kBmUnroll;
  float4 u_next[U];
#pragma unroll
  for (int k = 0; k < U; ++k) {
    u_next[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (RENOISE && first + k * stride < nb) u_next[k] = __ldcs(up4 + first + k * stride);
  }
  const BmTables tab = stage_bm_tables_wait(smem);
  uint32_t b = first;
  // Full rounds: all U blocks exist, and their FP64 chains interleave.
  for (; b + (U - 1) * stride < nb; b += U * stride) {
    float4 u[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      u[k] = u_next[k];
      const uint32_t bn = b + (U + k) * stride;
      if (RENOISE && bn < nb) u_next[k] = __ldcs(up4 + bn);
    }
    float4 o[U];
#pragma unroll
    for (int k = 0; k < U; ++k) o[k] = stream_block<RENOISE>(block0 + b + k * stride, k0, k1, tab, sigma, keep, u[k]);
#pragma unroll
    for (int k = 0; k < U; ++k) __stcs(out4 + b + k * stride, o[k]);
  }
  // The partial last round (up was prefetched for exactly these blocks).
#pragma unroll
  for (int k = 0; k < U; ++k) {
    if (b + k * stride < nb)
      __stcs(out4 + b + k * stride,
             stream_block<RENOISE>(block0 + b + k * stride, k0, k1, tab, sigma, keep, u_next[k]));
  }
  if (tail && first == 0) {
    double e[4];
    normals4(block0 + nb, k0, k1, tab, e);
#pragma unroll
    for (uint32_t t = 0; t < 4; ++t) {
      if (t < tail) {
        const size_t i = 4 * (size_t)nb + t;
        out[i] = RENOISE ? (float)fma(sigma, e[t], keep * (double)up[i]) : (float)e[t];
      }
    }
  }
}

__global__ void __launch_bounds__(kBmThreads, kBmBlocksPerSm)
    k_philox_normal(float* __restrict__ eps, uint32_t nb, uint32_t tail, uint32_t k0, uint32_t k1, uint64_t block0) {
  extern __shared__ __align__(16) uint8_t bm_smem[];
  normal_stream<false>(nullptr, eps, nb, tail, 0.0, k0, k1, block0, bm_smem);
}

__global__ void __launch_bounds__(kBmThreads, kBmBlocksPerSm)
    k_renoise(const float* up, float* x, uint32_t nb, uint32_t tail, double sigma, uint32_t k0, uint32_t k1,
              uint64_t block0) {
  extern __shared__ __align__(16) uint8_t bm_smem[];
  normal_stream<true>(up, x, nb, tail, sigma, k0, k1, block0, bm_smem);
}

// x += dt v with dt = sigma_next - sigma taken in FP32 (exact for the
// schedule by Sterbenz's lemma); one fused multiply-add per element.
constexpr int kEulerUnroll = 4;
__global__ void __launch_bounds__(kThreads) k_euler(float* __restrict__ x, const float* __restrict__ v, int64_t n,
                                                    float dt) {
  const int64_t n4 = n / 4;
  float4* x4 = reinterpret_cast<float4*>(x);
  const float4* v4 = reinterpret_cast<const float4*>(v);
  const int64_t stride = gstride();
  // Every pass issues all of its loads before any arithmetic, the last
  // (partial) pass included, so each thread keeps up to 2 x kEulerUnroll
  // 16-byte loads in flight to the end.
  for (int64_t i = gtid(); i < n4; i += kEulerUnroll * stride) {
    float4 a[kEulerUnroll], b[kEulerUnroll];
#pragma unroll
    for (int u = 0; u < kEulerUnroll; ++u) {
      const int64_t j = i + u * stride;
      if (j < n4) {
        a[u] = x4[j];
        b[u] = __ldcs(v4 + j);
      }
    }
#pragma unroll
    for (int u = 0; u < kEulerUnroll; ++u) {
      const int64_t j = i + u * stride;
      if (j < n4) {
        a[u].x = fmaf(dt, b[u].x, a[u].x);
        a[u].y = fmaf(dt, b[u].y, a[u].y);
        a[u].z = fmaf(dt, b[u].z, a[u].z);
        a[u].w = fmaf(dt, b[u].w, a[u].w);
        x4[j] = a[u];
      }
    }
  }
  if (gtid() == 0) {
    for (int64_t t = 4 * n4; t < n; ++t) x[t] = fmaf(dt, v[t], x[t]);
  }
}

// A_cat[off_i + r][k] = s_i A_i[r][k]  (float4 granularity; d_in % 4 == 0).
__global__ void __launch_bounds__(kThreads) k_merge_a(const MergeAParams p, float* __restrict__ A_cat) {
  const int64_t q = p.d_in / 4;
  const int64_t total = (int64_t)p.row_off[p.n_adapters] * q;
  for (int64_t i = gtid(); i < total; i += gstride()) {
    const int row = (int)(i / q);
    const int64_t c = i - (int64_t)row * q;
    int a = 0;
    while (a + 1 < p.n_adapters && row >= p.row_off[a + 1]) ++a;
    const float s = p.scale[a];
    const float4 v = reinterpret_cast<const float4*>(p.A[a])[(int64_t)(row - p.row_off[a]) * q + c];
    reinterpret_cast<float4*>(A_cat)[i] = make_float4(s * v.x, s * v.y, s * v.z, s * v.w);
  }
}

// B_cat[o][off_i + r] = B_i[o][r]  (ranks % 4 == 0, so a float4 never
// straddles two adapters).
__global__ void __launch_bounds__(kThreads) k_merge_b(const MergeBParams p, float* __restrict__ B_cat) {
  const int R = p.col_off[p.n_adapters];
  const int q = R / 4;
  const int64_t total = (int64_t)p.d_out * q;
  for (int64_t i = gtid(); i < total; i += gstride()) {
    const int64_t o = i / q;
    const int col = (int)(i - o * q) * 4;
    int a = 0;
    while (a + 1 < p.n_adapters && col >= p.col_off[a + 1]) ++a;
    const int r_a = p.col_off[a + 1] - p.col_off[a];
    const float4 v = *reinterpret_cast<const float4*>(p.B[a] + o * r_a + (col - p.col_off[a]));
    reinterpret_cast<float4*>(B_cat)[i] = v;
  }
}

// FP32 -> bf16 round-to-nearest-even, two arrays in one launch (n % 4 == 0).
__global__ void __launch_bounds__(kThreads) k_prep_bf16(const float* __restrict__ a, const float* __restrict__ b,
                                                        uint16_t* __restrict__ da, uint16_t* __restrict__ db,
                                                        int64_t na4, int64_t nb4) {
  for (int64_t i = gtid(); i < na4 + nb4; i += gstride()) {
    const bool first = i < na4;
    const int64_t j = first ? i : i - na4;
    const float4 v = reinterpret_cast<const float4*>(first ? a : b)[j];
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    reinterpret_cast<uint2*>(first ? da : db)[j] = o;
  }
}

}  // namespace

int elementwise_grid(int64_t work, int sm_count) {
  const int64_t want = (work + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)std::max(sm_count, 1) * 8;  // 8 x 256 threads = 2048 per SM
  return (int)std::max<int64_t>(1, std::min(want, cap));
}

cudaError_t launch_philox_u32(uint32_t* out, int64_t n_blocks, uint64_t seed, uint64_t block_offset, int sm_count,
                              cudaStream_t s) {
  k_philox_u32<<<elementwise_grid(n_blocks, sm_count), kThreads, 0, s>>>(
      reinterpret_cast<uint4*>(out), n_blocks, (uint32_t)seed, (uint32_t)(seed >> 32), block_offset);
  return cudaGetLastError();
}

// Lets the two Box-Muller kernels use the table image's dynamic shared
// memory, once per CUDA context (the setting belongs to the context).
cudaError_t configure_bm_kernels() {
  static std::mutex mu;
  static bool configured = false;
  static unsigned long long context = 0;
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  if (have_ctx && configured && context == ctx) return cudaSuccess;
  for (const void* k : {(const void*)k_renoise, (const void*)k_philox_normal}) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kBmSmemBytes);
    if (e != cudaSuccess) return e;
  }
  configured = have_ctx;
  context = ctx;
  return cudaSuccess;
}

// Normal stream / re-noise over n >= 1 elements starting at global element
// 4 block0, in launches of at most 2^30 Philox blocks (32-bit indices inside).
template <bool RENOISE>
cudaError_t launch_normal_stream(const float* up, float* out, int64_t n, double sigma, uint64_t seed,
                                 uint64_t block0, int sm_count, cudaStream_t s) {
  constexpr int64_t kChunkBlocks = (int64_t)1 << 30;
  const cudaError_t ce = configure_bm_kernels();
  if (ce != cudaSuccess) return ce;
  const int64_t full = n / 4;
  const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  for (int64_t done = 0;;) {
    const int64_t nb = std::min(full - done, kChunkBlocks);
    const bool last = done + nb == full;
    const uint32_t tail = last ? (uint32_t)(n % 4) : 0u;
    const int64_t want = (std::max<int64_t>(nb, 1) + kBmThreads - 1) / kBmThreads;
    const int grid = (int)std::min<int64_t>(want, (int64_t)kBmBlocksPerSm * std::max(sm_count, 1));
    if constexpr (RENOISE) {
      k_renoise<<<grid, kBmThreads, kBmSmemBytes, s>>>(up + 4 * done, out + 4 * done, (uint32_t)nb, tail, sigma, k0,
                                                       k1, block0 + (uint64_t)done);
    } else {
      k_philox_normal<<<grid, kBmThreads, kBmSmemBytes, s>>>(out + 4 * done, (uint32_t)nb, tail, k0, k1,
                                                             block0 + (uint64_t)done);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || last) return e;
    done += nb;
  }
}

cudaError_t launch_philox_normal(float* eps, int64_t n, uint64_t seed, uint64_t offset, int sm_count,
                                 cudaStream_t s) {
  return launch_normal_stream<false>(nullptr, eps, n, 0.0, seed, offset / 4, sm_count, s);
}

cudaError_t launch_renoise(const float* up, float* x, int64_t n, float sigma, uint64_t seed, uint64_t offset,
                           int sm_count, cudaStream_t s) {
  return launch_normal_stream<true>(up, x, n, (double)sigma, seed, offset / 4, sm_count, s);
}

cudaError_t launch_euler(float* x, const float* v, int64_t n, float dt, int sm_count, cudaStream_t s) {
  k_euler<<<elementwise_grid(std::max<int64_t>(n / 4, 1), sm_count), kThreads, 0, s>>>(x, v, n, dt);
  return cudaGetLastError();
}

cudaError_t launch_merge(const MergeAParams& pa, const MergeBParams& pb, float* A_cat, float* B_cat, int sm_count,
                         cudaStream_t s) {
  const int64_t wa = (int64_t)pa.row_off[pa.n_adapters] * (pa.d_in / 4);
  const int64_t wb = (int64_t)pb.d_out * (pb.col_off[pb.n_adapters] / 4);
  k_merge_a<<<elementwise_grid(wa, sm_count), kThreads, 0, s>>>(pa, A_cat);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_merge_b<<<elementwise_grid(wb, sm_count), kThreads, 0, s>>>(pb, B_cat);
  return cudaGetLastError();
}

cudaError_t launch_prep_bf16(const float* A_cat, const float* B_cat, uint16_t* dstA, uint16_t* dstB, int64_t nA,
                             int64_t nB, int sm_count, cudaStream_t s) {
  const int64_t w = nA / 4 + nB / 4;
  k_prep_bf16<<<elementwise_grid(w, sm_count), kThreads, 0, s>>>(A_cat, B_cat, dstA, dstB, nA / 4, nB / 4);
  return cudaGetLastError();
}

}  // namespace lg
