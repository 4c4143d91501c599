// Merged-LoRA linear layer on the sm_100a tensor cores:
//
//   y = x W^T + (x A_cat^T) B_cat^T
//
// with bf16 x [M, K], W [N, K], bf16 copies of the FP32 merged factors
// A_cat [R, K], B_cat [N, R], FP32 accumulation, bf16 y [M, N].  The linear
// layer is the frozen transformer's linear carrying the rank-axis merged LoRA
// of "Open-H3-Regenerate-2K：MiniMax H3 的开源 4K 精修方案" (section
// "三个步如何完成工作", rank 384 + 128 + 64 = 576 on 312 linear layers); the
// pages give no kernel design, so everything below is this library's.
//
// Design (one CTA per SM, persistent over 128-row token panels):
//   * TMEM (512 columns x 128 lanes, one lane per token row) holds the FP32
//     accumulator of one 128 x 224 output tile in columns [0, 224) and the
//     panel's rank-R intermediate h = x A_cat^T as packed bf16 pairs in
//     columns [224, 224 + R/2) -- 288 columns for R = 576.  h is computed
//     once per panel and never leaves the SM.
//   * Phase A (per panel): for each 192-wide rank chunk, a K loop of
//     tcgen05.mma (A = x tile, B = A_cat tile, both from shared memory)
//     accumulates the chunk of h in FP32 in the accumulator columns; the
//     epilogue warps round it to bf16 and store it into the h columns.
//   * Phase B (per 224-wide N tile): a K loop x W^T into the accumulator,
//     then R/16 more tcgen05.mma steps with A = h read straight from tensor
//     memory and B = the B_cat tile, into the same accumulator; the epilogue
//     warps convert the tile to bf16 and store it.
//   * Warp roles: warp 0 issues TMA loads into a 5-stage shared-memory ring
//     (128-byte swizzled K-major tiles), warp 1 issues the MMAs (one thread)
//     and owns the TMEM allocation, warps 2-5 are the epilogue (each reads
//     the 32 TMEM lanes its warp may access).
//   * Every mbarrier wait is bounded; on expiry the kernel records
//     LG_ERR_DEVICE_TIMEOUT in the device error word, drains its own TMA
//     copies and MMAs, frees its TMEM and returns.
#include <mutex>

#include <cudaTypedefs.h>

#include "../../include/lora_gemm.h"
#include "lg_device.cuh"
#include "lg_internal.h"

namespace lg {

__device__ int g_device_error;

namespace {

constexpr int BM = 128;  // token rows per panel = TMEM lanes
constexpr int BK = 64;   // K elements per stage: one 128-byte swizzle span
constexpr int BN = 224;  // output columns per tile
constexpr int HC = 192;  // rank columns per down-projection chunk
constexpr int STAGES = 5;
constexpr int RMAX = 576;
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KiB: x tile
constexpr uint32_t B_BYTES = BN * BK * 2;  // 28 KiB: W / A_cat / B_cat tile
constexpr uint32_t H_TILE_BYTES = HC * BK * 2;
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t H_COL = BN;
constexpr int NUM_THREADS = 192;
constexpr uint64_t TEARDOWN_LIMIT_NS = 200ull * 1000ull * 1000ull;

static_assert(H_COL + RMAX / 2 <= TMEM_COLS, "h does not fit next to the accumulator");
static_assert(H_TILE_BYTES <= B_BYTES, "A_cat chunk tile does not fit the B slot");
static_assert(A_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "tiles must stay 1024-byte aligned");

struct Control {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Control);

struct Args {
  uint16_t* y;
  int64_t M;
  int N;
  int R;
  int num_panels;
  int n_tiles;
  int n_chunks;
  int k_blocks;
  int r_blocks;
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ void record_timeout(volatile int* abort_flag) {
  *abort_flag = 1;
  atomicCAS(&g_device_error, 0, (int)LG_ERR_DEVICE_TIMEOUT);
}

// Wait for the phase of `bar` with parity `parity` to complete, giving up
// after limit_ns or as soon as another warp of the CTA has given up.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 >= limit_ns) {
      record_timeout(abort_flag);
      return false;
    }
  }
}

// Teardown wait: fixed limit, ignores the abort flag.
__device__ __noinline__ void wait_teardown(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 >= TEARDOWN_LIMIT_NS) {
      record_timeout(abort_flag);
      return;
    }
  }
}

__device__ __forceinline__ void advance(uint32_t& stage, uint32_t& phase) {
  if (++stage == STAGES) {
    stage = 0;
    phase ^= 1;
  }
}

__device__ void run_producer(const CUtensorMap* tm_x, const CUtensorMap* tm_w, const CUtensorMap* tm_a,
                             const CUtensorMap* tm_b, const Args& a, Control* ctl, uint32_t smem_base,
                             volatile int* abort_flag) {
  uint32_t stage = 0, phase = 0;
  uint64_t fills = 0;
  bool ok = true;
  const uint32_t full0 = smem_u32(&ctl->full[0]);
  const uint32_t empty0 = smem_u32(&ctl->empty[0]);
  for (int p = blockIdx.x; ok && p < a.num_panels; p += gridDim.x) {
    const int m0 = p * BM;
    // Phase A: x panel and A_cat chunks.
    for (int c = 0; ok && c < a.n_chunks; ++c) {
      for (int kb = 0; kb < a.k_blocks; ++kb) {
        if (!wait_bounded(empty0 + 8 * stage, phase ^ 1, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t bar = full0 + 8 * stage;
        mbar_arrive_expect_tx(bar, A_BYTES + H_TILE_BYTES);
        tma_load_2d(sa, tm_x, bar, kb * BK, m0);
        tma_load_2d(sa + A_BYTES, tm_a, bar, kb * BK, c * HC);
        ++fills;
        advance(stage, phase);
      }
    }
    // Phase B: x panel with W, then B_cat for the rank steps.
    for (int t = 0; ok && t < a.n_tiles; ++t) {
      const int n0 = t * BN;
      for (int kb = 0; kb < a.k_blocks; ++kb) {
        if (!wait_bounded(empty0 + 8 * stage, phase ^ 1, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t bar = full0 + 8 * stage;
        mbar_arrive_expect_tx(bar, A_BYTES + B_BYTES);
        tma_load_2d(sa, tm_x, bar, kb * BK, m0);
        tma_load_2d(sa + A_BYTES, tm_w, bar, kb * BK, n0);
        ++fills;
        advance(stage, phase);
      }
      for (int rb = 0; ok && rb < a.r_blocks; ++rb) {
        if (!wait_bounded(empty0 + 8 * stage, phase ^ 1, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint32_t bar = full0 + 8 * stage;
        mbar_arrive_expect_tx(bar, B_BYTES);
        tma_load_2d(sa + A_BYTES, tm_b, bar, rb * BK, n0);
        ++fills;
        advance(stage, phase);
      }
    }
  }
  // Let every copy this CTA issued land before the CTA may exit.
  for (uint32_t s = 0; s < (uint32_t)STAGES; ++s) {
    const uint64_t fs = fills / STAGES + (s < fills % STAGES ? 1 : 0);
    if (fs) wait_teardown(full0 + 8 * s, (uint32_t)((fs - 1) & 1), abort_flag);
  }
}

__device__ void run_mma(const Args& a, Control* ctl, uint32_t smem_base, uint32_t tmem,
                        volatile int* abort_flag) {
  uint32_t stage = 0, phase = 0, acc_phase = 0;
  bool ok = true;
  const uint32_t full0 = smem_u32(&ctl->full[0]);
  const uint32_t empty0 = smem_u32(&ctl->empty[0]);
  const uint32_t acc_full = smem_u32(&ctl->acc_full);
  const uint32_t acc_empty = smem_u32(&ctl->acc_empty);
  constexpr uint32_t idesc_h = idesc_bf16_f32(BM, HC);
  constexpr uint32_t idesc_y = idesc_bf16_f32(BM, BN);
  const uint32_t d_acc = tmem + ACC_COL;
  for (int p = blockIdx.x; ok && p < a.num_panels; p += gridDim.x) {
    for (int c = 0; ok && c < a.n_chunks; ++c) {
      if (!wait_bounded(acc_empty, acc_phase ^ 1, a.wait_limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int kb = 0; kb < a.k_blocks; ++kb) {
        if (!wait_bounded(full0 + 8 * stage, phase, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint64_t da = sw128_kmajor_desc(sa);
        const uint64_t db = sw128_kmajor_desc(sa + A_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          umma_ss(d_acc, da + 2 * kk, db + 2 * kk, idesc_h, (kb | kk) != 0);
        }
        umma_commit(empty0 + 8 * stage);
        advance(stage, phase);
      }
      if (!ok) break;
      umma_commit(acc_full);
      acc_phase ^= 1;
    }
    for (int t = 0; ok && t < a.n_tiles; ++t) {
      if (!wait_bounded(acc_empty, acc_phase ^ 1, a.wait_limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int kb = 0; kb < a.k_blocks; ++kb) {
        if (!wait_bounded(full0 + 8 * stage, phase, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint64_t da = sw128_kmajor_desc(sa);
        const uint64_t db = sw128_kmajor_desc(sa + A_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          umma_ss(d_acc, da + 2 * kk, db + 2 * kk, idesc_y, (kb | kk) != 0);
        }
        umma_commit(empty0 + 8 * stage);
        advance(stage, phase);
      }
      for (int rb = 0; ok && rb < a.r_blocks; ++rb) {
        if (!wait_bounded(full0 + 8 * stage, phase, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_base + stage * STAGE_BYTES;
        const uint64_t db = sw128_kmajor_desc(sa + A_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // 16 ranks of h = 8 packed columns.
          umma_ts(d_acc, tmem + H_COL + (uint32_t)(rb * (BK / 2) + kk * 8), db + 2 * kk, idesc_y, 1u);
        }
        umma_commit(empty0 + 8 * stage);
        advance(stage, phase);
      }
      if (!ok) break;
      umma_commit(acc_full);
      acc_phase ^= 1;
    }
  }
  // Every MMA this thread issued must finish before TMEM is freed.
  const uint32_t drain = smem_u32(&ctl->drain);
  umma_commit(drain);
  wait_teardown(drain, 0, abort_flag);
}

__device__ void run_epilogue(const Args& a, Control* ctl, uint32_t tmem, int warp, int lane,
                             volatile int* abort_flag) {
  const int q = warp & 3;  // TMEM lanes 32q .. 32q+31 belong to this warp
  const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
  const uint32_t acc_full = smem_u32(&ctl->acc_full);
  const uint32_t acc_empty = smem_u32(&ctl->acc_empty);
  uint32_t acc_phase = 0;
  bool ok = true;
  for (int p = blockIdx.x; ok && p < a.num_panels; p += gridDim.x) {
    const int64_t m0 = (int64_t)p * BM;
    for (int c = 0; ok && c < a.n_chunks; ++c) {
      ok = __all_sync(0xffffffffu, wait_bounded(acc_full, acc_phase, a.wait_limit_ns, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int valid = min(HC, a.R - c * HC);
      for (int j = 0; j < valid / 32; ++j) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(lane_base + ACC_COL + 32 * j, v);
        tmem_wait_ld();
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        tmem_st_32x32b_x16(lane_base + H_COL + (uint32_t)((c * HC + 32 * j) / 2), packed);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1;
    }
    for (int t = 0; ok && t < a.n_tiles; ++t) {
      ok = __all_sync(0xffffffffu, wait_bounded(acc_full, acc_phase, a.wait_limit_ns, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int64_t row = m0 + 32 * q + lane;
      const int n0 = t * BN;
      for (int j = 0; j < BN / 32; ++j) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(lane_base + ACC_COL + 32 * j, v);
        tmem_wait_ld();
        const int col = n0 + 32 * j;
        if (row < a.M && col < a.N) {
          uint4* dst = reinterpret_cast<uint4*>(a.y + row * (int64_t)a.N + col);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            dst[g] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * g + 0]), __uint_as_float(v[8 * g + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * g + 2]), __uint_as_float(v[8 * g + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * g + 4]), __uint_as_float(v[8 * g + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * g + 6]), __uint_as_float(v[8 * g + 7])));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1;
    }
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_lora_linear(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  Control* ctl = reinterpret_cast<Control*>(smem + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t smem_base = smem_u32(smem);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->acc_full), 1);
    mbar_init(smem_u32(&ctl->acc_empty), 4);
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    if (args.R > 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  volatile int* abort_flag = &ctl->abort_flag;

  if (warp == 0) {
    if (lane == 0) run_producer(&tm_x, &tm_w, &tm_a, &tm_b, args, ctl, smem_base, abort_flag);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) run_mma(args, ctl, smem_base, tmem, abort_flag);
    __syncwarp();
  } else {
    run_epilogue(args, ctl, tmem, warp, lane, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
  });
  return fn;
}

// Row-major bf16 matrix [outer, inner] read as tiles of box_outer rows x 64
// columns with the 128-byte swizzle; out-of-range rows read as zero.
bool make_map(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, uint64_t inner,
              uint64_t outer, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
  cuuint32_t elem_strides[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_lora_linear(const LinearLaunch& p, cudaStream_t s, bool* driver_failed) {
  *driver_failed = false;
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) {
    *driver_failed = true;
    return cudaErrorNotSupported;
  }
  CUtensorMap tm_x, tm_w, tm_a, tm_b;
  bool ok = make_map(enc, &tm_x, p.x, (uint64_t)p.K, (uint64_t)p.M, BM) &&
            make_map(enc, &tm_w, p.W, (uint64_t)p.K, (uint64_t)p.N, BN);
  if (ok && p.R > 0) {
    ok = make_map(enc, &tm_a, p.A_bf16, (uint64_t)p.K, (uint64_t)p.R, HC) &&
         make_map(enc, &tm_b, p.B_bf16, (uint64_t)p.R, (uint64_t)p.N, BN);
  } else {
    tm_a = tm_x;  // never read when R == 0
    tm_b = tm_x;
  }
  if (!ok) {
    *driver_failed = true;
    return cudaErrorInvalidValue;
  }

  static std::mutex mu;
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || !configured[dev]) {
      e = cudaFuncSetAttribute(k_lora_linear, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) configured[dev] = true;
    }
  }

  Args args;
  args.y = reinterpret_cast<uint16_t*>(p.y);
  args.M = p.M;
  args.N = p.N;
  args.R = p.R;
  args.num_panels = (int)((p.M + BM - 1) / BM);
  args.n_tiles = (p.N + BN - 1) / BN;
  args.n_chunks = (p.R + HC - 1) / HC;
  args.k_blocks = p.K / BK;
  args.r_blocks = p.R / BK;
  args.wait_limit_ns = p.wait_limit_ns;
  const int grid = args.num_panels < p.sm_count ? args.num_panels : p.sm_count;
  k_lora_linear<<<grid, NUM_THREADS, kSmemBytes, s>>>(tm_x, tm_w, tm_a, tm_b, args);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(cudaStream_t s, int* value) {
  *value = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  }
  *value = v;
  return e;
}

}  // namespace lg
