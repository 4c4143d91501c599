// C ABI entry points (include/lora_gemm.h): argument validation, device
// checks and kernel launches.  Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <mutex>

#include <cudaTypedefs.h>

#include "../../include/lora_gemm.h"
#include "lg_internal.h"

namespace {

constexpr uint64_t kDefaultWaitLimitNs = 4000000000ull;
constexpr int kMaxRank = 576;
constexpr int kMaxDim = 1 << 20;

std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [a, a + na) and [b, b + nb) in bytes.
bool overlaps(const void* a, uint64_t na, const void* b, uint64_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

uint64_t align256(uint64_t v) { return (v + 255u) & ~(uint64_t)255u; }

struct DeviceInfo {
  bool known = false;
  bool sm100 = false;
  int sm_count = 0;
};

// Compute capability and SM count of the current device (cached).
lg_status current_device(int* sm_count) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LG_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo local;
  DeviceInfo* info = (dev >= 0 && dev < 64) ? &cache[dev] : &local;
  if (!info->known) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return LG_ERR_CUDA;
    }
    info->sm100 = (major == 10 && minor == 0);
    info->sm_count = sms;
    info->known = true;
  }
  if (!info->sm100) return LG_ERR_NOT_SM100;
  *sm_count = info->sm_count;
  return LG_OK;
}

lg_status launched(cudaError_t e, uint64_t kernels) {
  if (e != cudaSuccess) return LG_ERR_CUDA;
  g_launches.fetch_add(kernels, std::memory_order_relaxed);
  return LG_OK;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace

extern "C" {

const char* lg_status_string(int status) {
  switch (status) {
    case LG_OK: return "ok";
    case LG_ERR_INVALID_ARG: return "invalid argument";
    case LG_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case LG_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case LG_ERR_WORKSPACE: return "workspace missing or too small";
    case LG_ERR_CUDA: return "CUDA call failed";
    case LG_ERR_DEVICE_TIMEOUT: return "bounded wait inside a kernel ran out";
    case LG_ERR_NOT_SM100: return "current device is not compute capability 10.0 (sm_100a)";
    default: return "unknown status";
  }
}

int lg_version(void) { return 10000; }

uint64_t lg_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void lg_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit_ns.store(limit_ns == 0 ? kDefaultWaitLimitNs : limit_ns, std::memory_order_relaxed);
}

lg_status lg_set_cluster_size(int g) {
  if (g != 0 && g != 1 && g != 2 && g != 4 && g != 8) return LG_ERR_INVALID_ARG;
  lg::set_cluster_override(g);
  return LG_OK;
}

lg_status lg_set_kernel_variant(int v) {
  if (v < 0 || v > 2) return LG_ERR_INVALID_ARG;
  lg::set_variant_override(v);
  return LG_OK;
}

lg_status lg_get_last_device_error(void* stream) {
  int v = 0;
  if (lg::read_and_clear_device_error(as_stream(stream), &v) != cudaSuccess) {
    cudaGetLastError();
    return LG_ERR_CUDA;
  }
  return (lg_status)v;
}

lg_status lg_lora_merge(int n_adapters, const float* const* A, const float* const* B, const int* ranks,
                        const float* scales, int d_in, int d_out, float* A_cat, float* B_cat, void* stream) {
  if (n_adapters < 1 || n_adapters > lg::kMaxAdapters || !A || !B || !ranks || !scales || !A_cat || !B_cat)
    return LG_ERR_INVALID_ARG;
  if (d_in < 1 || d_out < 1 || d_in > kMaxDim || d_out > kMaxDim || d_in % 4 || d_out % 4)
    return LG_ERR_UNSUPPORTED_SHAPE;
  lg::MergeAParams pa{};
  lg::MergeBParams pb{};
  int R = 0;
  for (int i = 0; i < n_adapters; ++i) {
    if (!A[i] || !B[i] || !std::isfinite(scales[i])) return LG_ERR_INVALID_ARG;
    if (ranks[i] < 1 || ranks[i] % 4 || ranks[i] > kMaxDim) return LG_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(A[i]) || !aligned16(B[i])) return LG_ERR_MISALIGNED;
    pa.A[i] = A[i];
    pa.scale[i] = scales[i];
    pa.row_off[i] = R;
    pb.B[i] = B[i];
    pb.col_off[i] = R;
    R += ranks[i];
    if (R > kMaxDim) return LG_ERR_UNSUPPORTED_SHAPE;
  }
  pa.row_off[n_adapters] = R;
  pb.col_off[n_adapters] = R;
  pa.n_adapters = pb.n_adapters = n_adapters;
  pa.d_in = d_in;
  pb.d_out = d_out;
  if (!aligned16(A_cat) || !aligned16(B_cat)) return LG_ERR_MISALIGNED;
  const uint64_t bytesA = 4ull * R * d_in, bytesB = 4ull * R * d_out;
  if (overlaps(A_cat, bytesA, B_cat, bytesB)) return LG_ERR_INVALID_ARG;
  for (int i = 0; i < n_adapters; ++i) {
    const uint64_t ai = 4ull * ranks[i] * d_in, bi = 4ull * ranks[i] * d_out;
    if (overlaps(A_cat, bytesA, A[i], ai) || overlaps(A_cat, bytesA, B[i], bi) ||
        overlaps(B_cat, bytesB, A[i], ai) || overlaps(B_cat, bytesB, B[i], bi))
      return LG_ERR_INVALID_ARG;
  }
  int sms = 0;
  lg_status st = current_device(&sms);
  if (st != LG_OK) return st;
  return launched(lg::launch_merge(pa, pb, A_cat, B_cat, sms, as_stream(stream)), 2);
}

size_t lg_mx_scale_bytes(int64_t rows, int K) {
  if (rows < 0 || K < 128 || K % 128 || K > kMaxDim) return 0;
  return (size_t)((rows + 127) / 128 * 128) * (size_t)(K / 32);
}

lg_status lg_mx_quantize(const void* in, int64_t rows, int K, void* codes, void* scales, void* stream) {
  if (rows < 0 || K < 0) return LG_ERR_INVALID_ARG;
  if (rows >= (int64_t)1 << 31 || K < 128 || K % 128 || K > kMaxDim) return LG_ERR_UNSUPPORTED_SHAPE;
  if (!in || !codes || !scales) return LG_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(codes)) return LG_ERR_MISALIGNED;
  const uint64_t bi = 2ull * rows * K, bc = 1ull * rows * K, bs = lg_mx_scale_bytes(rows, K);
  if (rows > 0 && (overlaps(in, bi, codes, bc) || overlaps(in, bi, scales, bs) || overlaps(codes, bc, scales, bs)))
    return LG_ERR_INVALID_ARG;
  if (rows == 0) return LG_OK;
  int sms = 0;
  lg_status st = current_device(&sms);
  if (st != LG_OK) return st;
  return launched(lg::launch_mx_quantize(reinterpret_cast<const uint16_t*>(in), rows, K,
                                         reinterpret_cast<uint8_t*>(codes), reinterpret_cast<uint8_t*>(scales), sms,
                                         as_stream(stream)),
                  1);
}

namespace {
// bf16 copies of A_cat [R, K] and B_cat [N, R], each padded to 256 bytes.
size_t factor_copy_bytes(int K, int N, int R) { return (size_t)(align256(2ull * R * K) + align256(2ull * N * R)); }
}  // namespace

size_t lg_lora_linear_workspace_size(int64_t M, int K, int N, int R) {
  if (M < 0 || K < 64 || N < 32 || K % 64 || N % 32 || K > kMaxDim || N > kMaxDim) return 0;
  if (R < 0 || R % 64 || R > kMaxRank) return 0;
  if (R == 0) return 0;
  return factor_copy_bytes(K, N, R);
}

size_t lg_lora_linear_euler_workspace_size(int64_t M, int K, int N, int R) {
  if (M < 0 || K < 64 || N < 1 || K % 64 || K > kMaxDim || N > kMaxDim) return 0;
  if (R < 0 || R % 64 || R > kMaxRank) return 0;
  if (R == 0) return 0;
  return factor_copy_bytes(K, N, R);
}

namespace {

// MXFP8 operands of lg_lora_linear_mxfp8 (null for the bf16 layer).
struct MxOperands {
  const void* xq;
  const void* xsf;
  const void* wq;
  const void* wsf;
};

// Fused SwiGLU output of lg_lora_linear_swiglu_mxfp8 (null otherwise).
struct SwigluOut {
  void* codes;
  void* scales;
};

// Fused Euler output of lg_lora_linear_euler (null otherwise).
struct EulerOut {
  float* z;
  void* z_bf16;
  int64_t frame_tokens;
  float dt;
};

// check_only: validate everything but the workspace (the caller brings its
// own, distinct from every argument) and the device, launch nothing.
lg_status lora_linear_impl(const void* x, const void* W, const float* A_cat, const float* B_cat, void* y, int64_t M,
                           int K, int N, int R, void* workspace, size_t ws_bytes, void* stream,
                           const MxOperands* mx, const SwigluOut* sw = nullptr, const EulerOut* eu = nullptr,
                           bool check_only = false) {
  if (M < 0 || K < 0 || N < 0 || R < 0) return LG_ERR_INVALID_ARG;
  // The Euler output takes any N >= 1 (its epilogue writes single values).
  const bool n_ok = eu ? N >= 1 : (N >= 32 && N % 32 == 0);
  if (M >= (int64_t)1 << 31 || K < 64 || !n_ok || K % 64 || K > kMaxDim || N > kMaxDim)
    return LG_ERR_UNSUPPORTED_SHAPE;
  if (R % 64 || R > kMaxRank) return LG_ERR_UNSUPPORTED_SHAPE;
  if (mx && K % 128) return LG_ERR_UNSUPPORTED_SHAPE;
  if (sw && (!mx || N % 256)) return LG_ERR_UNSUPPORTED_SHAPE;
  if (sw) {
    if (!sw->codes || !sw->scales) return LG_ERR_INVALID_ARG;
    if (!aligned16(sw->codes) || !aligned16(sw->scales)) return LG_ERR_MISALIGNED;
  }
  if (eu) {
    if (!eu->z || eu->frame_tokens < 1 || M % eu->frame_tokens || !std::isfinite(eu->dt)) return LG_ERR_INVALID_ARG;
    if (!aligned16(eu->z) || (eu->z_bf16 && !aligned16(eu->z_bf16))) return LG_ERR_MISALIGNED;
  }
  const bool no_y = sw || eu;
  if (!x || (!no_y && !y) || (!mx && !W)) return LG_ERR_INVALID_ARG;
  if (mx && (!mx->xq || !mx->xsf || !mx->wq || !mx->wsf)) return LG_ERR_INVALID_ARG;
  if (R > 0 && (!A_cat || !B_cat)) return LG_ERR_INVALID_ARG;
  if (!aligned16(x) || (!no_y && !aligned16(y)) || (!mx && !aligned16(W))) return LG_ERR_MISALIGNED;
  if (mx && (!aligned16(mx->xq) || !aligned16(mx->xsf) || !aligned16(mx->wq) || !aligned16(mx->wsf)))
    return LG_ERR_MISALIGNED;
  if (R > 0 && (!aligned16(A_cat) || !aligned16(B_cat))) return LG_ERR_MISALIGNED;
  const size_t need = R > 0 && !check_only ? factor_copy_bytes(K, N, R) : 0;
  if (R > 0 && !check_only) {
    if (!workspace || ws_bytes < need) return LG_ERR_WORKSPACE;
    if (!aligned16(workspace)) return LG_ERR_MISALIGNED;
  }
  const uint64_t bx = 2ull * M * K, bw = 2ull * N * K;
  // The output region: y, the SwiGLU codes and scales, or the latent z (and
  // its bf16 copy, checked here).
  const void* out = sw ? sw->codes : (eu ? eu->z : y);
  const uint64_t by = sw ? 1ull * M * (N / 2) : (eu ? 4ull * M * N : 2ull * M * N);
  if (eu && eu->z_bf16 && M > 0) {
    const uint64_t bb = 2ull * M * N;
    if (overlaps(eu->z_bf16, bb, eu->z, by) || overlaps(eu->z_bf16, bb, x, bx) || overlaps(eu->z_bf16, bb, W, bw) ||
        (R > 0 && (overlaps(eu->z_bf16, bb, A_cat, 4ull * R * K) || overlaps(eu->z_bf16, bb, B_cat, 4ull * N * R) ||
                   overlaps(eu->z_bf16, bb, workspace, need))))
      return LG_ERR_INVALID_ARG;
  }
  if (sw && M > 0) {
    const uint64_t bs = lg_mx_scale_bytes(M, N / 2);
    if (overlaps(sw->codes, by, sw->scales, bs) || overlaps(sw->scales, bs, x, bx) ||
        overlaps(sw->scales, bs, mx->xq, 1ull * M * K) || overlaps(sw->scales, bs, mx->wq, 1ull * N * K) ||
        (R > 0 && overlaps(sw->scales, bs, workspace, need)))
      return LG_ERR_INVALID_ARG;
  }
  y = const_cast<void*>(out);
  if (M > 0) {
    if (overlaps(y, by, x, bx) || (!mx && overlaps(y, by, W, bw))) return LG_ERR_INVALID_ARG;
    if (mx && (overlaps(y, by, mx->xq, 1ull * M * K) || overlaps(y, by, mx->wq, 1ull * N * K) ||
               overlaps(y, by, mx->xsf, lg_mx_scale_bytes(M, K)) || overlaps(y, by, mx->wsf, lg_mx_scale_bytes(N, K))))
      return LG_ERR_INVALID_ARG;
    if (R > 0 && (overlaps(y, by, A_cat, 4ull * R * K) || overlaps(y, by, B_cat, 4ull * N * R) ||
                  overlaps(y, by, workspace, need)))
      return LG_ERR_INVALID_ARG;
  }
  if (R > 0 && (overlaps(workspace, need, A_cat, 4ull * R * K) || overlaps(workspace, need, B_cat, 4ull * N * R) ||
                overlaps(workspace, need, x, bx) || (!mx && overlaps(workspace, need, W, bw))))
    return LG_ERR_INVALID_ARG;
  if (M == 0) return LG_OK;
  int sms = 0;
  lg_status st = current_device(&sms);
  if (st != LG_OK || check_only) return st;
  cudaStream_t s = as_stream(stream);
  uint16_t* wsA = nullptr;
  uint16_t* wsB = nullptr;
  if (R > 0) {
    wsA = reinterpret_cast<uint16_t*>(workspace);
    wsB = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(workspace) + align256(2ull * R * K));
    st = launched(lg::launch_prep_bf16(A_cat, B_cat, wsA, wsB, (int64_t)R * K, (int64_t)N * R, sms, s), 1);
    if (st != LG_OK) return st;
  }
  lg::LinearLaunch p;
  p.x = x;
  p.W = W;
  p.A_bf16 = wsA;
  p.B_bf16 = wsB;
  p.y = y;
  p.M = M;
  p.K = K;
  p.N = N;
  p.R = R;
  p.sm_count = sms;
  p.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  if (mx) {
    p.mx = true;
    p.xq = mx->xq;
    p.xsf = mx->xsf;
    p.wq = mx->wq;
    p.wsf = mx->wsf;
  }
  if (eu) {
    p.y = nullptr;
    p.eu_z = eu->z;
    p.eu_zb = eu->z_bf16;
    p.eu_frame = eu->frame_tokens;
    p.eu_dt = eu->dt;
  }
  if (sw) {
    p.y = nullptr;
    p.ffn = N / 2;
    p.q_codes = sw->codes;
    p.q_scales = sw->scales;
  }
  bool driver_failed = false;
  cudaError_t e = lg::launch_lora_linear(p, s, &driver_failed);
  if (e != cudaSuccess) cudaGetLastError();
  return launched(e, 1);
}

}  // namespace

}  // extern "C"

namespace lg {

int check_lora_linear(const void* x, const void* W, const float* A_cat, const float* B_cat, const void* y,
                      int64_t M, int K, int N, int R) {
  return lora_linear_impl(x, W, A_cat, B_cat, const_cast<void*>(y), M, K, N, R, nullptr, 0, nullptr, nullptr,
                          nullptr, nullptr, true);
}

bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    cudaGetLastError();
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace lg

extern "C" {

lg_status lg_lora_linear(const void* x, const void* W, const float* A_cat, const float* B_cat, void* y, int64_t M,
                         int K, int N, int R, void* workspace, size_t ws_bytes, void* stream) {
  return lora_linear_impl(x, W, A_cat, B_cat, y, M, K, N, R, workspace, ws_bytes, stream, nullptr);
}

lg_status lg_lora_linear_mxfp8(const void* x, const void* x_codes, const void* x_scales, const void* W_codes,
                               const void* W_scales, const float* A_cat, const float* B_cat, void* y, int64_t M,
                               int K, int N, int R, void* workspace, size_t ws_bytes, void* stream) {
  const MxOperands mx{x_codes, x_scales, W_codes, W_scales};
  return lora_linear_impl(x, nullptr, A_cat, B_cat, y, M, K, N, R, workspace, ws_bytes, stream, &mx);
}

lg_status lg_lora_linear_swiglu_mxfp8(const void* x, const void* x_codes, const void* x_scales, const void* W_codes,
                                      const void* W_scales, const float* A_cat, const float* B_cat, void* out_codes,
                                      void* out_scales, int64_t M, int K, int F, int R, void* workspace,
                                      size_t ws_bytes, void* stream) {
  if (F < 0 || F > kMaxDim / 2) return LG_ERR_UNSUPPORTED_SHAPE;
  if (F % 128) return LG_ERR_UNSUPPORTED_SHAPE;
  const MxOperands mx{x_codes, x_scales, W_codes, W_scales};
  const SwigluOut sw{out_codes, out_scales};
  return lora_linear_impl(x, nullptr, A_cat, B_cat, nullptr, M, K, 2 * F, R, workspace, ws_bytes, stream, &mx, &sw);
}

lg_status lg_lora_linear_euler(const void* x, const void* W, const float* A_cat, const float* B_cat, float* z,
                               void* z_bf16, int64_t M, int K, int N, int R, int64_t frame_tokens, float sigma,
                               float sigma_next, void* workspace, size_t ws_bytes, void* stream) {
  if (!std::isfinite(sigma) || !std::isfinite(sigma_next)) return LG_ERR_INVALID_ARG;
  // The step is taken in FP32, as lg_euler_step takes it.
  const EulerOut eu{z, z_bf16, frame_tokens, sigma_next - sigma};
  return lora_linear_impl(x, W, A_cat, B_cat, nullptr, M, K, N, R, workspace, ws_bytes, stream, nullptr, nullptr, &eu);
}

lg_status lg_renoise(const float* up, float* x, int64_t n, float sigma, uint64_t seed, uint64_t offset,
                     void* stream) {
  if (n < 0 || !std::isfinite(sigma) || sigma < 0.0f || sigma > 1.0f || offset % 4) return LG_ERR_INVALID_ARG;
  if (n == 0) return LG_OK;
  if (!up || !x) return LG_ERR_INVALID_ARG;
  if (!aligned16(up) || !aligned16(x)) return LG_ERR_MISALIGNED;
  if (up != x && overlaps(up, 4ull * n, x, 4ull * n)) return LG_ERR_INVALID_ARG;
  int sms = 0;
  lg_status st = current_device(&sms);
  if (st != LG_OK) return st;
  return launched(lg::launch_renoise(up, x, n, sigma, seed, offset, sms, as_stream(stream)), 1);
}

lg_status lg_euler_step(float* x, const float* v, int64_t n, float sigma, float sigma_next, void* stream) {
  if (n < 0 || !std::isfinite(sigma) || !std::isfinite(sigma_next)) return LG_ERR_INVALID_ARG;
  if (n == 0) return LG_OK;
  if (!x || !v) return LG_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(v)) return LG_ERR_MISALIGNED;
  if (overlaps(x, 4ull * n, v, 4ull * n)) return LG_ERR_INVALID_ARG;
  int sms = 0;
  lg_status st = current_device(&sms);
  if (st != LG_OK) return st;
  const float dt = sigma_next - sigma;
  return launched(lg::launch_euler(x, v, n, dt, sms, as_stream(stream)), 1);
}

lg_status lg_shift_ladder(float sigma0, int n_steps, double shift, float* out, int cap, int* len) {
  if (!out || !len || !(sigma0 > 0.0f && sigma0 <= 1.0f) || n_steps < 1 || n_steps > 4096 ||
      !std::isfinite(shift) || !(shift > 0.0)) {
    return LG_ERR_INVALID_ARG;
  }
  float ladder[4097 + 1];
  int count = 0;
  ladder[count++] = sigma0;
  for (int k = 0; k <= n_steps; ++k) {
    const double t = 1.0 - (double)k / (double)n_steps;
    const double num = shift * t;
    const double den = 1.0 + (shift - 1.0) * t;
    const float sig = (float)(num / den);
    if (sig < sigma0) ladder[count++] = sig;
  }
  if (cap < count) return LG_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) out[i] = ladder[i];
  *len = count;
  return LG_OK;
}

lg_status lg_philox_u32(uint32_t* out, int64_t n_blocks, uint64_t seed, uint64_t block_offset, void* stream) {
  if (n_blocks < 0) return LG_ERR_INVALID_ARG;
  if (n_blocks == 0) return LG_OK;
  if (!out) return LG_ERR_INVALID_ARG;
  if (!aligned16(out)) return LG_ERR_MISALIGNED;
  int sms = 0;
  lg_status st = current_device(&sms);
  if (st != LG_OK) return st;
  return launched(lg::launch_philox_u32(out, n_blocks, seed, block_offset, sms, as_stream(stream)), 1);
}

lg_status lg_philox_normal(float* eps, int64_t n, uint64_t seed, uint64_t offset, void* stream) {
  if (n < 0 || offset % 4) return LG_ERR_INVALID_ARG;
  if (n == 0) return LG_OK;
  if (!eps) return LG_ERR_INVALID_ARG;
  if (!aligned16(eps)) return LG_ERR_MISALIGNED;
  int sms = 0;
  lg_status st = current_device(&sms);
  if (st != LG_OK) return st;
  return launched(lg::launch_philox_normal(eps, n, seed, offset, sms, as_stream(stream)), 1);
}

}  // extern "C"
