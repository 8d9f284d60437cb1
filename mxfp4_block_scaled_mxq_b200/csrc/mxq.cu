// mxq.cu -- libmxq: the C ABI of include/mxq.h (host-side validation, TMA tensor-map
// encoding and launches) over the sm_100a kernels in quantize.cuh, gemm_pair.cuh and gemm_swap.cuh.
// One translation unit, so the library's device status word exists exactly once.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "mxq.h"
#include "gemm_common.cuh"
#include "gemm_pair.cuh"
#include "gemm_swap.cuh"
#include "policy.cuh"
#include "attention.cuh"
#include "quantize.cuh"

// Scratch of mxq_linear_w4a4_static: the quantised activations of one call, per device.
constexpr int64_t kStaticScratchBytes = MXQ_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_linear_scratch[kStaticScratchBytes];

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

constexpr int kMaxDevices = 64;

// Per-device facts, looked up once per device.
struct DeviceInfo {
  bool ok = false;
  int index = -1;
  int sm_count = 0;
};

DeviceInfo device_info(int dev) {
  static DeviceInfo info[kMaxDevices];
  static std::once_flag once[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return {};
  std::call_once(once[dev], [dev] {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return;
    info[dev].ok = (p.major == 10 && p.minor == 0);
    info[dev].index = dev;
    info[dev].sm_count = p.multiProcessorCount;
  });
  return info[dev];
}

mxq_status current_device(DeviceInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXQ_ERR_CUDA;
  *out = device_info(dev);
  if (!out->ok) return MXQ_ERR_UNSUPPORTED;
  return MXQ_OK;
}

// One-time set-up per device.  Kernel attributes (the opt-in shared memory size), the
// occupancy they allow and symbol addresses belong to one device's context, so every device
// runs `setup` (with that device current) before its first launch.  Only a successful set-up
// is remembered: a failed one returns false and runs again on the next call.
class PerDevice {
 public:
  template <typename Setup>
  bool ensure(int dev, Setup&& setup) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    if (done_[dev].load(std::memory_order_acquire)) return true;
    std::lock_guard<std::mutex> lock(mu_);
    if (!done_[dev].load(std::memory_order_relaxed) && setup()) done_[dev].store(true, std::memory_order_release);
    return done_[dev].load(std::memory_order_relaxed);
  }

 private:
  std::mutex mu_;
  std::atomic<bool> done_[kMaxDevices] = {};
};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

mxq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

// Launch with programmatic stream serialisation: the kernel may start while the kernel
// before it in the stream (normally the activation quantiser, which lets dependents start)
// finishes; the kernel executes griddepcontrol.wait before it reads any input.
template <typename... KArgs, typename... Args>
mxq_status launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t stream,
                            Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

// 2-D tensor map over a row-major [rows][cols] matrix.
bool make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D tensor map over a swizzled scale-factor buffer of `rows` rows and K columns:
// (byte in 128-byte chunk, chunk in atom, atom along K, 128-row tile); a box of
// {128, 4, atoms, row_tiles} lands as contiguous 512-byte atoms, [row tile][atom].
bool make_tmap_sf(CUtensorMap* m, const void* base, int64_t rows, int64_t K, uint32_t atoms, uint32_t row_tiles) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  const uint64_t atoms_per_row_tile = static_cast<uint64_t>(K) / 128;
  const cuuint64_t dims[4] = {128, 4, atoms_per_row_tile, static_cast<cuuint64_t>((rows + 127) / 128)};
  const cuuint64_t strides[3] = {128, 512, atoms_per_row_tile * 512};
  const cuuint32_t box[4] = {128, 4, atoms, row_tiles};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Two-CTA path (one 256 x 192 tile per CTA pair), persistent over as many pairs as
// can be resident at once.
template <bool kW4A8>
mxq_status launch_gemm_pair(const DeviceInfo& dev, const void* a, const void* a_sf, const void* b, const void* b_sf,
                            int64_t M, int64_t N, int64_t K, float alpha, const void* bias, void* d, int64_t ldd,
                            cudaStream_t stream) {
  using S = mxq::PairShape<kW4A8>;
  auto kernel = mxq::mx_gemm_pair_kernel<kW4A8>;
  static PerDevice setup;
  static int max_clusters_of[kMaxDevices];
  const bool ready = setup.ensure(dev.index, [&] {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes) != cudaSuccess)
      return false;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(mxq::kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = S::kSmemBytes;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) return false;
    max_clusters_of[dev.index] = n;
    return true;
  });
  if (!ready) return MXQ_ERR_CUDA;
  const int max_clusters = max_clusters_of[dev.index];

  CUtensorMap ta, tb, tsa, tsb;
  bool ok;
  if (kW4A8) {
    ok = make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, K, M, K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, b, K, N, K / 2, 128, S::kBRows,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    tsa = tb;  // unused: E4M3 activations carry unit scales
  } else {
    ok = make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, K / 2, M, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b, K / 2, N, K / 2, 128, S::kBRows,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_tmap_sf(&tsa, a_sf, M, K, S::kAtoms, 1);
  }
  ok = ok && make_tmap_sf(&tsb, b_sf, N, K, S::kAtoms, 2);
  if (!ok) return MXQ_ERR_CUDA;
  const int64_t tiles = ((M + 255) / 256) * ((N + mxq::kBN - 1) / mxq::kBN);
  const int clusters = static_cast<int>(tiles < max_clusters ? tiles : max_clusters);
  // 32-byte output stores need 32-byte aligned rows
  const int d_vec32 = (ldd % 16 == 0 && aligned(d, 32)) ? 1 : 0;
  return launch_dependent(kernel, dim3(static_cast<unsigned>(2 * clusters), 1, 1), dim3(mxq::kGemmThreads, 1, 1),
                          S::kSmemBytes, stream, ta, tb, tsa, tsb, static_cast<__nv_bfloat16*>(d), ldd, d_vec32,
                          static_cast<const __nv_bfloat16*>(bias), static_cast<int>(M), static_cast<int>(N),
                          static_cast<int>(K), alpha);
}

// Device address of g_linear_scratch on the current device `dev`, looked up once per device
// (a failed lookup is retried on the next call).
void* static_scratch(int dev) {
  static PerDevice setup;
  static void* addr[kMaxDevices];
  const bool ready = setup.ensure(dev, [dev] {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || !p) return false;
    addr[dev] = p;
    return true;
  });
  return ready ? addr[dev] : nullptr;
}

// Workspace of the quantized linear layer: the quantised activations (codes, then scales).
struct LinearWorkspace {
  int64_t codes = 0, sf = 0, bytes = 0;
};

LinearWorkspace linear_workspace(int64_t M, int64_t K) {
  auto up = [](int64_t v) { return (v + 1023) / 1024 * 1024; };
  LinearWorkspace w;
  w.codes = 0;
  w.sf = up(M * (K / 2));
  w.bytes = w.sf + up((M + 127) / 128 * 128 * ((K / 32 + 3) / 4 * 4));
  return w;
}

// Few tokens (M <= 128): D^T = W X^T with the weights on the MMA's 128-row side; one
// kernel instance per token tile width Mt (the tokens rounded up to 16).
template <bool kW4A8, int Mt>
mxq_status launch_gemm_swap_mt(const DeviceInfo& dev, const CUtensorMap& tw, const CUtensorMap& tt,
                               const CUtensorMap& tsw, const CUtensorMap& tst, int64_t M, int64_t N, int64_t K,
                               float alpha, const void* bias, void* d, int64_t ldd, cudaStream_t stream) {
  using S = mxq::SwapShape<kW4A8>;
  auto kernel = mxq::mx_gemm_swap_kernel<kW4A8, Mt>;
  constexpr int kMaxSmem = 232448;  // opt-in shared memory per CTA on sm_100
  static PerDevice setup;
  if (!setup.ensure(dev.index, [&] {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem) == cudaSuccess;
      }))
    return MXQ_ERR_CUDA;
  int stages = (kMaxSmem - S::kFixedBytes - S::out_bytes(Mt)) / S::stage_bytes(Mt);
  stages = stages > mxq::kSwapMaxStages ? mxq::kSwapMaxStages : stages;
  const int smem = S::kFixedBytes + S::out_bytes(Mt) + stages * S::stage_bytes(Mt);
  // D [M][N] BF16 written as [Mt][128] boxes (row stride ldd * 2 bytes: ldd % 8 == 0)
  CUtensorMap td;
  if (!make_tmap_2d(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d, N, M, ldd * 2, 128, Mt, CU_TENSOR_MAP_SWIZZLE_NONE))
    return MXQ_ERR_CUDA;
  const int64_t tiles = (N + 127) / 128;
  const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  return launch_dependent(kernel, dim3(static_cast<unsigned>(grid), 1, 1), dim3(mxq::kSwapThreads, 1, 1), smem,
                          stream, tw, tt, tsw, tst, td, static_cast<const __nv_bfloat16*>(bias), static_cast<int>(M),
                          static_cast<int>(N), static_cast<int>(K), alpha, stages);
}

template <bool kW4A8>
mxq_status launch_gemm_swap(const DeviceInfo& dev, const void* a, const void* a_sf, const void* b, const void* b_sf,
                            int64_t M, int64_t N, int64_t K, float alpha, const void* bias, void* d, int64_t ldd,
                            cudaStream_t stream) {
  using S = mxq::SwapShape<kW4A8>;
  const int Mt = static_cast<int>((M + 15) / 16 * 16);
  CUtensorMap tw, tt, tsw, tst;
  bool ok;
  if (kW4A8) {
    ok = make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, b, K, N, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_tmap_2d(&tt, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, K, M, K, 128, Mt, CU_TENSOR_MAP_SWIZZLE_128B);
    tst = tw;  // unused: E4M3 tokens carry unit scales
  } else {
    ok = make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, b, K / 2, N, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_tmap_2d(&tt, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, K / 2, M, K / 2, 128, Mt, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_tmap_sf(&tst, a_sf, M, K, S::kAtoms, 1);
  }
  ok = ok && make_tmap_sf(&tsw, b_sf, N, K, S::kAtoms, 1);
  if (!ok) return MXQ_ERR_CUDA;
  switch (Mt) {
#define MXQ_SWAP_CASE(T) \
  case T: return launch_gemm_swap_mt<kW4A8, T>(dev, tw, tt, tsw, tst, M, N, K, alpha, bias, d, ldd, stream);
    MXQ_SWAP_CASE(16) MXQ_SWAP_CASE(32) MXQ_SWAP_CASE(48) MXQ_SWAP_CASE(64)
    MXQ_SWAP_CASE(80) MXQ_SWAP_CASE(96) MXQ_SWAP_CASE(112) MXQ_SWAP_CASE(128)
#undef MXQ_SWAP_CASE
    default: return MXQ_ERR_SHAPE;
  }
}

template <bool kW4A8>
mxq_status launch_gemm(const void* a, const void* a_sf, const void* b, const void* b_sf, int64_t M, int64_t N,
                       int64_t K, float alpha, const void* bias, void* d, int64_t ldd, cudaStream_t stream) {
  DeviceInfo dev;
  mxq_status st = current_device(&dev);
  if (st != MXQ_OK) return st;
  if (M > mxq::kBM) return launch_gemm_pair<kW4A8>(dev, a, a_sf, b, b_sf, M, N, K, alpha, bias, d, ldd, stream);
  return launch_gemm_swap<kW4A8>(dev, a, a_sf, b, b_sf, M, N, K, alpha, bias, d, ldd, stream);
}

mxq_status check_gemm_shapes(const void* a, const void* b, const void* b_sf, const void* d, int64_t M, int64_t N,
                             int64_t K, int64_t ldd, const void* bias) {
  if (!a || !b || !b_sf || !d) return MXQ_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 128 || K % 128 != 0) return MXQ_ERR_SHAPE;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || K > (int64_t(1) << 22)) return MXQ_ERR_SHAPE;
  const int64_t tiles = ((M + mxq::kBM - 1) / mxq::kBM) * ((N + mxq::kBN - 1) / mxq::kBN);
  if (tiles > INT32_MAX) return MXQ_ERR_SHAPE;  // tile indices are 32-bit in the kernel
  if (ldd < N || ldd % 8 != 0) return MXQ_ERR_ALIGN;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(b_sf, 16) || !aligned(d, 16)) return MXQ_ERR_ALIGN;
  if (bias && !aligned(bias, 16)) return MXQ_ERR_ALIGN;
  return MXQ_OK;
}

mxq_status launch_mxfp4(bool weight, const void* x, int64_t rows, int64_t K, int64_t ld, mxq_scale_rule rule,
                        int hadamard, void* codes, void* sf, cudaStream_t stream) {
  // grid.x: 128-column tiles (K <= 2^22 keeps it <= 32768), grid.y: 128-row tiles.
  const dim3 grid(static_cast<unsigned>((K + 127) / 128), static_cast<unsigned>((rows + 127) / 128));
  const auto* xp = static_cast<const uint16_t*>(x);
  auto* cp = static_cast<uint8_t*>(codes);
  auto* sp = static_cast<uint8_t*>(sf);
  const bool uos = rule == MXQ_SCALE_UOS;
  const int sel = (hadamard ? 2 : 0) | (uos ? 1 : 0);
  if (weight) {
    switch (sel) {
      case 0: mxq::pack_weight_mxfp4_kernel<false, false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ld, cp, sp); break;
      case 1: mxq::pack_weight_mxfp4_kernel<false, true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ld, cp, sp); break;
      case 2: mxq::pack_weight_mxfp4_kernel<true, false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ld, cp, sp); break;
      default: mxq::pack_weight_mxfp4_kernel<true, true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ld, cp, sp); break;
    }
  } else {
    switch (sel) {
      case 0: mxq::quantize_act_mxfp4_kernel<false, false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ld, cp, sp); break;
      case 1: mxq::quantize_act_mxfp4_kernel<false, true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ld, cp, sp); break;
      case 2: mxq::quantize_act_mxfp4_kernel<true, false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ld, cp, sp); break;
      default: mxq::quantize_act_mxfp4_kernel<true, true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ld, cp, sp); break;
    }
  }
  return launch_status();
}

mxq_status check_quant_args(const void* x, int64_t rows, int64_t K, int64_t ld, mxq_scale_rule rule, int hadamard,
                            const void* q, const void* sf) {
  if (!x || !q || !sf) return MXQ_ERR_INVALID_ARG;
  if (rule != MXQ_SCALE_OCP && rule != MXQ_SCALE_UOS) return MXQ_ERR_INVALID_ARG;
  // rows <= 65535 * 128 keeps grid.y within its limit
  if (rows < 1 || rows > int64_t(65535) * 128 || K < 32 || K % 32 != 0 || K > (int64_t(1) << 22)) return MXQ_ERR_SHAPE;
  if (hadamard && K % 128 != 0) return MXQ_ERR_SHAPE;
  // 16 BF16 values per load: 16-byte aligned rows (32-byte loads where rows allow them)
  if (ld < K || ld % 8 != 0) return MXQ_ERR_ALIGN;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sf, 16)) return MXQ_ERR_ALIGN;
  return MXQ_OK;
}

}  // namespace

extern "C" {

const char* mxq_status_string(mxq_status s) {
  switch (s) {
    case MXQ_OK: return "MXQ_OK";
    case MXQ_ERR_INVALID_ARG: return "MXQ_ERR_INVALID_ARG";
    case MXQ_ERR_SHAPE: return "MXQ_ERR_SHAPE";
    case MXQ_ERR_ALIGN: return "MXQ_ERR_ALIGN";
    case MXQ_ERR_UNSUPPORTED: return "MXQ_ERR_UNSUPPORTED";
    case MXQ_ERR_CUDA: return "MXQ_ERR_CUDA";
    case MXQ_ERR_TIMEOUT: return "MXQ_ERR_TIMEOUT";
  }
  return "MXQ_ERR_UNKNOWN";
}

int64_t mxq_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 1 || K < 32 || K % 32 != 0) return -1;
  return (rows + 127) / 128 * 128 * ((K / 32 + 3) / 4 * 4);
}

mxq_status mxq_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, mxq_act_format fmt,
                            mxq_scale_rule rule, int hadamard128, float act_scale, void* q_out, void* sf_out,
                            mxq_stream_t stream) {
  if (fmt == MXQ_ACT_FP8_E4M3) {
    if (!x_bf16 || !q_out || sf_out) return MXQ_ERR_INVALID_ARG;
    if (rule != MXQ_SCALE_OCP || hadamard128) return MXQ_ERR_INVALID_ARG;
    if (!(act_scale > 0.f) || !std::isfinite(act_scale)) return MXQ_ERR_INVALID_ARG;
    if (M < 1 || M > (int64_t(1) << 31) || K < 32 || K % 32 != 0 || K > (int64_t(1) << 22)) return MXQ_ERR_SHAPE;
    if (ldx < K || ldx % 8 != 0) return MXQ_ERR_ALIGN;
    if (!aligned(x_bf16, 16) || !aligned(q_out, 16)) return MXQ_ERR_ALIGN;
    const float inv = 1.0f / act_scale;  // fl32(1 / s), IEEE division on the host
    if (!std::isfinite(inv)) return MXQ_ERR_INVALID_ARG;
    DeviceInfo dev;
    mxq_status st = current_device(&dev);
    if (st != MXQ_OK) return st;
    // grid.x: groups of 64 chunk columns (K <= 2^22: at most 4096); grid.y: groups of
    // kFp8Rows rows, at most 65535 (the kernel strides over the rest)
    const int64_t gx = (K / 16 + 63) / 64;
    const int64_t gy = std::min<int64_t>((M + mxq::kFp8Rows - 1) / mxq::kFp8Rows, 65535);
    const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    mxq::quantize_act_fp8_kernel<<<grid, mxq::kQuantThreads, 0, stream>>>(
        static_cast<const uint16_t*>(x_bf16), M, K, ldx, inv, static_cast<uint8_t*>(q_out));
    return launch_status();
  }
  if (fmt != MXQ_ACT_MXFP4) return MXQ_ERR_INVALID_ARG;
  mxq_status st = check_quant_args(x_bf16, M, K, ldx, rule, hadamard128, q_out, sf_out);
  if (st != MXQ_OK) return st;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MXQ_OK) return st;
  return launch_mxfp4(false, x_bf16, M, K, ldx, rule, hadamard128, q_out, sf_out, stream);
}

mxq_status mxq_pack_weight(const void* w_bf16, int64_t N, int64_t K, int64_t ldw, mxq_scale_rule rule,
                           int hadamard128, void* codes_out, void* sf_out, mxq_stream_t stream) {
  mxq_status st = check_quant_args(w_bf16, N, K, ldw, rule, hadamard128, codes_out, sf_out);
  if (st != MXQ_OK) return st;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MXQ_OK) return st;
  return launch_mxfp4(true, w_bf16, N, K, ldw, rule, hadamard128, codes_out, sf_out, stream);
}

mxq_status mxq_gemm_w4a4(const void* a_codes, const void* a_sf, const void* b_codes, const void* b_sf, int64_t M,
                         int64_t N, int64_t K, float alpha, const void* bias_bf16, void* d_bf16, int64_t ldd,
                         mxq_stream_t stream) {
  if (!a_sf) return MXQ_ERR_INVALID_ARG;
  if (!std::isfinite(alpha)) return MXQ_ERR_INVALID_ARG;
  mxq_status st = check_gemm_shapes(a_codes, b_codes, b_sf, d_bf16, M, N, K, ldd, bias_bf16);
  if (st != MXQ_OK) return st;
  if (!aligned(a_sf, 16)) return MXQ_ERR_ALIGN;
  return launch_gemm<false>(a_codes, a_sf, b_codes, b_sf, M, N, K, alpha, bias_bf16, d_bf16, ldd, stream);
}

mxq_status mxq_gemm_w4a8(const void* a_e4m3, float act_scale, const void* b_codes, const void* b_sf, int64_t M,
                         int64_t N, int64_t K, const void* bias_bf16, void* d_bf16, int64_t ldd,
                         mxq_stream_t stream) {
  if (!(act_scale > 0.f) || !std::isfinite(act_scale)) return MXQ_ERR_INVALID_ARG;
  mxq_status st = check_gemm_shapes(a_e4m3, b_codes, b_sf, d_bf16, M, N, K, ldd, bias_bf16);
  if (st != MXQ_OK) return st;
  if (!aligned(b_codes, 32)) return MXQ_ERR_ALIGN;  // 16U4_ALIGN16B tensor maps need 32-byte bases
  return launch_gemm<true>(a_e4m3, nullptr, b_codes, b_sf, M, N, K, act_scale, bias_bf16, d_bf16, ldd, stream);
}

mxq_status mxq_dequant_mxfp4(const void* codes, const void* sf, int64_t rows, int64_t K, void* out_bf16,
                             int64_t ldo, mxq_stream_t stream) {
  if (!codes || !sf || !out_bf16) return MXQ_ERR_INVALID_ARG;
  if (rows < 1 || rows > (int64_t(1) << 31) || K < 32 || K % 32 != 0 || K > (int64_t(1) << 22)) return MXQ_ERR_SHAPE;
  if (ldo < K || ldo % 8 != 0) return MXQ_ERR_ALIGN;
  if (!aligned(codes, 16) || !aligned(out_bf16, 16)) return MXQ_ERR_ALIGN;
  DeviceInfo dev;
  mxq_status st = current_device(&dev);
  if (st != MXQ_OK) return st;
  const int64_t units = rows * (K / 16);
  const int64_t per_block = int64_t(mxq::kQuantThreads) * mxq::kDequantUnroll;
  int64_t blocks = (units + per_block - 1) / per_block;
  // Grid-stride: exactly the CTAs that fit at once, so none starts late (a second, partial
  // round of a latency-bound kernel costs as much as a full one).
  static PerDevice setup;
  static int resident_of[kMaxDevices];
  setup.ensure(dev.index, [&] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, mxq::dequant_mxfp4_kernel, mxq::kQuantThreads, 0) !=
            cudaSuccess || n < 1)
      return false;
    resident_of[dev.index] = n;
    return true;
  });
  const int resident = resident_of[dev.index] > 0 ? resident_of[dev.index] : 1;
  const int64_t cap = static_cast<int64_t>(dev.sm_count) * resident;
  if (blocks > cap) blocks = cap;
  mxq::dequant_mxfp4_kernel<<<static_cast<unsigned>(blocks), mxq::kQuantThreads, 0, stream>>>(
      static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(sf), rows, K,
      static_cast<uint16_t*>(out_bf16), ldo);
  return launch_status();
}

mxq_status mxq_qdq_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, mxq_act_format fmt,
                       mxq_scale_rule rule, int hadamard128, float act_scale, void* out_bf16, int64_t ldo,
                       mxq_stream_t stream) {
  if (!x_bf16 || !out_bf16) return MXQ_ERR_INVALID_ARG;
  if (fmt != MXQ_ACT_MXFP4 && fmt != MXQ_ACT_FP8_E4M3) return MXQ_ERR_INVALID_ARG;
  if (rule != MXQ_SCALE_OCP && rule != MXQ_SCALE_UOS) return MXQ_ERR_INVALID_ARG;
  float inv = 0.f;
  if (fmt == MXQ_ACT_FP8_E4M3) {
    if (rule != MXQ_SCALE_OCP || hadamard128) return MXQ_ERR_INVALID_ARG;
    if (!(act_scale > 0.f) || !std::isfinite(act_scale)) return MXQ_ERR_INVALID_ARG;
    inv = 1.0f / act_scale;  // fl32(1 / s), as in the quantiser
    if (!std::isfinite(inv)) return MXQ_ERR_INVALID_ARG;
  }
  const int64_t max_rows = fmt == MXQ_ACT_FP8_E4M3 ? (int64_t(1) << 31) : int64_t(65535) * 128;
  if (M < 1 || M > max_rows || K < 32 || K % 32 != 0 || K > (int64_t(1) << 22)) return MXQ_ERR_SHAPE;
  if (hadamard128 && K % 128 != 0) return MXQ_ERR_SHAPE;
  if (ldx < K || ldx % 8 != 0 || ldo < K || ldo % 8 != 0) return MXQ_ERR_ALIGN;
  if (!aligned(x_bf16, 16) || !aligned(out_bf16, 16)) return MXQ_ERR_ALIGN;
  DeviceInfo dev;
  mxq_status st = current_device(&dev);
  if (st != MXQ_OK) return st;
  const auto* xp = static_cast<const uint16_t*>(x_bf16);
  auto* op = static_cast<uint16_t*>(out_bf16);
  if (fmt == MXQ_ACT_FP8_E4M3) {
    const int64_t chunks = M * (K / 16);
    int64_t blocks = (chunks + mxq::kQuantThreads - 1) / mxq::kQuantThreads;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * 16;
    if (blocks > cap) blocks = cap;
    mxq::qdq_act_fp8_kernel<<<static_cast<unsigned>(blocks), mxq::kQuantThreads, 0, stream>>>(xp, M, K, ldx, inv,
                                                                                             act_scale, op, ldo);
    return launch_status();
  }
  const dim3 grid(static_cast<unsigned>((K + 127) / 128), static_cast<unsigned>((M + 127) / 128));
  const int sel = (hadamard128 ? 2 : 0) | (rule == MXQ_SCALE_UOS ? 1 : 0);
  switch (sel) {
    case 0: mxq::qdq_act_mxfp4_kernel<false, false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, M, K, ldx, op, ldo); break;
    case 1: mxq::qdq_act_mxfp4_kernel<false, true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, M, K, ldx, op, ldo); break;
    case 2: mxq::qdq_act_mxfp4_kernel<true, false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, M, K, ldx, op, ldo); break;
    default: mxq::qdq_act_mxfp4_kernel<true, true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, M, K, ldx, op, ldo); break;
  }
  return launch_status();
}

mxq_status mxq_channel_absmax(const void* x_bf16, int64_t rows, int64_t K, int64_t ldx, int hadamard128,
                              int accumulate, float* amax_out, mxq_stream_t stream) {
  if (!amax_out) return MXQ_ERR_INVALID_ARG;
  // same tiling and limits as the quantiser (the scale pointers are not used)
  mxq_status st = check_quant_args(x_bf16, rows, K, ldx, MXQ_SCALE_OCP, hadamard128, amax_out, amax_out);
  if (st != MXQ_OK) return st;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MXQ_OK) return st;
  if (!accumulate && cudaMemsetAsync(amax_out, 0, static_cast<size_t>(K) * sizeof(float), stream) != cudaSuccess)
    return MXQ_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>((K + 127) / 128), static_cast<unsigned>((rows + 127) / 128));
  const auto* xp = static_cast<const uint16_t*>(x_bf16);
  if (hadamard128)
    mxq::channel_absmax_kernel<true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ldx, amax_out);
  else
    mxq::channel_absmax_kernel<false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ldx, amax_out);
  return launch_status();
}

mxq_status mxq_smooth_factors(const float* amax_x, const float* amax_w, int64_t K, float alpha, float* lambda_out,
                              float* inv_lambda_out, mxq_stream_t stream) {
  if (!amax_x || !amax_w || !lambda_out || !inv_lambda_out) return MXQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.f && alpha <= 1.f)) return MXQ_ERR_INVALID_ARG;
  if (K < 1 || K > (int64_t(1) << 22)) return MXQ_ERR_SHAPE;
  DeviceInfo dev;
  mxq_status st = current_device(&dev);
  if (st != MXQ_OK) return st;
  const unsigned blocks = static_cast<unsigned>((K + 255) / 256);
  mxq::smooth_factors_kernel<<<blocks, 256, 0, stream>>>(amax_x, amax_w, K, alpha, lambda_out, inv_lambda_out);
  return launch_status();
}

mxq_status mxq_quantize_smooth(const void* x_bf16, int64_t rows, int64_t K, int64_t ldx, mxq_scale_rule rule,
                               int hadamard128, const float* chan_scale, void* codes_out, void* sf_out,
                               mxq_stream_t stream) {
  if (!chan_scale) return MXQ_ERR_INVALID_ARG;
  mxq_status st = check_quant_args(x_bf16, rows, K, ldx, rule, hadamard128, codes_out, sf_out);
  if (st != MXQ_OK) return st;
  if (!aligned(chan_scale, 16)) return MXQ_ERR_ALIGN;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MXQ_OK) return st;
  const dim3 grid(static_cast<unsigned>((K + 127) / 128), static_cast<unsigned>((rows + 127) / 128));
  const auto* xp = static_cast<const uint16_t*>(x_bf16);
  auto* cp = static_cast<uint8_t*>(codes_out);
  auto* sp = static_cast<uint8_t*>(sf_out);
  const int sel = (hadamard128 ? 2 : 0) | (rule == MXQ_SCALE_UOS ? 1 : 0);
  switch (sel) {
    case 0: mxq::quantize_smooth_mxfp4_kernel<false, false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ldx, chan_scale, cp, sp); break;
    case 1: mxq::quantize_smooth_mxfp4_kernel<false, true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ldx, chan_scale, cp, sp); break;
    case 2: mxq::quantize_smooth_mxfp4_kernel<true, false><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ldx, chan_scale, cp, sp); break;
    default: mxq::quantize_smooth_mxfp4_kernel<true, true><<<grid, mxq::kQuantThreads, 0, stream>>>(xp, rows, K, ldx, chan_scale, cp, sp); break;
  }
  return launch_status();
}

mxq_status mxq_sqnr_accumulate(const void* y_bf16, int64_t ldy, const void* ref_bf16, int64_t ldr, int64_t M,
                               int64_t N, int accumulate, double* acc, mxq_stream_t stream) {
  if (!y_bf16 || !ref_bf16 || !acc) return MXQ_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || M > (int64_t(1) << 31) || N > (int64_t(1) << 31)) return MXQ_ERR_SHAPE;
  if (ldy < N || ldr < N || ldy % 8 != 0 || ldr % 8 != 0) return MXQ_ERR_ALIGN;
  if (!aligned(y_bf16, 16) || !aligned(ref_bf16, 16) || !aligned(acc, 8)) return MXQ_ERR_ALIGN;
  DeviceInfo dev;
  mxq_status st = current_device(&dev);
  if (st != MXQ_OK) return st;
  if (!accumulate && cudaMemsetAsync(acc, 0, 2 * sizeof(double), stream) != cudaSuccess) return MXQ_ERR_CUDA;
  const int64_t chunks = M * ((N + 7) / 8);
  int64_t blocks = (chunks + mxq::kSqnrThreads - 1) / mxq::kSqnrThreads;
  const int64_t cap = static_cast<int64_t>(dev.sm_count) * 8;
  if (blocks > cap) blocks = cap;
  mxq::sqnr_sums_kernel<<<static_cast<unsigned>(blocks), mxq::kSqnrThreads, 0, stream>>>(
      static_cast<const uint16_t*>(y_bf16), ldy, static_cast<const uint16_t*>(ref_bf16), ldr, M, N, acc);
  return launch_status();
}

double mxq_sqnr_db(double signal, double noise) {
  if (!(noise > 0.0)) return HUGE_VAL;
  if (!(signal > 0.0)) return -HUGE_VAL;
  return 10.0 * std::log10(signal / noise);
}

mxq_precision mxq_select_precision(double sqnr_plain_db, double sqnr_transform_db, double high_db,
                                   double low_db) {
  if (sqnr_plain_db >= high_db) return MXQ_PREC_W4A4;
  if (sqnr_transform_db >= high_db) return MXQ_PREC_W4A4_TRANSFORM;
  if ((sqnr_plain_db > sqnr_transform_db ? sqnr_plain_db : sqnr_transform_db) >= low_db) return MXQ_PREC_W4A8;
  return MXQ_PREC_BF16;
}

void mxq_attn_code_poly(float coeffs[4]) {
  if (!coeffs) return;
  coeffs[0] = 1.0f;
  coeffs[1] = mxq::kCodeA1;
  coeffs[2] = mxq::kCodeA2;
  coeffs[3] = mxq::kCodeA3;
}

int64_t mxq_attn_padded_keys(int64_t S_kv) {
  if (S_kv < 1 || S_kv > (int64_t(1) << 23)) return -1;
  return (S_kv + mxq::kAttnBN - 1) / mxq::kAttnBN * mxq::kAttnBN;
}

mxq_status mxq_quantize_vt(const void* v_bf16, int64_t S, int64_t HD, int64_t ldv, mxq_scale_rule rule,
                           void* codes_out, void* sf_out, mxq_stream_t stream) {
  if (!v_bf16 || !codes_out || !sf_out) return MXQ_ERR_INVALID_ARG;
  if (rule != MXQ_SCALE_OCP && rule != MXQ_SCALE_UOS) return MXQ_ERR_INVALID_ARG;
  const int64_t Sp = mxq_attn_padded_keys(S);
  if (Sp < 0 || HD < 128 || HD % 128 != 0 || HD > (int64_t(1) << 16)) return MXQ_ERR_SHAPE;
  if (ldv < HD || ldv % 8 != 0) return MXQ_ERR_ALIGN;
  if (!aligned(v_bf16, 16) || !aligned(codes_out, 16)) return MXQ_ERR_ALIGN;
  DeviceInfo dev;
  mxq_status st = current_device(&dev);
  if (st != MXQ_OK) return st;
  const dim3 grid(static_cast<unsigned>(HD / 128), static_cast<unsigned>(Sp / 128));
  const auto* vp = static_cast<const uint16_t*>(v_bf16);
  auto* cp = static_cast<uint8_t*>(codes_out);
  auto* sp = static_cast<uint8_t*>(sf_out);
  if (rule == MXQ_SCALE_UOS)
    mxq::quantize_vt_kernel<true><<<grid, 256, 0, stream>>>(vp, S, ldv, Sp, cp, sp);
  else
    mxq::quantize_vt_kernel<false><<<grid, 256, 0, stream>>>(vp, S, ldv, Sp, cp, sp);
  return launch_status();
}

mxq_status mxq_attention_mxfp4(const void* q_codes, const void* q_sf, const void* k_codes, const void* k_sf,
                               const void* vt_codes, const void* vt_sf, int64_t S_q, int64_t S_kv, int64_t H,
                               int64_t d, mxq_scale_rule rule, void* out_bf16, int64_t ldo, mxq_stream_t stream) {
  if (!q_codes || !q_sf || !k_codes || !k_sf || !vt_codes || !vt_sf || !out_bf16) return MXQ_ERR_INVALID_ARG;
  if (rule != MXQ_SCALE_OCP && rule != MXQ_SCALE_UOS) return MXQ_ERR_INVALID_ARG;
  if (d != mxq::kAttnD) return MXQ_ERR_UNSUPPORTED;
  const int64_t Sp = mxq_attn_padded_keys(S_kv);
  if (Sp < 0 || S_q < 1 || S_q > (int64_t(65535) * mxq::kAttnBM) || H < 1 || H > 65535 || H * d > (int64_t(1) << 16))
    return MXQ_ERR_SHAPE;
  const int64_t HD = H * d;
  if (ldo < HD || ldo % 8 != 0) return MXQ_ERR_ALIGN;
  if (!aligned(q_codes, 16) || !aligned(k_codes, 16) || !aligned(vt_codes, 16) || !aligned(q_sf, 16) ||
      !aligned(k_sf, 16) || !aligned(vt_sf, 16) || !aligned(out_bf16, 16))
    return MXQ_ERR_ALIGN;
  DeviceInfo dev;
  mxq_status st = current_device(&dev);
  if (st != MXQ_OK) return st;

  CUtensorMap tq, tsq, tk, tsk, tv, tsv;
  const bool ok =
      make_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_codes, HD / 2, S_q, HD / 2, 64, mxq::kAttnBM,
                   CU_TENSOR_MAP_SWIZZLE_64B) &&
      make_tmap_sf(&tsq, q_sf, S_q, HD, 1, 1) &&
      make_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_codes, HD / 2, S_kv, HD / 2, 64, mxq::kAttnBN,
                   CU_TENSOR_MAP_SWIZZLE_64B) &&
      make_tmap_sf(&tsk, k_sf, S_kv, HD, 1, 2) &&
      make_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, vt_codes, Sp / 2, HD, Sp / 2, 128, mxq::kAttnD,
                   CU_TENSOR_MAP_SWIZZLE_128B) &&
      make_tmap_sf(&tsv, vt_sf, HD, Sp, 2, 1);
  if (!ok) return MXQ_ERR_CUDA;

  mxq::AttnParams prm;
  prm.t_scale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  prm.Sq = static_cast<int>(S_q);
  prm.Skv = static_cast<int>(S_kv);
  prm.num_tiles = static_cast<int>(Sp / mxq::kAttnBN);

  auto kernel = rule == MXQ_SCALE_UOS ? mxq::mx_attention_kernel<true> : mxq::mx_attention_kernel<false>;
  static PerDevice setup;
  if (!setup.ensure(dev.index, [] {
        return cudaFuncSetAttribute(mxq::mx_attention_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    mxq::kAttnSmemBytes) == cudaSuccess &&
               cudaFuncSetAttribute(mxq::mx_attention_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    mxq::kAttnSmemBytes) == cudaSuccess;
      }))
    return MXQ_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>((S_q + mxq::kAttnBM - 1) / mxq::kAttnBM), static_cast<unsigned>(H));
  kernel<<<grid, mxq::kAttnThreads, mxq::kAttnSmemBytes, stream>>>(tq, tsq, tk, tsk, tv, tsv,
                                                                   static_cast<__nv_bfloat16*>(out_bf16), ldo, prm);
  return launch_status();
}

int64_t mxq_linear_workspace_bytes(int64_t M, int64_t K) {
  if (M < 1 || M > (int64_t(1) << 30) || K < 128 || K % 128 != 0 || K > (int64_t(1) << 22)) return -1;
  return linear_workspace(M, K).bytes;
}

mxq_status mxq_linear_w4a4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, mxq_scale_rule rule,
                           const void* w_codes, const void* w_sf, int64_t N, float alpha, const void* bias_bf16,
                           void* workspace, int64_t workspace_bytes, void* d_bf16, int64_t ldd, mxq_stream_t stream) {
  if (!x_bf16 || !workspace) return MXQ_ERR_INVALID_ARG;
  if (rule != MXQ_SCALE_OCP && rule != MXQ_SCALE_UOS) return MXQ_ERR_INVALID_ARG;
  if (!std::isfinite(alpha)) return MXQ_ERR_INVALID_ARG;
  const int64_t need = mxq_linear_workspace_bytes(M, K);
  if (need < 0 || M > int64_t(65535) * 128) return MXQ_ERR_SHAPE;
  if (workspace_bytes < need) return MXQ_ERR_INVALID_ARG;
  if (ldx < K || ldx % 8 != 0 || !aligned(x_bf16, 16) || !aligned(workspace, 16)) return MXQ_ERR_ALIGN;
  const LinearWorkspace ws = linear_workspace(M, K);
  auto* base = static_cast<uint8_t*>(workspace);
  void* a_codes = base + ws.codes;
  void* a_sf = base + ws.sf;
  mxq_status st = check_gemm_shapes(a_codes, w_codes, w_sf, d_bf16, M, N, K, ldd, bias_bf16);
  if (st != MXQ_OK) return st;
  DeviceInfo dev;
  st = current_device(&dev);
  if (st != MXQ_OK) return st;
  st = launch_mxfp4(false, x_bf16, M, K, ldx, rule, 0, a_codes, a_sf, stream);
  if (st != MXQ_OK) return st;
  return launch_gemm<false>(a_codes, a_sf, w_codes, w_sf, M, N, K, alpha, bias_bf16, d_bf16, ldd, stream);
}

mxq_status mxq_linear_w4a4_static(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, mxq_scale_rule rule,
                                  const void* w_codes, const void* w_sf, int64_t N, float alpha,
                                  const void* bias_bf16, void* d_bf16, int64_t ldd, mxq_stream_t stream) {
  const int64_t need = mxq_linear_workspace_bytes(M, K);
  if (need < 0 || need > kStaticScratchBytes) return MXQ_ERR_SHAPE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXQ_ERR_CUDA;
  void* scratch = static_scratch(dev);
  if (!scratch) return MXQ_ERR_CUDA;
  // Nothing in the scratch has to start at zero: the quantiser writes every byte the GEMM
  // reads (codes of all M rows, whole scale atoms including their padding).
  return mxq_linear_w4a4(x_bf16, M, K, ldx, rule, w_codes, w_sf, N, alpha, bias_bf16, scratch, kStaticScratchBytes,
                         d_bf16, ldd, stream);
}

mxq_status mxq_selftest_wait_timeout(mxq_stream_t stream) {
  DeviceInfo dev;
  const mxq_status st = current_device(&dev);
  if (st != MXQ_OK) return st;
  mxq::selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return launch_status();
}

mxq_status mxq_debug_poll(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return MXQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, mxq::g_status, sizeof v) != cudaSuccess) return MXQ_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(mxq::g_status, &zero, sizeof zero) != cudaSuccess) return MXQ_ERR_CUDA;
    return static_cast<mxq_status>(v);
  }
  return MXQ_OK;
}

}  // extern "C"
