// The C ABI of libany4: argument validation (before any CUDA call, so a bad
// call launches nothing) and dispatch to the kernels.
#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"

namespace any4 {

// Two-pass prefill for large M (prefill.cu): the weights dequantised into the
// workspace, then streamed to the tensor cores by TMA.
bool prefill_use_two_pass(int64_t M, int64_t N, int64_t K);
size_t prefill_two_pass_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G);
any4_status launch_prefill_two_pass(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                                    int64_t lut_row_stride, const uint16_t* scale,
                                    const uint16_t* offset, uint16_t* y, float* y32, int64_t M,
                                    int64_t N, int64_t K, int64_t G, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, bool test_stall,
                                    cudaStream_t stream, const DeviceInfo& dev);
// The same with codes of 2 or 3 bits (the n-bit dequant as the first pass).
any4_status launch_prefill_two_pass_bits(const uint16_t* x, const uint8_t* packed,
                                         const uint16_t* lut, int64_t lut_row_stride,
                                         const uint16_t* scale, const uint16_t* offset,
                                         uint16_t* y, float* y32, int64_t M, int64_t N, int64_t K,
                                         int64_t G, int bits, void* workspace,
                                         size_t workspace_bytes, int32_t* dev_status,
                                         bool test_stall, cudaStream_t stream,
                                         const DeviceInfo& dev);

// Table learning (quantize.cu): one thread block per weight row; bits = 2, 3, 4.
size_t quantize_smem_bytes(int64_t K, int64_t G);
any4_status launch_quantize(const uint16_t* w, const float* ex, int64_t N, int64_t K, int64_t G,
                            int bits, int32_t max_iter, uint8_t* packed, uint16_t* lut,
                            uint16_t* scale, uint16_t* offset, int32_t* iters,
                            cudaStream_t stream, const DeviceInfo& dev);
// n-bit storage below 4 bits (nbit.cu): bits = 2 or 3.
any4_status launch_pack_bits(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K,
                             int bits, int32_t* dev_status, cudaStream_t stream,
                             const DeviceInfo& dev);

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape rules shared by dequant and matmul (see any4.h).
bool shape_ok(int64_t N, int64_t K, int64_t G) {
  if (N < 1 || K < 32 || G < 32) return false;
  if (K % 32 != 0 || G % 32 != 0 || K % G != 0) return false;
  // keep every byte offset well inside int64 (N*K*2 bytes of bf16 W)
  if (N > (int64_t(1) << 40) / K) return false;
  return true;
}

bool stride_ok(int64_t lut_row_stride) { return lut_row_stride == 0 || lut_row_stride == 16; }

constexpr int64_t kDecodeMaxM = 16;
}  // namespace

any4_status current_device(DeviceInfo* info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ANY4_ERR_CUDA;
  any4_status st = ANY4_OK;
  std::call_once(g_dev_once[dev], [&] {
    DeviceInfo d;
    d.device = dev;
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      d.device = -1;
    }
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess)
      d.smem_optin = (size_t)optin;
    g_dev[dev] = d;
  });
  if (g_dev[dev].device < 0) return ANY4_ERR_CUDA;
  // The kernels are built for sm_100a only.
  if (g_dev[dev].cc_major != 10 || g_dev[dev].cc_minor != 0) st = ANY4_ERR_UNSUPPORTED;
  *info = g_dev[dev];
  return st;
}

int cached_occupancy(const void* kernel, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, size_t, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const auto key = std::make_tuple(kernel, threads, smem, dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) != cudaSuccess)
    return 0;
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = occ;
  return occ;
}

any4_status ensure_dynamic_smem(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> opted;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ANY4_ERR_CUDA;
  const auto key = std::make_pair(kernel, dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = opted.find(key);
  if (it != opted.end() && it->second >= bytes) return ANY4_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return ANY4_ERR_CUDA;
  }
  opted[key] = bytes;
  return ANY4_OK;
}

}  // namespace any4

using namespace any4;

extern "C" {

int32_t any4_version(void) { return 10000; }

const char* any4_status_string(int32_t s) {
  switch (s) {
    case ANY4_OK: return "ok";
    case ANY4_ERR_NULL: return "a required pointer is NULL";
    case ANY4_ERR_SHAPE: return "a size breaks the shape rules";
    case ANY4_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case ANY4_ERR_RANGE: return "a code above 15 was given to any4_pack";
    case ANY4_ERR_CUDA: return "a CUDA runtime call or launch failed";
    case ANY4_ERR_TIMEOUT: return "a bounded pipeline wait gave up on the device";
    case ANY4_ERR_UNSUPPORTED: return "no kernel for this request on this device";
    case ANY4_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "several device errors (bits OR-ed) or an unknown status";
  }
}

double any4_bits_per_weight(int64_t K, int64_t G) {
  if (K <= 0 || G <= 0) return 0.0;
  // 4-bit code + (16-bit scale + 16-bit offset) per G + 16 x 16-bit table per K
  return 4.0 + 32.0 / (double)G + 256.0 / (double)K;
}

any4_status any4_pack(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K,
                      int32_t* dev_status, any4_stream_t stream) {
  if (!idx || !packed) return ANY4_ERR_NULL;
  if (N < 1 || K < 32 || K % 32 != 0 || N > (int64_t(1) << 40) / K) return ANY4_ERR_SHAPE;
  if (!aligned16(idx) || !aligned16(packed)) return ANY4_ERR_ALIGN;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return ANY4_ERR_ALIGN;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  return launch_pack(idx, packed, N, K, dev_status, (cudaStream_t)stream, dev);
}

any4_status any4_repack(const uint8_t* packed, uint8_t* repacked, int64_t N, int64_t K,
                        any4_stream_t stream) {
  if (!packed || !repacked) return ANY4_ERR_NULL;
  if (N < 1 || K < 1024 || K % 1024 != 0 || N > (int64_t(1) << 40) / K) return ANY4_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(repacked)) return ANY4_ERR_ALIGN;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(packed), b0 = reinterpret_cast<uintptr_t>(repacked);
  const uintptr_t bytes = (uintptr_t)(N * (K / 2));
  if (a0 < b0 + bytes && b0 < a0 + bytes) return ANY4_ERR_SHAPE;  // the buffers overlap
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  return launch_repack(packed, repacked, N, K, (cudaStream_t)stream, dev);
}

any4_status any4_quantize(const uint16_t* w, const float* ex_abs, int64_t N, int64_t K,
                          int64_t G, int32_t max_iter, uint8_t* packed, uint16_t* lut,
                          uint16_t* scale, uint16_t* offset, int32_t* iters,
                          any4_stream_t stream) {
  return any4_quantize_bits(w, ex_abs, N, K, G, 4, max_iter, packed, lut, scale, offset, iters,
                            stream);
}

any4_status any4_quantize_bits(const uint16_t* w, const float* ex_abs, int64_t N, int64_t K,
                               int64_t G, int32_t bits, int32_t max_iter, uint8_t* packed,
                               uint16_t* lut, uint16_t* scale, uint16_t* offset, int32_t* iters,
                               any4_stream_t stream) {
  if (!w || !ex_abs || !packed || !lut || !scale || !offset) return ANY4_ERR_NULL;
  if (bits < 2 || bits > 4) return ANY4_ERR_SHAPE;
  if (!shape_ok(N, K, G) || K > ANY4_QUANTIZE_MAX_K || N > INT32_MAX || max_iter < 0 ||
      max_iter > ANY4_QUANTIZE_MAX_ITER)
    return ANY4_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(ex_abs) || !aligned16(packed) || !aligned16(lut) ||
      !aligned16(scale) || !aligned16(offset))
    return ANY4_ERR_ALIGN;
  if (iters && (reinterpret_cast<uintptr_t>(iters) & 3u)) return ANY4_ERR_ALIGN;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  return launch_quantize(w, ex_abs, N, K, G, bits, max_iter, packed, lut, scale, offset, iters,
                         (cudaStream_t)stream, dev);
}

any4_status any4_pack_bits(const uint8_t* idx, uint8_t* packed, int64_t N, int64_t K,
                           int32_t bits, int32_t* dev_status, any4_stream_t stream) {
  if (bits == 4) return any4_pack(idx, packed, N, K, dev_status, stream);
  if (!idx || !packed) return ANY4_ERR_NULL;
  if (bits < 2 || bits > 3 || N < 1 || K < 32 || K % 32 != 0 || N > (int64_t(1) << 40) / K)
    return ANY4_ERR_SHAPE;
  if (!aligned16(idx) || !aligned16(packed)) return ANY4_ERR_ALIGN;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return ANY4_ERR_ALIGN;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  return launch_pack_bits(idx, packed, N, K, bits, dev_status, (cudaStream_t)stream, dev);
}

any4_status any4_dequant_bits(const uint8_t* packed, const uint16_t* lut, int64_t lut_row_stride,
                              const uint16_t* scale, const uint16_t* offset, uint16_t* W,
                              int64_t N, int64_t K, int64_t G, int32_t bits,
                              any4_stream_t stream) {
  if (bits == 4)
    return any4_dequant(packed, lut, lut_row_stride, scale, offset, W, N, K, G, stream);
  if (!packed || !lut || !scale || !offset || !W) return ANY4_ERR_NULL;
  if (bits < 2 || bits > 3 || !shape_ok(N, K, G) ||
      (lut_row_stride != 0 && lut_row_stride != (int64_t(1) << bits)))
    return ANY4_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(lut) || !aligned16(scale) || !aligned16(offset) ||
      !aligned16(W))
    return ANY4_ERR_ALIGN;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  return launch_dequant_bits(packed, lut, lut_row_stride, scale, offset, W, N, K, G, bits,
                             (cudaStream_t)stream, dev);
}

any4_status any4_dequant(const uint8_t* packed, const uint16_t* lut, int64_t lut_row_stride,
                         const uint16_t* scale, const uint16_t* offset, uint16_t* W,
                         int64_t N, int64_t K, int64_t G, any4_stream_t stream) {
  if (!packed || !lut || !scale || !offset || !W) return ANY4_ERR_NULL;
  if (!shape_ok(N, K, G) || !stride_ok(lut_row_stride)) return ANY4_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(lut) || !aligned16(scale) || !aligned16(offset) ||
      !aligned16(W))
    return ANY4_ERR_ALIGN;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  return launch_dequant(packed, lut, lut_row_stride, scale, offset, W, N, K, G,
                        (cudaStream_t)stream, dev);
}

any4_status any4_matmul_grouped(const uint16_t* x, const any4_weight* w, int32_t count,
                                int64_t M, int64_t K, int64_t G, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, any4_path path,
                                uint32_t flags, any4_stream_t stream) {
  if (!x || !w) return ANY4_ERR_NULL;
  if (count < 1 || count > ANY4_GROUP_MAX) return ANY4_ERR_SHAPE;
  for (int i = 0; i < count; ++i) {
    if (!w[i].packed || !w[i].lut || !w[i].scale || !w[i].offset || !w[i].y)
      return ANY4_ERR_NULL;
    if (M < 1 || !shape_ok(w[i].N, K, G) || !stride_ok(w[i].lut_row_stride))
      return ANY4_ERR_SHAPE;
    if (!aligned16(w[i].packed) || !aligned16(w[i].lut) || !aligned16(w[i].scale) ||
        !aligned16(w[i].offset) || !aligned16(w[i].y))
      return ANY4_ERR_ALIGN;
  }
  if (!aligned16(x)) return ANY4_ERR_ALIGN;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return ANY4_ERR_ALIGN;
  if (flags & ~(uint32_t)(ANY4_FLAG_OVERLAP_PRIOR | ANY4_FLAG_FP32_OUT | ANY4_FLAG_TEST_STALL |
                         ANY4_FLAG_PAIR_TABLE | ANY4_FLAG_DECODE_LAYOUT))
    return ANY4_ERR_UNSUPPORTED;
  const any4_path chosen = path == ANY4_PATH_AUTO ? any4_matmul_choose_path(M, 1, K, G) : path;
  const bool decode_layout = (flags & ANY4_FLAG_DECODE_LAYOUT) != 0;
  if (decode_layout) {
    if (chosen != ANY4_PATH_DECODE || (flags & ANY4_FLAG_PAIR_TABLE)) return ANY4_ERR_UNSUPPORTED;
    for (int i = 0; i < count; ++i)
      if (!decode_layout_supported(M, w[i].N, K, G)) return ANY4_ERR_UNSUPPORTED;
  }
  bool one_launch = chosen == ANY4_PATH_DECODE && !(flags & ANY4_FLAG_PAIR_TABLE);
  for (int i = 0; i < count && one_launch; ++i)
    one_launch = decode_tma_supported(M, w[i].N, K, G);
  if (one_launch) {
    DeviceInfo dev;
    any4_status st = current_device(&dev);
    if (st != ANY4_OK) return st;
    const bool fp32 = (flags & ANY4_FLAG_FP32_OUT) != 0;
    DecodeWeights dw[ANY4_GROUP_MAX];
    for (int i = 0; i < count; ++i)
      dw[i] = {w[i].packed, w[i].lut, w[i].lut_row_stride, w[i].scale, w[i].offset,
               fp32 ? nullptr : w[i].y, fp32 ? reinterpret_cast<float*>(w[i].y) : nullptr,
               w[i].N};
    return launch_decode_tma_group(x, dw, count, K, G, 4, (flags & ANY4_FLAG_OVERLAP_PRIOR) != 0,
                                   dev_status, (flags & ANY4_FLAG_TEST_STALL) != 0,
                                   (cudaStream_t)stream, dev, decode_layout);
  }
  for (int i = 0; i < count; ++i) {
    const any4_status st =
        any4_matmul_ex(x, w[i].packed, w[i].lut, w[i].lut_row_stride, w[i].scale, w[i].offset,
                       w[i].y, M, w[i].N, K, G, workspace, workspace_bytes, dev_status, path,
                       flags, stream);
    if (st != ANY4_OK) return st;
  }
  return ANY4_OK;
}

size_t any4_matmul_bits_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G,
                                       int32_t bits) {
  if (bits == 4) return any4_matmul_workspace_size(M, N, K, G);
  if (bits < 2 || bits > 3 || M < 1 || !shape_ok(N, K, G)) return 0;
  if (decode_tma_supported(M, N, K, G, bits)) return 0;
  return prefill_two_pass_workspace_size(M, N, K, G);
}

any4_status any4_matmul_bits(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                             int64_t lut_row_stride, const uint16_t* scale,
                             const uint16_t* offset, uint16_t* y, int64_t M, int64_t N, int64_t K,
                             int64_t G, int32_t bits, void* workspace, size_t workspace_bytes,
                             int32_t* dev_status, uint32_t flags, any4_stream_t stream) {
  if (bits == 4)
    return any4_matmul_ex(x, packed, lut, lut_row_stride, scale, offset, y, M, N, K, G,
                          workspace, workspace_bytes, dev_status, ANY4_PATH_AUTO, flags, stream);
  if (!x || !packed || !lut || !scale || !offset || !y) return ANY4_ERR_NULL;
  if (bits < 2 || bits > 3 || M < 1 || !shape_ok(N, K, G) ||
      (lut_row_stride != 0 && lut_row_stride != (int64_t(1) << bits)))
    return ANY4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(lut) || !aligned16(scale) ||
      !aligned16(offset) || !aligned16(y))
    return ANY4_ERR_ALIGN;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return ANY4_ERR_ALIGN;
  if (workspace && !aligned16(workspace)) return ANY4_ERR_ALIGN;
  if (flags & ~(uint32_t)(ANY4_FLAG_OVERLAP_PRIOR | ANY4_FLAG_FP32_OUT | ANY4_FLAG_TEST_STALL))
    return ANY4_ERR_UNSUPPORTED;
  const size_t need = any4_matmul_bits_workspace_size(M, N, K, G, bits);
  if (need > 0 && (!workspace || workspace_bytes < need)) return ANY4_ERR_WORKSPACE;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  const bool fp32 = (flags & ANY4_FLAG_FP32_OUT) != 0;
  float* y32 = fp32 ? reinterpret_cast<float*>(y) : nullptr;
  const bool test_stall = (flags & ANY4_FLAG_TEST_STALL) != 0;
  if (need == 0) {
    const DecodeWeights w = {packed, lut, lut_row_stride, scale, offset, fp32 ? nullptr : y, y32,
                             N};
    return launch_decode_tma_group(x, &w, 1, K, G, bits, (flags & ANY4_FLAG_OVERLAP_PRIOR) != 0,
                                   dev_status, test_stall, (cudaStream_t)stream, dev);
  }
  return launch_prefill_two_pass_bits(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N,
                                      K, G, bits, workspace, workspace_bytes, dev_status,
                                      test_stall, (cudaStream_t)stream, dev);
}

any4_status any4_group_sums(const uint16_t* x, float* xsum, int64_t M, int64_t K, int64_t G,
                             any4_stream_t stream) {
  if (!x || !xsum) return ANY4_ERR_NULL;
  if (M < 1 || !shape_ok(M, K, G)) return ANY4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(xsum)) return ANY4_ERR_ALIGN;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  return launch_group_sums(x, xsum, M, K, G, (cudaStream_t)stream, dev);
}

any4_status any4_read_probe(const void* buf, int64_t bytes, uint32_t* out,
                            any4_stream_t stream) {
  if (!out || (!buf && bytes > 0)) return ANY4_ERR_NULL;
  if (bytes < 0 || bytes % 16 != 0) return ANY4_ERR_SHAPE;
  if ((buf && !aligned16(buf)) || reinterpret_cast<uintptr_t>(out) % 4 != 0) return ANY4_ERR_ALIGN;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  return launch_read_probe(buf, bytes, out, (cudaStream_t)stream, dev);
}

any4_path any4_matmul_choose_path(int64_t M, int64_t N, int64_t K, int64_t G) {
  (void)N; (void)K; (void)G;
  return M <= kDecodeMaxM ? ANY4_PATH_DECODE : ANY4_PATH_PREFILL;
}

size_t any4_matmul_workspace_size_ex(int64_t M, int64_t N, int64_t K, int64_t G,
                                     any4_path path) {
  if (M < 1 || !shape_ok(N, K, G)) return 0;
  if (path == ANY4_PATH_AUTO) path = any4_matmul_choose_path(M, N, K, G);
  if (path == ANY4_PATH_PREFILL)
    return prefill_use_two_pass(M, N, K) ? prefill_two_pass_workspace_size(M, N, K, G)
                                         : prefill_workspace_size(M, N, K, G);
  // decode: the pair-table kernel's stream-K exchange (M <= 2); sized for the
  // current device, or for a 160-SM grid where there is none
  DeviceInfo dev;
  if (current_device(&dev) != ANY4_OK) {
    dev = DeviceInfo();
    dev.sm_count = 160;
  }
  return decode_pair_workspace_size(M, N, K, G, dev);
}

size_t any4_matmul_workspace_size(int64_t M, int64_t N, int64_t K, int64_t G) {
  return any4_matmul_workspace_size_ex(M, N, K, G, ANY4_PATH_AUTO);
}

any4_status any4_matmul_ex(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                           int64_t lut_row_stride, const uint16_t* scale,
                           const uint16_t* offset, uint16_t* y, int64_t M, int64_t N,
                           int64_t K, int64_t G, void* workspace, size_t workspace_bytes,
                           int32_t* dev_status, any4_path path, uint32_t flags,
                           any4_stream_t stream) {
  if (!x || !packed || !lut || !scale || !offset || !y) return ANY4_ERR_NULL;
  if (M < 1 || !shape_ok(N, K, G) || !stride_ok(lut_row_stride)) return ANY4_ERR_SHAPE;
  if (M > (int64_t(1) << 40) / K || M > (int64_t(1) << 40) / N) return ANY4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(lut) || !aligned16(scale) ||
      !aligned16(offset) || !aligned16(y))
    return ANY4_ERR_ALIGN;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return ANY4_ERR_ALIGN;
  if (workspace && !aligned16(workspace)) return ANY4_ERR_ALIGN;
  if (path == ANY4_PATH_AUTO) path = any4_matmul_choose_path(M, N, K, G);
  if (path != ANY4_PATH_DECODE && path != ANY4_PATH_PREFILL) return ANY4_ERR_UNSUPPORTED;
  if (flags & ~(uint32_t)(ANY4_FLAG_OVERLAP_PRIOR | ANY4_FLAG_FP32_OUT | ANY4_FLAG_TEST_STALL |
                         ANY4_FLAG_PAIR_TABLE | ANY4_FLAG_DECODE_LAYOUT))
    return ANY4_ERR_UNSUPPORTED;
  const bool decode_layout = (flags & ANY4_FLAG_DECODE_LAYOUT) != 0;
  if (decode_layout && (path != ANY4_PATH_DECODE || (flags & ANY4_FLAG_PAIR_TABLE) ||
                        !decode_layout_supported(M, N, K, G)))
    return ANY4_ERR_UNSUPPORTED;
  float* y32 = (flags & ANY4_FLAG_FP32_OUT) ? reinterpret_cast<float*>(y) : nullptr;
  const bool test_stall = (flags & ANY4_FLAG_TEST_STALL) != 0;
  if (path == ANY4_PATH_DECODE && M > kDecodeMaxM) return ANY4_ERR_UNSUPPORTED;
  // the prefill path runs in one pass with at least prefill_workspace_size
  // bytes, and in two passes (large M) when the workspace also holds the
  // dequantised weights
  const size_t need = path == ANY4_PATH_PREFILL ? prefill_workspace_size(M, N, K, G) : 0;
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return ANY4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ANY4_ERR_ALIGN;
  }
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  if (decode_layout)  // only the folded-table M = 1 kernel reads this layout
    return launch_decode_tma(x, packed, lut, lut_row_stride, scale, offset, y, y32, N, K, G,
                             (flags & ANY4_FLAG_OVERLAP_PRIOR) != 0, dev_status, test_stall,
                             (cudaStream_t)stream, dev, true);
  if (path == ANY4_PATH_DECODE) {
    return launch_decode(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N, K, G,
                         workspace, workspace_bytes, (flags & ANY4_FLAG_OVERLAP_PRIOR) != 0,
                         (flags & ANY4_FLAG_PAIR_TABLE) != 0, dev_status, test_stall,
                         (cudaStream_t)stream, dev);
  }
  if (prefill_use_two_pass(M, N, K) &&
      workspace_bytes >= prefill_two_pass_workspace_size(M, N, K, G))
    return launch_prefill_two_pass(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N, K,
                                   G, workspace, workspace_bytes, dev_status, test_stall,
                                   (cudaStream_t)stream, dev);
  return launch_prefill(x, packed, lut, lut_row_stride, scale, offset, y, y32, M, N, K, G,
                        workspace, workspace_bytes, dev_status, test_stall, (cudaStream_t)stream,
                        dev);
}

// The prefill kernel with the library's fixed scratch array (static_scratch.cu)
// in place of a workspace; same validation as any4_matmul_ex.
any4_status any4_matmul_static_scratch(const uint16_t* x, const uint8_t* packed,
                                       const uint16_t* lut, int64_t lut_row_stride,
                                       const uint16_t* scale, const uint16_t* offset,
                                       uint16_t* y, int64_t M, int64_t N, int64_t K, int64_t G,
                                       int32_t* dev_status, any4_stream_t stream) {
  if (!x || !packed || !lut || !scale || !offset || !y) return ANY4_ERR_NULL;
  if (M < 1 || !shape_ok(N, K, G) || !stride_ok(lut_row_stride)) return ANY4_ERR_SHAPE;
  if (M > (int64_t(1) << 40) / K || M > (int64_t(1) << 40) / N) return ANY4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(lut) || !aligned16(scale) ||
      !aligned16(offset) || !aligned16(y))
    return ANY4_ERR_ALIGN;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return ANY4_ERR_ALIGN;
  DeviceInfo dev;
  any4_status st = current_device(&dev);
  if (st != ANY4_OK) return st;
  if (prefill_workspace_size(M, N, K, G) > ANY4_STATIC_SCRATCH_BYTES) return ANY4_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = static_scratch(dev.device, &scratch);
  if (st != ANY4_OK) return st;
  return launch_prefill(x, packed, lut, lut_row_stride, scale, offset, y, nullptr, M, N, K, G,
                        scratch, ANY4_STATIC_SCRATCH_BYTES, dev_status, false,
                        (cudaStream_t)stream, dev);
}

any4_status any4_matmul(const uint16_t* x, const uint8_t* packed, const uint16_t* lut,
                        int64_t lut_row_stride, const uint16_t* scale,
                        const uint16_t* offset, uint16_t* y, int64_t M, int64_t N,
                        int64_t K, int64_t G, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, any4_stream_t stream) {
  return any4_matmul_ex(x, packed, lut, lut_row_stride, scale, offset, y, M, N, K, G, workspace,
                        workspace_bytes, dev_status, ANY4_PATH_AUTO, ANY4_FLAG_NONE, stream);
}

}  // extern "C"
