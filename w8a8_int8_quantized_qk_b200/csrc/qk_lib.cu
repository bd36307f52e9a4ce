// qk_lib.cu -- the C ABI of libqk.so (declared in include/qk.h): argument
// checks on the host, then one kernel launch per stage on the caller's
// stream.  All kernels of the library are compiled in this one translation
// unit, so the device status word is a single symbol.
//
// Interface source: "16. Deploying Custom Kernels", C++ Kernel Interface
// (GemmConfig's m, n, k, int8 a / b, int32 c, scale_a, scale_b,
// output_scale, stream; a status-returning entry point) and Python Bindings
// (the same fields passed as plain integers, pointers and a float).
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "gemm_sm100.cuh"
#include "gemv.cuh"
#include "mma_probe.cuh"
#include "qk_common.cuh"
#include "quant.cuh"

namespace qk {
namespace {

struct DeviceInfo {
  bool valid = false;
  int sms = 0;
  int major = 0;
  int minor = 0;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_devices_mu;

// Properties of the current device (cached); nullptr on a CUDA error.
const DeviceInfo* current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_devices_mu);
  DeviceInfo& d = g_devices[dev];
  if (!d.valid) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return nullptr;
    d.valid = true;
  }
  return &d;
}

// The kernels are built for sm_100a only, which runs on compute capability
// 10.0 devices.
qk_status check_device(const DeviceInfo** out) {
  const DeviceInfo* d = current_device();
  if (d == nullptr) return QK_ERR_CUDA;
  if (d->major != 10 || d->minor != 0) return QK_ERR_UNSUPPORTED;
  *out = d;
  return QK_OK;
}

// With QK_DEBUG set in the environment, a failing CUDA call is reported on
// stderr (the call still just returns QK_ERR_CUDA).
qk_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return QK_OK;
  static const bool debug = std::getenv("QK_DEBUG") != nullptr;
  if (debug) std::fprintf(stderr, "libqk: %s: %s\n", where, cudaGetErrorString(e));
  return QK_ERR_CUDA;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// K * 127^2 < 2^31  <=>  K <= 133144
constexpr int kMaxK = 133144;
// asymmetric activations: |q - zp| <= 255, so k * 255 * 127 < 2^31
constexpr int kMaxKAsym = 66311;

qk_status quant_common(int m, int k, const void* x, const void* up, int64_t ld, qk_dtype dt,
                       int8_t* q, float* scale, qk_stream stream, bool silu, bool fp8 = false,
                       const float* ub = nullptr) {
  if (m < 0 || k <= 0 || (k % 16) != 0) return QK_ERR_INVALID_ARG;
  if (dt != QK_F32 && dt != QK_BF16) return QK_ERR_INVALID_ARG;
  if (ld < k) return QK_ERR_INVALID_ARG;
  if (m == 0) return QK_OK;
  if (x == nullptr || q == nullptr || scale == nullptr || (silu && up == nullptr))
    return QK_ERR_INVALID_ARG;
  const int64_t esize = dt == QK_BF16 ? 2 : 4;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale, 4) || (silu && !aligned(up, 16)) ||
      !aligned(ub, 4) || (ld * esize) % 16 != 0)
    return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  quant::Args a;
  a.m = m;
  a.k = k;
  a.x = x;
  a.up = up;
  a.ld = ld;
  a.q = q;
  a.scale = scale;
  a.fp8 = fp8 ? 1 : 0;
  a.ub = fp8 ? ub : nullptr;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = silu ? quant::launch<true>(a, dt == QK_BF16, dev->sms, s)
                             : quant::launch<false>(a, dt == QK_BF16, dev->sms, s);
  return cuda_status(e, "quantize launch");
}

// Which kernel runs a GEMM of this shape.
enum class GemmPath { kGemv, kTensorChannel, kTensorPair, kTensorGroup };

GemmPath gemm_path(int m, int n, int k, int group_k) {
  if (group_k != 0) return GemmPath::kTensorGroup;
  if (m <= gemv::max_tokens()) return GemmPath::kGemv;
  if (m <= 128) return GemmPath::kTensorChannel;
  if (m <= 256) {
    const DeviceInfo* dev = nullptr;
    int dev_id = 0;
    if (check_device(&dev) == QK_OK && cudaGetDevice(&dev_id) == cudaSuccess &&
        gemm::prefer_channel_split(m, n, k, dev->sms, dev_id))
      return GemmPath::kTensorChannel;
  }
  return GemmPath::kTensorPair;
}

qk_status gemm_check(int m, int n, int k, int group_k) {
  if (m < 0 || n < 0 || k <= 0) return QK_ERR_INVALID_ARG;
  if ((k % 16) != 0 || (n % 8) != 0) return QK_ERR_INVALID_ARG;
  if (group_k != 0 && group_k != 128) return QK_ERR_INVALID_ARG;
  if (group_k == 128 && (k % 128) != 0) return QK_ERR_INVALID_ARG;
  if (k > kMaxK) return QK_ERR_OVERFLOW_BOUND;
  return QK_OK;
}

// Device-side bounded-wait check: one thread waits on a barrier that no one
// arrives at.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
    mbar_wait(smem_addr(&bar), 0u, nullptr, limit_ns);
  }
}

// Every finite binary32 g in [first, first + count): the fused SiLU product
// as the quantisers compute it (quant::silu_mul2, partly on packed pairs)
// against the scalar chain (quant::silu_mul), u = 1.  Counts the g whose results differ in any bit and keeps the
// smallest such bit pattern.
__global__ void __launch_bounds__(256) selftest_silu_kernel(uint32_t first, uint64_t count,
                                                            unsigned long long* mismatches,
                                                            uint32_t* first_mismatch) {
  const uint64_t pairs = (count + 1) / 2;
  unsigned long long local = 0;
  uint32_t low = 0xFFFFFFFFu;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < pairs;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const uint64_t o0 = 2 * i, o1 = 2 * i + 1;
    const uint32_t b0 = first + static_cast<uint32_t>(o0);
    const uint32_t b1 = first + static_cast<uint32_t>(o1 < count ? o1 : o0);
    const float g0 = __uint_as_float(b0), g1 = __uint_as_float(b1);
    float h0, h1;
    quant::silu_mul2(g0, g1, 1.0f, 1.0f, h0, h1);
    const float r0 = quant::silu_mul(g0, 1.0f), r1 = quant::silu_mul(g1, 1.0f);
    if (isfinite(g0) && __float_as_uint(h0) != __float_as_uint(r0)) {
      ++local;
      low = b0 < low ? b0 : low;
    }
    if (o1 < count && isfinite(g1) && __float_as_uint(h1) != __float_as_uint(r1)) {
      ++local;
      low = b1 < low ? b1 : low;
    }
  }
  if (local) {
    atomicAdd(mismatches, local);
    if (first_mismatch) atomicMin(first_mismatch, low);
  }
}

// Scratch for qk_w8a8_gemm_noalloc: a split-K workspace that lives in the
// library's own device memory (zero at module load).  Host code only ever sees
// a stand-in for this symbol; its device address comes from
// cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QK_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, or nullptr.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace qk

using namespace qk;

extern "C" {

int qk_abi_version(void) { return QK_ABI_VERSION; }

const char* qk_status_string(int status) {
  switch (status) {
    case QK_OK: return "ok";
    case QK_ERR_INVALID_ARG: return "invalid argument";
    case QK_ERR_MISALIGNED: return "misaligned pointer or row stride";
    case QK_ERR_UNSUPPORTED: return "unsupported (needs a compute capability 10.0 device)";
    case QK_ERR_OVERFLOW_BOUND: return "k too large: k * 127^2 must stay below 2^31";
    case QK_ERR_CUDA: return "CUDA error";
    case QK_ERR_TIMEOUT: return "a kernel's bounded wait expired";
    case QK_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

qk_status qk_quantize_per_token(int m, int k, const void* x, qk_dtype x_dtype, int8_t* q,
                                float* scale, qk_stream stream) {
  return quant_common(m, k, x, nullptr, k, x_dtype, q, scale, stream, false);
}

qk_status qk_silu_mul_quant_per_token(int m, int k, const void* gate, const void* up,
                                      int64_t ld_in, qk_dtype in_dtype, int8_t* q, float* scale,
                                      qk_stream stream) {
  return quant_common(m, k, gate, up, ld_in, in_dtype, q, scale, stream, true);
}

qk_status qk_quantize_per_token_fp8(int m, int k, const void* x, qk_dtype x_dtype,
                                    const float* scale_ub, uint8_t* q, float* scale,
                                    qk_stream stream) {
  return quant_common(m, k, x, nullptr, k, x_dtype, reinterpret_cast<int8_t*>(q), scale, stream,
                      false, true, scale_ub);
}

qk_status qk_silu_mul_quant_per_token_fp8(int m, int k, const void* gate, const void* up,
                                          int64_t ld_in, qk_dtype in_dtype, const float* scale_ub,
                                          uint8_t* q, float* scale, qk_stream stream) {
  return quant_common(m, k, gate, up, ld_in, in_dtype, reinterpret_cast<int8_t*>(q), scale,
                      stream, true, true, scale_ub);
}

namespace {
// The pair kernel's plan for this problem on the current device; false when
// the problem takes no workspace (another kernel, or bad arguments).
bool pair_plan_for(int m, int n, int k, int group_k, gemm::PairPlan* pl) {
  if (gemm_check(m, n, k, group_k) != QK_OK || m == 0 || n == 0) return false;
  if (gemm_path(m, n, k, group_k) != GemmPath::kTensorPair) return false;
  const DeviceInfo* dev = nullptr;
  if (check_device(&dev) != QK_OK) return false;
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  *pl = gemm::pair_plan(m, n, k, gemm::max_pairs(dev_id, dev->sms), dev_id);
  return true;
}
}  // namespace

namespace {
// The output-only group kernel's plan for this problem on the current device
// (false: not group mode, or bad arguments).
bool group_plan_for(int m, int n, int k, int group_k, gemm::GroupPlan* g) {
  if (group_k == 0 || gemm_check(m, n, k, group_k) != QK_OK || m == 0 || n == 0) return false;
  const DeviceInfo* dev = nullptr;
  if (check_device(&dev) != QK_OK) return false;
  int dev_id = 0;
  if (cudaGetDevice(&dev_id) != cudaSuccess) return false;
  *g = gemm::group_plan(m, n, k, dev_id, dev->sms);
  return true;
}
}  // namespace

size_t qk_w8a8_gemm_workspace_size(int m, int n, int k, int group_k) {
  if (group_k != 0) {
    gemm::GroupPlan g;
    return group_plan_for(m, n, k, group_k, &g) ? gemm::group_plan_workspace_bytes(g) : 0;
  }
  gemm::PairPlan pl;
  return pair_plan_for(m, n, k, group_k, &pl) ? gemm::pair_workspace_bytes(pl) : 0;
}

namespace {
// The GEMM of qk_w8a8_gemm, and of qk_w8a8_gemm_asym when zp / wsum are
// given (per channel only; the caller has checked them).
qk_status gemm_common(int m, int n, int k, const int8_t* a, const int8_t* b,
                      const float* scale_a, const float* scale_b, int group_k,
                      float output_scale, int32_t* c, void* out, qk_dtype out_dtype,
                      void* workspace, size_t workspace_bytes, qk_stream stream,
                      const int32_t* zp, const int32_t* wsum);
}  // namespace

qk_status qk_w8a8_gemm(int m, int n, int k, const int8_t* a, const int8_t* b,
                       const float* scale_a, const float* scale_b, int group_k,
                       float output_scale, int32_t* c, void* out, qk_dtype out_dtype,
                       void* workspace, size_t workspace_bytes, qk_stream stream) {
  return gemm_common(m, n, k, a, b, scale_a, scale_b, group_k, output_scale, c, out, out_dtype,
                     workspace, workspace_bytes, stream, nullptr, nullptr);
}

qk_status qk_w8a8_gemm_asym(int m, int n, int k, const int8_t* a, const int32_t* zero_point_a,
                            const int8_t* b, const int32_t* wsum_b, const float* scale_a,
                            const float* scale_b, float output_scale, int32_t* c, void* out,
                            qk_dtype out_dtype, void* workspace, size_t workspace_bytes,
                            qk_stream stream) {
  if (k > kMaxKAsym) return QK_ERR_OVERFLOW_BOUND;
  if (m > 0 && n > 0 && (zero_point_a == nullptr || wsum_b == nullptr)) return QK_ERR_INVALID_ARG;
  if (!aligned(zero_point_a, 4) || !aligned(wsum_b, 16)) return QK_ERR_MISALIGNED;
  return gemm_common(m, n, k, a, b, scale_a, scale_b, 0, output_scale, c, out, out_dtype,
                     workspace, workspace_bytes, stream, zero_point_a, wsum_b);
}

qk_status qk_quantize_per_token_asym(int m, int k, const void* x, qk_dtype x_dtype, int8_t* q,
                                     float* scale, int32_t* zero_point, qk_stream stream) {
  if (m < 0 || k <= 0 || (k % 16) != 0) return QK_ERR_INVALID_ARG;
  if (x_dtype != QK_F32 && x_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (m == 0) return QK_OK;
  if (x == nullptr || q == nullptr || scale == nullptr || zero_point == nullptr)
    return QK_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale, 4) || !aligned(zero_point, 4))
    return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  quant::AsymArgs a;
  a.m = m;
  a.k = k;
  a.x = x;
  a.q = q;
  a.scale = scale;
  a.zp = zero_point;
  return cuda_status(quant::launch_asym(a, x_dtype == QK_BF16, reinterpret_cast<cudaStream_t>(stream)),
                     "asymmetric quantize launch");
}

// tokens per expert, on average, from which the MoE GEMM runs on CTA pairs
constexpr int kMoePairTokens = 128;

qk_status qk_w8a8_moe_gemm(int num_experts, int total_m, int n, int k, int max_m_per_expert,
                           const int32_t* expert_offsets, const int8_t* a, const int8_t* b,
                           const float* scale_a, const float* scale_b, float output_scale,
                           void* out, qk_dtype out_dtype, qk_stream stream) {
  if (num_experts < 1 || total_m < 0 || n < 0 || k <= 0 || max_m_per_expert < 0)
    return QK_ERR_INVALID_ARG;
  if ((k % 16) != 0 || (n % 8) != 0) return QK_ERR_INVALID_ARG;
  if (k > kMaxK) return QK_ERR_OVERFLOW_BOUND;
  if (out_dtype != QK_F32 && out_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (total_m == 0 || n == 0 || max_m_per_expert == 0) return QK_OK;
  if (static_cast<int64_t>(num_experts) * n > INT32_MAX) return QK_ERR_INVALID_ARG;
  if (expert_offsets == nullptr || a == nullptr || b == nullptr || scale_a == nullptr ||
      scale_b == nullptr || out == nullptr)
    return QK_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16) || !aligned(scale_a, 4) ||
      !aligned(scale_b, 16) || !aligned(expert_offsets, 4))
    return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  gemm::Args g = {};
  g.m = total_m;
  g.n = n;
  g.k = k;
  g.sa = scale_a;
  g.sw = scale_b;
  g.alpha = output_scale;
  g.out = out;
  g.out_bf16 = out_dtype == QK_BF16;
  cudaError_t e = cudaSuccess;
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  // Experts averaging at least 128 tokens: 256-row tiles on CTA pairs (half
  // the operand traffic per multiply-add of the 1-SM tile); fewer: 128-row
  // tiles on single SMs, which pad small experts less.
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool pair = static_cast<int64_t>(total_m) >= static_cast<int64_t>(kMoePairTokens) * num_experts &&
                    gemm::max_pairs(dev_id, dev->sms) > 0;
  const int r = pair ? gemm::launch_moe_pair(g, a, b, num_experts, (max_m_per_expert + 255) / 256,
                                             expert_offsets, dev_id, dev->sms, s, &e)
                     : gemm::launch_moe(g, a, b, num_experts, (max_m_per_expert + 127) / 128,
                                        expert_offsets, dev_id, dev->sms, s, &e);
  if (r == 1) return cuda_status(cudaErrorInvalidValue, "tensor map encoding");
  return r == 0 ? QK_OK : cuda_status(e, "moe gemm launch");
}

qk_status qk_quantize_static(int m, int k, const void* x, qk_dtype x_dtype, const float* scale,
                             int8_t* q, qk_stream stream) {
  if (m < 0 || k <= 0 || (k % 16) != 0) return QK_ERR_INVALID_ARG;
  if (x_dtype != QK_F32 && x_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (m == 0) return QK_OK;
  if (x == nullptr || scale == nullptr || q == nullptr) return QK_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale, 4)) return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  return cuda_status(quant::launch_static(static_cast<int64_t>(m) * k, x, x_dtype == QK_BF16, scale, q,
                                          dev->sms, reinterpret_cast<cudaStream_t>(stream)),
                     "static quantize launch");
}

qk_status qk_weight_row_sums(int n, int k, const int8_t* w, int32_t* wsum, qk_stream stream) {
  if (n < 0 || k <= 0 || (k % 16) != 0) return QK_ERR_INVALID_ARG;
  if (k > kMaxK) return QK_ERR_OVERFLOW_BOUND;
  if (n == 0) return QK_OK;
  if (w == nullptr || wsum == nullptr) return QK_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(wsum, 4)) return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  return cuda_status(quant::launch_weight_row_sums(n, k, w, wsum, reinterpret_cast<cudaStream_t>(stream)),
                     "weight row sums launch");
}

namespace {
qk_status gemm_common(int m, int n, int k, const int8_t* a, const int8_t* b,
                      const float* scale_a, const float* scale_b, int group_k,
                      float output_scale, int32_t* c, void* out, qk_dtype out_dtype,
                      void* workspace, size_t workspace_bytes, qk_stream stream,
                      const int32_t* zp, const int32_t* wsum) {
  qk_status st = gemm_check(m, n, k, group_k);
  if (st != QK_OK) return st;
  if (out != nullptr && out_dtype != QK_F32 && out_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return QK_OK;
  if (a == nullptr || b == nullptr || (c == nullptr && out == nullptr)) return QK_ERR_INVALID_ARG;
  if (out != nullptr && (scale_a == nullptr || scale_b == nullptr)) return QK_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(c, 16) || !aligned(out, 16) ||
      !aligned(scale_a, 16) || !aligned(scale_b, 16))
    return QK_ERR_MISALIGNED;
  const size_t need = qk_w8a8_gemm_workspace_size(m, n, k, group_k);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)))
    return QK_ERR_WORKSPACE;
  const DeviceInfo* dev = nullptr;
  st = check_device(&dev);
  if (st != QK_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const GemmPath path = gemm_path(m, n, k, group_k);
  if (path == GemmPath::kGemv) {
    gemv::Args g = {};
    g.m = m;
    g.n = n;
    g.k = k;
    g.a = a;
    g.w = b;
    g.sa = scale_a;
    g.sw = scale_b;
    g.alpha = output_scale;
    g.c = c;
    g.out = out;
    g.out_bf16 = out_dtype == QK_BF16;
    g.zp = zp;
    g.wsum = wsum;
    return cuda_status(gemv::launch(g, dev->sms, s), "gemv launch");
  }
  gemm::Args g = {};
  g.m = m;
  g.n = n;
  g.k = k;
  g.sa = scale_a;
  g.sw = scale_b;
  g.alpha = output_scale;
  g.c = c;
  g.out = out;
  g.out_bf16 = out_dtype == QK_BF16;
  g.sk.splits = 1;  // the split-K plan is the launcher's
  g.asym.zp = zp;
  g.asym.wsum = wsum;
  cudaError_t e = cudaSuccess;
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  int r = 0;
  if (path == GemmPath::kTensorPair) {
    r = gemm::launch_pair(g, a, b, dev_id, dev->sms, workspace, s, &e);
  } else {
    r = gemm::launch(g, a, b, path == GemmPath::kTensorGroup, dev_id, dev->sms, s, &e,
                     need > 0 ? workspace : nullptr);
  }
  if (r == 1) return cuda_status(cudaErrorInvalidValue, "tensor map encoding");
  return r == 0 ? QK_OK : cuda_status(e, "gemm launch");
}
}  // namespace

const char* qk_w8a8_gemm_kernel(int m, int n, int k, int group_k, int with_c) {
  thread_local char text[160];
  if (gemm_check(m, n, k, group_k) != QK_OK) return "unsupported";
  if (m == 0 || n == 0) return "none (empty output)";
  const DeviceInfo* dev = nullptr;
  if (check_device(&dev) != QK_OK) return "no device";
  int dev_id = 0;
  if (cudaGetDevice(&dev_id) != cudaSuccess) return "no device";
  switch (gemm_path(m, n, k, group_k)) {
    case GemmPath::kGemv:
      return gemv::pref_supported(m, k) ? "gemv_i8_prefetch_kernel (CUDA cores, dp4a)"
                                        : "gemv_i8_kernel (CUDA cores, dp4a)";
    case GemmPath::kTensorChannel: {
      const gemm::ChannelPlan pl = gemm::channel_plan(m, n, k, dev->sms, dev_id);
      if (pl.splits > 1)
        snprintf(text, sizeof text,
                 "gemm_i8_channel_kernel (1 SM, 128x%d tiles, cluster split-K in %d slices)", pl.bn,
                 pl.splits);
      else
        snprintf(text, sizeof text, "gemm_i8_channel_kernel (1 SM, 128x%d tiles)", pl.bn);
      return text;
    }
    case GemmPath::kTensorPair: {
      const int pairs = gemm::max_pairs(dev_id, dev->sms);
      const gemm::PairPlan pl = gemm::pair_plan(m, n, k, pairs, dev_id);
      const bool split = pl.splits > 1 && static_cast<int64_t>(pl.tiles) * pl.splits <= pairs;
      if (pl.tail_splits > 1)
        snprintf(text, sizeof text,
                 "gemm_i8_pair_kernel (CTA pair, 256x256 tiles, last wave cut into %d K slices)",
                 pl.tail_splits);
      else if (split && pl.csplit)
        snprintf(text, sizeof text,
                 "gemm_i8_pair_kernel (CTA pair, 256x256 tiles, cluster split-K in %d slices)",
                 pl.splits);
      else if (split)
        snprintf(text, sizeof text,
                 "gemm_i8_pair_kernel (CTA pair, 256x256 tiles, split-K in %d slices through the "
                 "workspace)",
                 pl.splits);
      else
        snprintf(text, sizeof text, "gemm_i8_pair_kernel (CTA pair, 256x256 tiles)");
      return text;
    }
    case GemmPath::kTensorGroup:
      break;
  }
  if (with_c || !gemm::group_wide_ok(dev_id))
    return "gemm_i8_group_kernel (1 SM, 128x128 tiles)";
  return gemm::group_plan(m, n, k, dev_id, dev->sms).pair
             ? "gemm_i8_group_pair_kernel (CTA pair, 256x256 tiles)"
             : "gemm_i8_group_wide_kernel (1 SM, 128x256 tiles)";
}

qk_status qk_fp8_gemm(int m, int n, int k, const uint8_t* a, const uint8_t* b,
                      const float* scale_a, const float* scale_b, float output_scale, void* out,
                      qk_dtype out_dtype, qk_stream stream) {
  if (m < 0 || n < 0 || k <= 0 || (k % 16) != 0 || (n % 8) != 0) return QK_ERR_INVALID_ARG;
  if (out_dtype != QK_F32 && out_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return QK_OK;
  if (a == nullptr || b == nullptr || scale_a == nullptr || scale_b == nullptr || out == nullptr)
    return QK_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16) || !aligned(scale_a, 16) ||
      !aligned(scale_b, 16))
    return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  gemm::Args g = {};
  g.m = m;
  g.n = n;
  g.k = k;
  g.sa = scale_a;
  g.sw = scale_b;
  g.alpha = output_scale;
  g.c = nullptr;
  g.out = out;
  g.out_bf16 = out_dtype == QK_BF16;
  g.sk.splits = 1;
  g.f8 = 1;
  cudaError_t e = cudaSuccess;
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int8_t* ai = reinterpret_cast<const int8_t*>(a);
  const int8_t* bi = reinterpret_cast<const int8_t*>(b);
  // m <= 128: the 1-SM kernel (rows beyond m read as zero); otherwise the
  // CTA-pair kernel.  Few tiles: split-K over the CTAs of a cluster (no
  // workspace); otherwise whole tiles.
  const int r = m <= 128 ? gemm::launch(g, ai, bi, false, dev_id, dev->sms, s, &e)
                         : gemm::launch_pair(g, ai, bi, dev_id, dev->sms, nullptr, s, &e);
  if (r == 1) return cuda_status(cudaErrorInvalidValue, "tensor map encoding");
  return r == 0 ? QK_OK : cuda_status(e, "fp8 gemm launch");
}

// The linear layer's workspace: the GEMM's own (offset 0, so its
// zero-on-return contract covers it), then 256 bytes of flags for the fused
// decode kernel (zero before and after every call, like the GEMM's part),
// then q [m, k] int8, then the scales.
namespace {
inline size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
constexpr size_t kLinearFlagBytes = 256;  // m + 1 <= 64 ints (the fused form has m <= 8)
}  // namespace

size_t qk_w8a8_linear_workspace_size(int m, int n, int k, int group_k) {
  if (gemm_check(m, n, k, group_k) != QK_OK || m == 0 || n == 0) return 0;
  const size_t g = round256(qk_w8a8_gemm_workspace_size(m, n, k, group_k));
  return g + kLinearFlagBytes + round256(static_cast<size_t>(m) * static_cast<size_t>(k)) +
         round256(static_cast<size_t>(m) * 4);
}

qk_status qk_w8a8_linear(int m, int n, int k, const void* x, qk_dtype x_dtype, const int8_t* b,
                         const float* scale_b, int group_k, float output_scale,
                         float* scale_a_out, void* out, qk_dtype out_dtype, void* workspace,
                         size_t workspace_bytes, qk_stream stream) {
  qk_status st = gemm_check(m, n, k, group_k);
  if (st != QK_OK) return st;
  if (x_dtype != QK_F32 && x_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (out_dtype != QK_F32 && out_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return QK_OK;
  if (x == nullptr || b == nullptr || scale_b == nullptr || out == nullptr)
    return QK_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(b, 16) || !aligned(scale_b, 16) || !aligned(out, 16) ||
      !aligned(scale_a_out, 4))
    return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  st = check_device(&dev);
  if (st != QK_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t need = qk_w8a8_linear_workspace_size(m, n, k, group_k);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256))
    return QK_ERR_WORKSPACE;
  // workspace: [GEMM workspace | flag words of qk_w8a8_linear_fused | q | scales]
  const size_t g_bytes = round256(qk_w8a8_gemm_workspace_size(m, n, k, group_k));
  int8_t* q = reinterpret_cast<int8_t*>(static_cast<char*>(workspace) + g_bytes + kLinearFlagBytes);
  float* sa = reinterpret_cast<float*>(static_cast<char*>(workspace) + g_bytes + kLinearFlagBytes +
                                       round256(static_cast<size_t>(m) * static_cast<size_t>(k)));
  st = quant_common(m, k, x, nullptr, k, x_dtype, q, sa, stream, false);
  if (st != QK_OK) return st;
  st = qk_w8a8_gemm(m, n, k, q, b, sa, scale_b, group_k, output_scale, nullptr, out, out_dtype,
                    g_bytes > 0 ? workspace : nullptr, g_bytes, stream);
  if (st != QK_OK || scale_a_out == nullptr) return st;
  return cuda_status(cudaMemcpyAsync(scale_a_out, sa, static_cast<size_t>(m) * 4,
                                     cudaMemcpyDeviceToDevice, s),
                     "scale copy");
}

qk_status qk_w8a8_linear_fused(int m, int n, int k, const void* x, qk_dtype x_dtype, const int8_t* b,
                               const float* scale_b, float output_scale, float* scale_a_out, void* out,
                               qk_dtype out_dtype, void* workspace, size_t workspace_bytes,
                               qk_stream stream) {
  qk_status st = gemm_check(m, n, k, 0);
  if (st != QK_OK) return st;
  if (x_dtype != QK_F32 && x_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (out_dtype != QK_F32 && out_dtype != QK_BF16) return QK_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return QK_OK;
  if (x == nullptr || b == nullptr || scale_b == nullptr || out == nullptr)
    return QK_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(b, 16) || !aligned(scale_b, 16) || !aligned(out, 16) ||
      !aligned(scale_a_out, 4))
    return QK_ERR_MISALIGNED;
  if (gemm_path(m, n, k, 0) != GemmPath::kGemv || !gemv::pref_supported(m, k))
    return QK_ERR_UNSUPPORTED;
  const DeviceInfo* dev = nullptr;
  st = check_device(&dev);
  if (st != QK_OK) return st;
  const size_t need = qk_w8a8_linear_workspace_size(m, n, k, 0);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256))
    return QK_ERR_WORKSPACE;
  // the workspace layout of qk_w8a8_linear (the GEMV takes no GEMM workspace)
  const size_t g_bytes = round256(qk_w8a8_gemm_workspace_size(m, n, k, 0));
  int* flags = reinterpret_cast<int*>(static_cast<char*>(workspace) + g_bytes);
  int8_t* q = reinterpret_cast<int8_t*>(static_cast<char*>(workspace) + g_bytes + kLinearFlagBytes);
  float* sa = reinterpret_cast<float*>(static_cast<char*>(workspace) + g_bytes + kLinearFlagBytes +
                                       round256(static_cast<size_t>(m) * static_cast<size_t>(k)));
  gemv::FusedArgs fa = {};
  fa.g.m = m;
  fa.g.n = n;
  fa.g.k = k;
  fa.g.a = q;
  fa.g.w = b;
  fa.g.sa = sa;
  fa.g.sw = scale_b;
  fa.g.alpha = output_scale;
  fa.g.out = out;
  fa.g.out_bf16 = out_dtype == QK_BF16;
  fa.x = x;
  fa.flags = flags;
  int dev_id = 0;
  cudaGetDevice(&dev_id);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  const bool launched = x_dtype == QK_BF16 ? gemv::launch_fused<true>(fa, dev_id, dev->sms, s, &e)
                                           : gemv::launch_fused<false>(fa, dev_id, dev->sms, s, &e);
  if (!launched) return QK_ERR_UNSUPPORTED;
  st = cuda_status(e, "fused decode launch");
  if (st != QK_OK || scale_a_out == nullptr) return st;
  return cuda_status(cudaMemcpyAsync(scale_a_out, sa, static_cast<size_t>(m) * 4,
                                     cudaMemcpyDeviceToDevice, s),
                     "scale copy");
}

qk_status qk_w8a8_gemm_noalloc(int m, int n, int k, const int8_t* a, const int8_t* b,
                               const float* scale_a, const float* scale_b, int group_k,
                               float output_scale, int32_t* c, void* out, qk_dtype out_dtype,
                               qk_stream stream) {
  const qk_status st = gemm_check(m, n, k, group_k);
  if (st != QK_OK) return st;
  const size_t need = qk_w8a8_gemm_workspace_size(m, n, k, group_k);
  if (need == 0)
    return qk_w8a8_gemm(m, n, k, a, b, scale_a, scale_b, group_k, output_scale, c, out,
                        out_dtype, nullptr, 0, stream);
  if (need > QK_NOALLOC_SCRATCH_BYTES) return QK_ERR_WORKSPACE;
  void* scratch = noalloc_scratch();
  if (scratch == nullptr) return QK_ERR_CUDA;
  // The arrival counters, the group split's flags and the split-K
  // accumulators must start at zero (partials and running sums need no
  // initialisation).
  gemm::PairPlan pl;
  gemm::GroupPlan gp;
  const size_t zero = group_plan_for(m, n, k, group_k, &gp) ? gemm::group_plan_flag_bytes(gp)
                      : pair_plan_for(m, n, k, group_k, &pl) ? gemm::pair_workspace_zero_bytes(pl)
                                                             : need;
  if (cudaMemsetAsync(scratch, 0, zero, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return QK_ERR_CUDA;
  return qk_w8a8_gemm(m, n, k, a, b, scale_a, scale_b, group_k, output_scale, c, out, out_dtype,
                      scratch, QK_NOALLOC_SCRATCH_BYTES, stream);
}

qk_status qk_device_status(qk_stream stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return QK_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, qk::g_status, sizeof v) != cudaSuccess) return QK_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(qk::g_status, &zero, sizeof zero) != cudaSuccess) return QK_ERR_CUDA;
  return static_cast<qk_status>(v);
}

qk_status qk_selftest_bounded_wait(int timeout_us, qk_stream stream) {
  if (timeout_us < 1 || timeout_us > 2000000) return QK_ERR_INVALID_ARG;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? QK_OK : QK_ERR_CUDA;
}

qk_status qk_selftest_silu(uint32_t first, uint64_t count, unsigned long long* mismatches,
                           uint32_t* first_mismatch, qk_stream stream) {
  if (count == 0 || count > (1ull << 32) || static_cast<uint64_t>(first) + count > (1ull << 32) ||
      mismatches == nullptr)
    return QK_ERR_INVALID_ARG;
  if (!aligned(mismatches, 8) || !aligned(first_mismatch, 4)) return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  const uint64_t pairs = (count + 1) / 2;
  uint64_t blocks = (pairs + 255) / 256;
  const uint64_t cap = static_cast<uint64_t>(dev->sms) * 8;
  if (blocks > cap) blocks = cap;
  selftest_silu_kernel<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      first, count, mismatches, first_mismatch);
  return cuda_status(cudaGetLastError(), "silu selftest launch");
}

qk_status qk_selftest_mma_rate(int cta_group, int n, int iters, int ctas, uint32_t operand_seed,
                               unsigned long long* cycles, qk_stream stream) {
  if ((cta_group != 1 && cta_group != 2) || n < 32 || n > 256 || (n % 16) != 0)
    return QK_ERR_INVALID_ARG;
  if (iters < 1 || iters > (1 << 20) || ctas < 1 || ctas > 65535 || (ctas % cta_group) != 0)
    return QK_ERR_INVALID_ARG;
  if (!aligned(cycles, 8)) return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  return cuda_status(probe::launch(cta_group == 2, n, iters, ctas, operand_seed, cycles,
                                   reinterpret_cast<cudaStream_t>(stream)),
                     "mma rate probe launch");
}

qk_status qk_selftest_mma_interference(int companion, int groups, int ctas, unsigned long long* cycles,
                                       qk_stream stream) {
  if (companion < 0 || companion > 6 || groups < 1 || groups > (1 << 18) || ctas < 2 || ctas > 65535 ||
      (ctas % 2) != 0)
    return QK_ERR_INVALID_ARG;
  if (!aligned(cycles, 8)) return QK_ERR_MISALIGNED;
  const DeviceInfo* dev = nullptr;
  const qk_status st = check_device(&dev);
  if (st != QK_OK) return st;
  return cuda_status(probe::launch_mix(companion, groups, ctas, cycles, reinterpret_cast<cudaStream_t>(stream)),
                     "mma interference probe launch");
}

}  // extern "C"
