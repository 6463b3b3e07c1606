// tasq_linear_forward_noalloc: the masked INT8 linear for callers that cannot allocate device
// memory, e.g. code running inside an allocator callback, a host that owns every byte of device
// memory through its own arena, or a capture/replay harness that forbids cudaMalloc. The pages
// have no counterpart; this is a deployment convenience around the same two kernels.
//
// The activation codes and scales that tasq_linear_forward keeps in its context workspace live
// here in one file-scope device array of fixed size, reserved once per device when the library's
// module is loaded and held until the process exits. The caller passes inputs and outputs; the
// entry point itself calls no cudaMalloc, cudaFree or allocating library routine.
//
// Host code must not use the array's name as a device address (in host code it is a host-side
// stand-in): the device address is fetched with cudaGetSymbolAddress on the first call made with
// a device current, and cached together with the CUDA context it belongs to. A call made under
// another context of that device (a non-primary driver context, or the primary one created anew
// after cudaDeviceReset, where the module and its array are loaded again) looks the address up
// again instead of using a stale one.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>
#include <string>

#include "../../include/tasq.h"
#include "tasq_internal.h"

namespace {

// [0, 256): control block (byte 0: the bit width the GEMM reads; bytes 4..7: the status word of
// calls made with device_status == NULL); [256, ...): per-token scales, then the INT8 codes at a
// 1024-byte aligned offset.
static __device__ __align__(256) unsigned char g_tasq_noalloc_scratch[TASQ_NOALLOC_SCRATCH_BYTES];

constexpr size_t kSxOffset = 256;
constexpr size_t kStatusOffset = 4;

// Bytes of the array one call needs: the control block and M scales, rounded up to 1 KiB, then
// M * Kp codes.
size_t scratch_bytes(int64_t M, int32_t Kp) {
  return tasq::round_up(kSxOffset + static_cast<size_t>(M) * sizeof(float), 1024) +
         static_cast<size_t>(M) * static_cast<size_t>(Kp);
}

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
unsigned char* g_scratch_ptr[kMaxDevices] = {nullptr};
CUcontext g_scratch_ctx[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// The array's device address under the current context of device `dev` (and the device's SM
// count), looked up on the first call under that context. A call with no context current yet gets
// the runtime's primary context from the lookup itself.
tasq_status device_setup(int dev, unsigned char** scratch, int* num_sms) {
  if (dev < 0 || dev >= kMaxDevices) return tasq::fail(TASQ_ERR_INVALID_ARG, "device index out of range");
  CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr) return tasq::fail(TASQ_ERR_CUDA, "cuCtxGetCurrent is not available from the driver");
  CUcontext cur = nullptr;
  if (get(&cur) != CUDA_SUCCESS) return tasq::fail(TASQ_ERR_CUDA, "cuCtxGetCurrent failed");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (cur == nullptr || g_scratch_ptr[dev] == nullptr || g_scratch_ctx[dev] != cur) {
    cudaDeviceProp prop;
    cudaError_t e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return tasq::fail_cuda(e, "cudaGetDeviceProperties");
    if (prop.major != 10 || prop.minor != 0)
      return tasq::fail(TASQ_ERR_UNSUPPORTED_ARCH, std::string("device ") + prop.name + " is not sm_100");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_tasq_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return tasq::fail_cuda(e, "cudaGetSymbolAddress(scratch)");
    if (get(&cur) != CUDA_SUCCESS || cur == nullptr) return tasq::fail(TASQ_ERR_CUDA, "no current CUDA context");
    g_num_sms[dev] = prop.multiProcessorCount;
    g_scratch_ptr[dev] = static_cast<unsigned char*>(p);
    g_scratch_ctx[dev] = cur;
  }
  *scratch = g_scratch_ptr[dev];
  *num_sms = g_num_sms[dev];
  return TASQ_OK;
}

}  // namespace

extern "C" tasq_status tasq_linear_forward_noalloc(const void* x, int64_t M, int64_t ldx, int32_t K, const int8_t* w,
                                                   const float* s_w, int32_t N, int32_t bits, int32_t hadamard_n,
                                                   void* y, int64_t ldy, int32_t out_dtype, uint32_t* device_status,
                                                   void* stream) {
  tasq::set_last_error("");
  using tasq::fail;
  if (hadamard_n != 64 && hadamard_n != 128) return fail(TASQ_ERR_INVALID_ARG, "hadamard_n must be 64 or 128");
  if (N <= 0 || K < 8 || K % 8 != 0) return fail(TASQ_ERR_INVALID_ARG, "need N >= 1 and K >= 8 with K % 8 == 0");
  if (bits < 1 || bits > 8) return fail(TASQ_ERR_INVALID_ARG, "bits must be in [1, 8]");
  if (out_dtype != TASQ_OUT_F16 && out_dtype != TASQ_OUT_BF16) return fail(TASQ_ERR_INVALID_ARG, "bad out_dtype");
  if (M < 0 || M > 0x7fffffffLL) return fail(TASQ_ERR_INVALID_ARG, "M out of range");
  const int32_t Kp = (K + hadamard_n - 1) / hadamard_n * hadamard_n;
  if (Kp > TASQ_MAX_KP) return fail(TASQ_ERR_INVALID_ARG, "padded K exceeds TASQ_MAX_KP");
  const size_t xq_off = tasq::round_up(kSxOffset + static_cast<size_t>(M) * sizeof(float), 1024);
  const size_t need = scratch_bytes(M, Kp);
  if (need > TASQ_NOALLOC_SCRATCH_BYTES)
    return fail(TASQ_ERR_WORKSPACE, "M = " + std::to_string(static_cast<long long>(M)) + " tokens at Kp = " +
                                        std::to_string(Kp) + " need " + std::to_string(need) +
                                        " bytes of the fixed scratch of " +
                                        std::to_string(static_cast<unsigned long long>(TASQ_NOALLOC_SCRATCH_BYTES)) +
                                        " bytes");
  if (x == nullptr || !tasq::aligned16(x) || ldx < K || ldx % 8 != 0)
    return fail(TASQ_ERR_INVALID_ARG, "x must be 16-byte aligned with a row stride >= K and % 8 == 0");
  if (y == nullptr || !tasq::aligned16(y) || ldy < N || ldy % 8 != 0)
    return fail(TASQ_ERR_INVALID_ARG, "y must be 16-byte aligned with a row stride >= N and % 8 == 0");
  if (w == nullptr || !tasq::aligned16(w) || s_w == nullptr)
    return fail(TASQ_ERR_INVALID_ARG, "w must be a 16-byte aligned [N, Kp] buffer and s_w non-NULL");
  if (M == 0) return TASQ_OK;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tasq::fail_cuda(e, "cudaGetDevice");
  unsigned char* scratch = nullptr;
  int num_sms = 0;
  tasq_status st = device_setup(dev, &scratch, &num_sms);
  if (st != TASQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  uint8_t* bits_byte = scratch;
  uint32_t* status =
      device_status != nullptr ? device_status : reinterpret_cast<uint32_t*>(scratch + kStatusOffset);
  float* s_x = reinterpret_cast<float*>(scratch + kSxOffset);
  int8_t* xq = reinterpret_cast<int8_t*>(scratch + xq_off);
  // the array keeps the previous call's contents: set the bit width, clear the fallback status
  if ((e = cudaMemsetAsync(bits_byte, bits, 1, s)) != cudaSuccess) return tasq::fail_cuda(e, "set bit width");
  if (device_status == nullptr && (e = cudaMemsetAsync(status, 0, sizeof(uint32_t), s)) != cudaSuccess)
    return tasq::fail_cuda(e, "clear status");

  tasq::PrologueArgs a{};
  a.x = x;
  a.ldx = ldx;
  a.K = K;
  a.Kp = Kp;
  a.M = M;
  a.xq = xq;
  a.s_x = s_x;
  a.n = hadamard_n;
  a.sx_factor = static_cast<float>(1.0 / (127.0 * std::sqrt(static_cast<double>(hadamard_n))));
  a.status = status;
  a.wait_limit_ns = 1000000000ull;
  a.num_sms = num_sms;
  tasq::g_last_error.clear();
  if ((e = tasq::launch_prologue(a, s)) != cudaSuccess) {
    // the launcher may have left a more precise message (a failed per-device kernel set-up)
    if (!tasq::g_last_error.empty()) return fail(TASQ_ERR_CUDA, "prologue launch: " + tasq::g_last_error);
    return tasq::fail_cuda(e, "prologue launch");
  }

  CUtensorMap tw, tx, ty;
  if ((st = tasq::make_tmap_u8(&tw, w, Kp, N, tasq::kGemmBlockK, tasq::kGemmTileCh)) != TASQ_OK) return st;
  if ((st = tasq::make_tmap_u8(&tx, xq, Kp, M, tasq::kGemmBlockK, tasq::kGemmTileTok)) != TASQ_OK) return st;
  const bool bf16 = out_dtype == TASQ_OUT_BF16;
  if ((st = tasq::make_tmap_out(&ty, y, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                                N, M, ldy)) != TASQ_OK)
    return st;
  tasq::GemmArgs g{};
  g.M = static_cast<int32_t>(M);
  g.N = N;
  g.num_kb = (Kp + tasq::kGemmBlockK - 1) / tasq::kGemmBlockK;
  g.num_m_tiles = static_cast<int32_t>((M + tasq::kGemmTileTok - 1) / tasq::kGemmTileTok);
  g.num_n_tiles = (N + tasq::kGemmTileCh - 1) / tasq::kGemmTileCh;
  g.band_tiles = tasq::gemm_band_tiles(g.num_m_tiles, tasq::kGemmTileTok, Kp);
  g.bits_table = bits_byte;
  g.bits_index = 0;
  g.s_x = s_x;
  g.s_w = s_w;
  g.y = y;
  g.ldy = ldy;
  g.status = status;
  g.wait_limit_ns = 1000000000ull;
  // the caller's weights, masked in shared memory by the GEMM's mask warps as they land
  e = tasq::launch_masked_gemm(tw, tx, ty, g, bf16 ? tasq::OutKind::BF16 : tasq::OutKind::F16, num_sms, s);
  if (e != cudaSuccess) return tasq::fail_cuda(e, "masked GEMM launch");
  return TASQ_OK;
}

extern "C" tasq_status tasq_noalloc_device_status(uint32_t* status_out, int32_t clear, void* stream) {
  tasq::set_last_error("");
  if (status_out == nullptr) return tasq::fail(TASQ_ERR_INVALID_ARG, "status_out is NULL");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tasq::fail_cuda(e, "cudaGetDevice");
  unsigned char* scratch = nullptr;
  int num_sms = 0;
  tasq_status st = device_setup(dev, &scratch, &num_sms);
  if (st != TASQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* word = reinterpret_cast<uint32_t*>(scratch + kStatusOffset);
  uint32_t v = 0;
  e = cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return tasq::fail_cuda(e, "read of the status word");
  if (clear) {
    e = cudaMemsetAsync(word, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return tasq::fail_cuda(e, "clear of the status word");
  }
  *status_out = v;
  return TASQ_OK;
}
