// Masked INT8 GEMM with fused dequantization on the 5th-generation tensor cores (sm_100a).
//
//   acc[m, c] = sum_k xq[m, k] * W_k[c, k],   W_k = W & ~(2^k - 1),  k = 8 - bits[layer][step]
//   y[m, c]   = acc[m, c] * s_x[m] * s_w[c]    (or raw acc for the INT32 test epilogue)
//
// The weight mask is the TASQ temporal-spatial LSB mask (TASQ technical summary, section 2,
// "Representacao de Peso Compartilhada e Mascaramento de LSB": the stored 8-bit weight with
// its least-significant bit planes truncated per layer and stage); the integer GEMM plus FP
// rescale is HQ-DM's "core computation is integer matrix products" (section 2.1, "Eficiencia
// de Hardware"). The bit width is read from the device schedule table inside the kernel, so a
// new step needs no new weights and no different kernel.
//
// Design (one persistent CTA per SM, warp-specialised, 320 threads):
//   tile            128 output channels x 256 tokens; the weight tile is the MMA's A operand
//                   (M = 128), the activation-code tile its B operand (N = 256); K advances in
//                   stages of 128 bytes = four tcgen05.mma.kind::i8 of K = 32.
//   warp 4          TMA producer: loads the 16 KB weight tile and the 32 KB code tile of each
//                   stage into 128-byte-swizzled shared memory (4 stages in flight).
//   warps 6-9       mask warps (only when k > 0): AND every weight byte of a landed stage with
//                   0xFF << k in place (layout-agnostic, 8 x 16 B per thread), fence the
//                   generic-proxy writes to the async proxy and release the stage to the MMA.
//   warp 5          TMEM allocation (512 columns = two 256-column INT32 accumulators) and the
//                   single MMA-issuing thread; tcgen05.commit frees stages and publishes
//                   finished accumulators.
//   warps 0-3       epilogue: tcgen05.ld 32 lanes x 32 columns, scale, convert, store. Thread =
//                   output channel, so a warp's store of one token row is 32 consecutive
//                   channels. The accumulator is released as soon as it has been read, so the
//                   MMA of the next tile overlaps the stores of this one.
// Every wait is bounded (ptx::wait_bounded); a wait that runs out records a status bit, raises
// a CTA-wide abort flag, and every role winds down: the producer waits (bounded) for the loads
// it issued, the MMA thread for its MMAs, then TMEM is freed and the CTA exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/tasq.h"
#include "ptx.cuh"
#include "tasq_internal.h"

namespace tasq {
namespace {

constexpr int kTileCh = kGemmTileCh;      // 128
constexpr int kTileTok = kGemmTileTok;    // 256
constexpr int kBlockK = kGemmBlockK;      // 128 bytes
constexpr int kUmmaK = 32;
constexpr int kStages = 4;
constexpr int kABytes = kTileCh * kBlockK;
constexpr int kBBytes = kTileTok * kBlockK;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kAccCols = kTileTok;
constexpr int kAccStages = 2;
constexpr uint32_t kTmemCols = kAccCols * kAccStages;   // 512: the whole TMEM of the SM
constexpr int kEpiWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kMaskWarp0 = 6;
constexpr int kMaskWarps = 4;
constexpr int kThreads = 32 * (kEpiWarps + 2 + kMaskWarps);
constexpr int kMaskThreads = 32 * kMaskWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;

constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kNumBars = 3 * kStages + 2 * kAccStages + 1;
constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOffset + kNumBars * 8 + 16;

static_assert(kABytes % (16 * kMaskThreads) == 0, "mask pass must tile the weight stage");
static_assert(kTileTok % 16 == 0 && kTileTok <= 256, "UMMA N");
static_assert(kBlockK % kUmmaK == 0, "stage K");

struct Bars {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t masked(int s) const { return base + 8u * (kStages + s); }
  __device__ uint32_t empty(int s) const { return base + 8u * (2 * kStages + s); }
  __device__ uint32_t acc_full(int i) const { return base + 8u * (3 * kStages + i); }
  __device__ uint32_t acc_empty(int i) const { return base + 8u * (3 * kStages + kAccStages + i); }
  __device__ uint32_t drain() const { return base + 8u * (3 * kStages + 2 * kAccStages); }
};

__device__ __forceinline__ void raise_failure(uint32_t* status, volatile int* abort_flag, uint32_t bit) {
  atomicOr(status, bit);
  *abort_flag = 1;
}

template <int OUT>
__device__ __forceinline__ void store_out(void* y, int64_t idx, float v, uint32_t raw) {
  if constexpr (OUT == static_cast<int>(OutKind::S32)) {
    static_cast<int32_t*>(y)[idx] = static_cast<int32_t>(raw);
  } else if constexpr (OUT == static_cast<int>(OutKind::F16)) {
    static_cast<__half*>(y)[idx] = __float2half_rn(v);
  } else {
    static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
  }
}

template <int OUT>
__global__ void __launch_bounds__(kThreads, 1)
    masked_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                       const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const Bars bars{sbase + kBarOffset};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOffset + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // schedule lookup: the step's bit width for this layer
  int bits = g.bits_table[g.bits_index];
  if (bits < 1 || bits > 8) {
    if (threadIdx.x == 0) atomicOr(g.status, TASQ_DEVICE_BAD_BITS);
    bits = 8;
  }
  const int k_drop = 8 - bits;
  const bool masking = k_drop > 0;
  const uint32_t mask32 = 0x01010101u * ((0xFFu << k_drop) & 0xFFu);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.masked(s), kMaskThreads);
      ptx::mbar_init(bars.empty(s), 1);
    }
    for (int i = 0; i < kAccStages; ++i) {
      ptx::mbar_init(bars.acc_full(i), 1);
      ptx::mbar_init(bars.acc_empty(i), kEpiThreads);
    }
    ptx::mbar_init(bars.drain(), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_x);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::tc_fence_after_sync();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  const int num_tiles = g.num_m_tiles * g.num_n_tiles;
  const uint64_t limit = g.wait_limit_ns;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      uint32_t s = 0, ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mt = tile % g.num_m_tiles;
        const int nt = tile / g.num_m_tiles;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!ptx::wait_bounded(bars.empty(s), ph ^ 1u, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bars.full(s), kStageBytes);
          ptx::tma_load_2d(sbase + s * kABytes, &tmap_w, bars.full(s), kb * kBlockK, nt * kTileCh);
          ptx::tma_load_2d(sbase + kStages * kABytes + s * kBBytes, &tmap_x, bars.full(s), kb * kBlockK,
                           mt * kTileTok);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // every load this thread issued must have landed before the CTA may exit
      for (int i = 0; i < kStages; ++i) {
        if ((issued >> i) & 1u) {
          if (!ptx::wait_bounded(bars.full(i), (issued_par >> i) & 1u, limit, nullptr))
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = ptx::idesc_i8_s32(kTileCh, kTileTok);
      uint32_t s = 0, ph = 0, as = 0, aph = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!ptx::wait_bounded(bars.acc_empty(as), aph ^ 1u, limit, abort_flag)) {
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
          break;
        }
        ptx::tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + as * kAccCols;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          const uint32_t ready = masking ? bars.masked(s) : bars.full(s);
          if (!ptx::wait_bounded(ready, ph, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
          const uint64_t a_desc = ptx::smem_desc_k_sw128(sbase + s * kABytes);
          const uint64_t b_desc = ptx::smem_desc_k_sw128(sbase + kStages * kABytes + s * kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBlockK / kUmmaK; ++kk) {
            // +32 bytes along K inside the 128-byte swizzle row = +2 in the address field
            ptx::mma_i8_ss(d_tmem, a_desc + 2u * kk, b_desc + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          ptx::mma_commit(bars.empty(s));
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(bars.acc_full(as));
        as ^= 1u;
        if (as == 0) aph ^= 1u;
      }
      // every MMA this thread issued must have completed before TMEM is freed
      if (issued_any) {
        ptx::mma_commit(bars.drain());
        if (!ptx::wait_bounded(bars.drain(), 0, limit, nullptr))
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_DRAIN);
      }
    }
  } else if (warp >= kMaskWarp0) {
    // -------------------------------------------------------------------- mask warps
    if (masking) {
      const int t = threadIdx.x - kMaskWarp0 * 32;
      uint32_t s = 0, ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!ptx::wait_bounded(bars.full(s), ph, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MASK);
            ok = false;
            break;
          }
          uint4* wt = reinterpret_cast<uint4*>(smem + s * kABytes);
#pragma unroll
          for (int i = 0; i < kABytes / 16 / kMaskThreads; ++i) {
            uint4 w = wt[i * kMaskThreads + t];
            w.x &= mask32;
            w.y &= mask32;
            w.z &= mask32;
            w.w &= mask32;
            wt[i * kMaskThreads + t] = w;
          }
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(bars.masked(s));
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue warps
    const int ew = warp;  // == warp % 4: this warp may access TMEM lanes [32 ew, 32 ew + 32)
    uint32_t as = 0, aph = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mt = tile % g.num_m_tiles;
      const int nt = tile / g.num_m_tiles;
      const bool got = ptx::wait_bounded(bars.acc_full(as), aph, limit, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_EPILOGUE);
        break;
      }
      ptx::tc_fence_after_sync();
      const int ch = nt * kTileCh + ew * 32 + lane;
      const bool ch_ok = ch < g.N;
      float sw = 0.0f;
      if constexpr (OUT != static_cast<int>(OutKind::S32)) {
        if (ch_ok) sw = g.s_w[ch];
      }
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + as * kAccCols;
#pragma unroll 1
      for (int chunk = 0; chunk < kTileTok / 32; ++chunk) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(tacc + chunk * 32, r);
        ptx::tmem_ld_wait();
        if (chunk == kTileTok / 32 - 1) {
          // the accumulator has been read: hand it back to the MMA before storing
          ptx::tc_fence_before_sync();
          ptx::mbar_arrive(bars.acc_empty(as));
        }
        const int t0 = mt * kTileTok + chunk * 32;
        if (t0 >= g.M) continue;
        float sx_lane = 0.0f;
        if constexpr (OUT != static_cast<int>(OutKind::S32)) {
          if (t0 + lane < g.M) sx_lane = g.s_x[t0 + lane];
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float sxj = __shfl_sync(0xffffffffu, sx_lane, j);
          const float v = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(r[j])), sxj), sw);
          if (ch_ok && t0 + j < g.M) store_out<OUT>(g.y, static_cast<int64_t>(t0 + j) * g.ldy + ch, v, r[j]);
        }
      }
      as ^= 1u;
      if (as == 0) aph ^= 1u;
    }
  }

  __syncwarp();
  ptx::tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int OUT>
cudaError_t launch_out(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& g, int num_sms,
                       cudaStream_t stream) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(masked_gemm_kernel<OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int tiles = g.num_m_tiles * g.num_n_tiles;
  const int grid = tiles < num_sms ? tiles : num_sms;
  masked_gemm_kernel<OUT><<<grid, kThreads, kSmemBytes, stream>>>(tw, tx, g);
  return cudaGetLastError();
}

__global__ void stuck_wait_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_addr(&bar), 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on this barrier: the wait has to run out
    if (!ptx::wait_bounded(ptx::smem_addr(&bar), 0, limit_ns, nullptr)) atomicOr(status, TASQ_DEVICE_TIMEOUT_MMA);
  }
}

}  // namespace

cudaError_t launch_masked_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const GemmArgs& g,
                               OutKind out, int num_sms, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  switch (out) {
    case OutKind::F16: return launch_out<static_cast<int>(OutKind::F16)>(tmap_w, tmap_x, g, num_sms, stream);
    case OutKind::BF16: return launch_out<static_cast<int>(OutKind::BF16)>(tmap_w, tmap_x, g, num_sms, stream);
    case OutKind::S32: return launch_out<static_cast<int>(OutKind::S32)>(tmap_w, tmap_x, g, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_stuck_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t stream) {
  stuck_wait_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace tasq
