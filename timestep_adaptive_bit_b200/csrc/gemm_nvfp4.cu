// Block-scaled NVFP4 GEMM with fused dequantization on the 5th-generation tensor cores (sm_100a),
// the GEMM of an NVFP4 step (6Bit-Diffusion technical summary, section 2.A: stable layers are
// compressed to NVFP4, Blackwell's native 4-bit format, beside the INT8 path):
//
//   acc[m, c] = sum over 16-blocks b of  sx4[m, b] * sw4[c, b] * sum_{k in b} ex[m, k] * ew[c, k]
//   y[m, c]   = acc[m, c] * s_x[m] * s_w[c]         (or the raw FP32 acc for the test hook)
//
// with E2M1 codes ex, ew and UE4M3 block scales sx4, sw4 made by the NVFP4 prologue launch.
//
// Design (one persistent CTA per SM, warp-specialised, 320 threads):
//   tile       128 output channels x 128 tokens; the weight codes are the MMA's A operand (M = 128),
//              the token codes its B operand (N = 128). A stage covers 256 elements of K: 128
//              bytes of codes per row (128-byte swizzle, as in the INT8 kernels) plus the four
//              512-byte scale chunks of each operand (four MMAs of K = 64).
//   warp 8     producer: two TMA tile loads and two 2 KB bulk copies of scale chunks per stage
//              (5 stages in flight).
//   warp 9     TMEM allocation (two 128-column FP32 accumulators and 32 columns of scales) and the
//              single issuing thread: per stage it copies the eight scale chunks into TMEM with
//              tcgen05.cp (32x128b.warpx4: row i of a chunk to lane i of every lane quarter) and
//              issues the four block-scaled MMAs, all in one ordered stream.
//   warps 0-7  the INT8 kernels' epilogue, reading FP32 accumulators.
// Every wait is bounded; a wait that runs out records a status bit, raises the CTA's abort flag,
// and every role winds down as in the INT8 kernels.
#include <mutex>

#include "gemm_common.cuh"

namespace tasq {
namespace {

using namespace gemm;

constexpr int kTileCh = 128;                   // weight rows per tile (MMA M)
constexpr int kTileTok = 128;                  // token rows per tile (MMA N)
constexpr int kCodeBytes = 128;                // bytes of codes per row and stage (256 elements)
constexpr int kABytes = kTileCh * kCodeBytes;  // 16 KB
constexpr int kBBytes = kTileTok * kCodeBytes; // 16 KB
constexpr int kSfBytes = 4 * kNvfp4ChunkBytes; // four K = 64 chunks of 128 rows: 2 KB per operand
constexpr int kStageBytes = kABytes + kBBytes + 2 * kSfBytes;
constexpr int kStages = 5;
constexpr int kWarps = kEpiWarps + 2;
constexpr int kThreadsF4 = 32 * kWarps;
constexpr uint32_t kAccColsF4 = 128;           // one accumulator: 128 FP32 columns
constexpr uint32_t kSfCol = 2 * kAccColsF4;    // scales of A at columns 256..271, of B at 272..287
static_assert(kEpiWarps == 8 && kProducerWarp == 8 && kMmaWarp == 9, "warp roles");

template <int OUT>
struct PlanF4 {
  static constexpr int kEpiOffset = kStages * kStageBytes;
  static constexpr int kSxOffset = kEpiOffset + kEpiWarps * OutTraits<OUT>::kStageBytes;
  static constexpr int kBarOffset = kSxOffset + kEpiWarps * kSxBytesPerWarp;
  static constexpr int kNumBars = 2 * kStages + 2 * kAccStages + 1;
  static constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOffset + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= kMaxSmem, "shared memory");
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
};

struct BarsF4 {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t empty(int s) const { return base + 8u * (kStages + s); }
  __device__ uint32_t acc_full(int i) const { return base + 8u * (2 * kStages + i); }
  __device__ uint32_t acc_empty(int i) const { return base + 8u * (2 * kStages + kAccStages + i); }
  __device__ uint32_t drain() const { return base + 8u * (2 * kStages + 2 * kAccStages); }
};

template <int OUT>
__global__ void __launch_bounds__(kThreadsF4, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_y, const GemmArgs g, const Nvfp4GemmArgs f) {
  using P = PlanF4<OUT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const BarsF4 bars{sbase + P::kBarOffset};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + P::kBarOffset + P::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  ptx::grid_dep_launch_dependents();
  if (g.bits_table != nullptr && gated_out(g.gate, g.bits_table, g.bits_index)) return;

  // the schedule entry of an NVFP4 step is 0
  if (threadIdx.x == 0 && g.bits_table != nullptr && g.bits_table[g.bits_index] != 0)
    atomicOr(g.status, TASQ_DEVICE_BAD_BITS);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.empty(s), 1);
    }
    for (int i = 0; i < kAccStages; ++i) {
      ptx::mbar_init(bars.acc_full(i), 1);
      ptx::mbar_init(bars.acc_empty(i), kEpiWarps);
    }
    ptx::mbar_init(bars.drain(), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_y);
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
  // stage s: A codes, B codes, A scales, B scales
  auto a_smem = [&](int s) { return sbase + static_cast<uint32_t>(s * kStageBytes); };
  auto b_smem = [&](int s) { return a_smem(s) + kABytes; };
  auto sfa_smem = [&](int s) { return b_smem(s) + kBBytes; };
  auto sfb_smem = [&](int s) { return sfa_smem(s) + kSfBytes; };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      uint32_t s = 0, ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      // the codes and scales come from the prologue kernel just before this one
      ptx::grid_dep_wait();
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, g.num_m_tiles, g.num_n_tiles, g.band_tiles, mt, nt);
        const uint8_t* sfa_src = f.w_sf + (static_cast<int64_t>(nt) * f.sf_chunks) * kNvfp4ChunkBytes;
        const uint8_t* sfb_src = f.x_sf + (static_cast<int64_t>(mt) * f.sf_chunks) * kNvfp4ChunkBytes;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!ptx::wait_bounded(bars.empty(s), ph ^ 1u, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bars.full(s), kStageBytes);
          ptx::tma_load_2d(a_smem(s), &tmap_w, bars.full(s), kb * kCodeBytes, nt * kTileCh);
          ptx::tma_load_2d(b_smem(s), &tmap_x, bars.full(s), kb * kCodeBytes, mt * kTileTok);
          ptx::bulk_load(sfa_smem(s), sfa_src + kb * kSfBytes, kSfBytes, bars.full(s));
          ptx::bulk_load(sfb_smem(s), sfb_src + kb * kSfBytes, kSfBytes, bars.full(s));
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      for (int i = 0; i < kStages; ++i) {
        if ((issued >> i) & 1u) {
          if (!ptx::wait_bounded(bars.full(i), (issued_par >> i) & 1u, limit, nullptr))
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_nvfp4(kTileCh, kTileTok);
      const uint32_t sfa_t = tmem_base + kSfCol;        // 4 chunks x 4 columns
      const uint32_t sfb_t = tmem_base + kSfCol + 16;   // 4 chunks x 4 columns
      uint32_t s = 0, ph = 0, as = 0, aph = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!ptx::wait_bounded(bars.acc_empty(as), aph ^ 1u, limit, abort_flag)) {
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
          break;
        }
        ptx::tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + as * kAccColsF4;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!ptx::wait_bounded(bars.full(s), ph, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            ptx::tmem_cp_32x128b_warpx4(sfa_t + 4u * c, ptx::smem_desc_rows16(sfa_smem(s) + c * kNvfp4ChunkBytes));
            ptx::tmem_cp_32x128b_warpx4(sfb_t + 4u * c, ptx::smem_desc_rows16(sfb_smem(s) + c * kNvfp4ChunkBytes));
          }
          const uint64_t a_desc = ptx::smem_desc_k_sw128(a_smem(s));
          const uint64_t b_desc = ptx::smem_desc_k_sw128(b_smem(s));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // +32 bytes (64 elements) along K inside the 128-byte swizzle row = +2 in the address field
            ptx::mma_nvfp4_ss(d_tmem, a_desc + 2u * kk, b_desc + 2u * kk, idesc, sfa_t + 4u * kk, sfb_t + 4u * kk,
                              (kb | kk) != 0 ? 1u : 0u);
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
      if (issued_any) {
        ptx::mma_commit(bars.drain());
        if (!ptx::wait_bounded(bars.drain(), 0, limit, nullptr))
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_DRAIN);
      }
    }
  } else {
    epilogue_role<OUT, false, kTileTok, true>(g, &tmap_y, tmem_base,
                                              smem + P::kEpiOffset + warp * OutTraits<OUT>::kStageBytes,
                                              reinterpret_cast<float*>(smem + P::kSxOffset + warp * kSxBytesPerWarp),
                                              warp, lane, blockIdx.x, gridDim.x, num_tiles, kTileCh, 0,
                                              bars.acc_full(0), bars.acc_empty(0), limit, abort_flag);
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
cudaError_t launch_f4(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ty, const GemmArgs& g,
                      const Nvfp4GemmArgs& f, int num_sms, cudaStream_t stream) {
  static bool configured[64] = {false};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      e = cudaFuncSetAttribute(gemm_nvfp4_kernel<OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PlanF4<OUT>::kSmemBytes);
      if (e != cudaSuccess) return e;
      configured[dev] = true;
    }
  }
  const int tiles = g.num_m_tiles * g.num_n_tiles;
  const int grid = tiles < num_sms ? tiles : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreadsF4, 1, 1);
  cfg.dynamicSmemBytes = PlanF4<OUT>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = use_pdl() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_kernel<OUT>, tw, tx, ty, g, f);
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const CUtensorMap& tmap_y,
                              const GemmArgs& g, const Nvfp4GemmArgs& f, OutKind out, int num_sms,
                              cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (reinterpret_cast<uintptr_t>(f.w_sf) % 16 != 0 || reinterpret_cast<uintptr_t>(f.x_sf) % 16 != 0 ||
      f.sf_chunks != g.num_kb * 4)
    return cudaErrorInvalidValue;
  switch (out) {
    case OutKind::F16:
      return launch_f4<static_cast<int>(OutKind::F16)>(tmap_w, tmap_x, tmap_y, g, f, num_sms, stream);
    case OutKind::BF16:
      return launch_f4<static_cast<int>(OutKind::BF16)>(tmap_w, tmap_x, tmap_y, g, f, num_sms, stream);
    case OutKind::S32:
      return launch_f4<static_cast<int>(OutKind::S32)>(tmap_w, tmap_x, tmap_y, g, f, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tasq
