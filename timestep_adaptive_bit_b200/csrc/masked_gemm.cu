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
// Design (one persistent CTA per SM, warp-specialised, 576 threads; the pair kernel in
// masked_gemm_pair.cu shares the roles and the epilogue):
//   tile            128 output channels x 256 tokens; the weight tile is the MMA's A operand
//                   (M = 128), the activation-code tile its B operand (N = 256); K advances in
//                   stages of 128 bytes = four tcgen05.mma.kind::i8 of K = 32.
//   warp 8          TMA producer: loads the 16 KB weight tile and the 32 KB code tile of each
//                   stage into 128-byte-swizzled shared memory (4 stages in flight).
//   warps 10-17     mask warps, two groups of four taking alternate K blocks (one group on the
//                   3-stage ring of the INT32 test output; only when k > 0 and the weights were not
//                   masked ahead by the prologue launch): AND every
//                   weight byte of a landed stage with 0xFF << k in place (layout-agnostic,
//                   8 x 16 B per thread), fence the generic-proxy writes to the async proxy and
//                   release the stage to the MMA.
//   warp 9          TMEM allocation (512 columns = two 256-column INT32 accumulators) and the
//                   single MMA-issuing thread; tcgen05.commit frees stages and publishes
//                   finished accumulators.
//   warps 0-7       epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its 32 channels) and
//                   accumulator columns 128 (w / 4) .. +127 (its 128 tokens) in chunks of 32
//                   columns, scales, converts, writes a 32 x 32 tile into its private shared
//                   staging buffer in output row order and stores it with one TMA bulk store.
//                   The accumulator is released as soon as it has been read, so the MMA of the
//                   next tile overlaps the stores of this one. Warps never wait on each other.
// Every wait is bounded (ptx::wait_bounded); a wait that runs out records a status bit, raises
// a CTA-wide abort flag, and every role winds down: the producer waits (bounded) for the loads
// it issued, the MMA thread for its MMAs, then TMEM is freed and the CTA exits.
#include <mutex>

#include "gemm_common.cuh"

namespace tasq {
namespace {

using namespace gemm;

constexpr int kTileCh = kGemmTileCh;      // 128 output channels per tile
constexpr int kABytes = kTileCh * kBlockK;
constexpr int kMaxMaskGroups = 2;         // groups of kMaskWarps mask warps, taking alternate K blocks
constexpr int kThreads1 = kThreads + 32 * kMaskWarps * (kMaxMaskGroups - 1);

// Mask groups of a ring of STAGES stages. A group waits for the `full` barrier of every G-th K block.
// TMA loads may land out of order, so a group knows of no block's landing but its own: its parity
// wait for block j is unambiguous only if block j - STAGES (the slot's previous phase) is one of its
// own, i.e. STAGES is a multiple of G. The 4-stage ring takes two groups, the 3-stage one one.
template <int STAGES>
constexpr int mask_groups() {
  return STAGES % kMaxMaskGroups == 0 ? kMaxMaskGroups : 1;
}
static_assert(kABytes % (16 * kMaskThreads) == 0, "mask pass must tile the weight stage");

// Shared-memory plan of one instantiation: stages of (weights, codes), the epilogue's output
// staging (one 32 x 32 box per warp), its s_x slices, the barriers.
template <int OUT>
struct Plan {
  static constexpr int kTok = kGemmTileTok;
  static constexpr int kBBytes = kTok * kBlockK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = OutTraits<OUT>::kS32 ? 3 : 4;
  static constexpr int kEpiOffset = kStages * kStageBytes;
  static constexpr int kSxOffset = kEpiOffset + kEpiWarps * OutTraits<OUT>::kStageBytes;
  static constexpr int kBarOffset = kSxOffset + kEpiWarps * kSxBytesPerWarp;
  static constexpr int kNumBars = 3 * kStages + 2 * kAccStages + 1;
  static constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOffset + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= kMaxSmem, "shared memory");
  static_assert(kAccStages * kTok <= static_cast<int>(kTmemCols), "TMEM");
  static constexpr int kMaskGroups = mask_groups<kStages>();
  static_assert(kStages % kMaskGroups == 0, "a mask group's parity waits must stay unambiguous");
};

template <int STAGES>
struct Bars {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t masked(int s) const { return base + 8u * (STAGES + s); }
  __device__ uint32_t empty(int s) const { return base + 8u * (2 * STAGES + s); }
  __device__ uint32_t acc_full(int i) const { return base + 8u * (3 * STAGES + i); }
  __device__ uint32_t acc_empty(int i) const { return base + 8u * (3 * STAGES + kAccStages + i); }
  __device__ uint32_t drain() const { return base + 8u * (3 * STAGES + 2 * kAccStages); }
};

template <int OUT>
__global__ void __launch_bounds__(kThreads1, 1)
    masked_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_y, const GemmArgs g) {
  using P = Plan<OUT>;
  constexpr int kStages = P::kStages;
  constexpr int kTok = P::kTok;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const Bars<kStages> bars{sbase + P::kBarOffset};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + P::kBarOffset + P::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the next kernel of the stream may be scheduled; it waits for this one before reading
  ptx::grid_dep_launch_dependents();
  if (gated_out(g.gate, g.bits_table, g.bits_index)) return;

  // schedule lookup: the step's bit width for this layer
  int bits = g.bits_table[g.bits_index];
  if (bits < 1 || bits > 8) {
    if (threadIdx.x == 0) atomicOr(g.status, TASQ_DEVICE_BAD_BITS);
    bits = 8;
  }
  const int k_drop = 8 - bits;
  // weights masked ahead of this kernel need no pass here
  const bool masking = k_drop > 0 && g.premasked == 0;
  const uint32_t mask32 = 0x01010101u * ((0xFFu << k_drop) & 0xFFu);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.masked(s), kMaskWarps);
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
  const uint32_t a_base = sbase;
  const uint32_t b_base = sbase + kStages * kABytes;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      uint32_t s = 0, ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      // the activation codes come from the prologue kernel just before this one
      ptx::grid_dep_wait();
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, g.num_m_tiles, g.num_n_tiles, g.band_tiles, mt, nt);
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!ptx::wait_bounded(bars.empty(s), ph ^ 1u, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bars.full(s), P::kStageBytes);
          ptx::tma_load_2d(a_base + s * kABytes, &tmap_w, bars.full(s), kb * kBlockK, nt * kTileCh);
          ptx::tma_load_2d(b_base + s * P::kBBytes, &tmap_x, bars.full(s), kb * kBlockK, mt * kTok);
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
      constexpr uint32_t idesc = ptx::idesc_i8_s32(kTileCh, kTok);
      uint32_t s = 0, ph = 0, as = 0, aph = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!ptx::wait_bounded(bars.acc_empty(as), aph ^ 1u, limit, abort_flag)) {
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
          break;
        }
        ptx::tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + as * kTok;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!ptx::wait_bounded(masking ? bars.masked(s) : bars.full(s), ph, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
          const uint64_t a_desc = ptx::smem_desc_k_sw128(a_base + s * kABytes);
          const uint64_t b_desc = ptx::smem_desc_k_sw128(b_base + s * P::kBBytes);
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
    // Two groups of four warps take alternate K blocks of the CTA's sequence (group 0 the even
    // ones), so that one group's load-mask-store latency overlaps the other's; with a 3-stage ring
    // group 0 takes them all (see mask_groups).
    const int grp = (warp - kMaskWarp0) / kMaskWarps;
    const int t = threadIdx.x - (kMaskWarp0 + grp * kMaskWarps) * 32;
    // stage s of this group's next K block, and its phase
    uint32_t s = grp, ph = 0;
    uint32_t seq = 0;   // K blocks of the CTA's sequence so far
    bool ok = true;
    if (masking) {
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < g.num_kb; ++kb, ++seq) {
          if (static_cast<int>(seq % P::kMaskGroups) != grp) continue;
          if (!ptx::wait_bounded(bars.full(s), ph, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MASK);
            ok = false;
            break;
          }
          mask_stage<kABytes>(smem + s * kABytes, t, mask32);
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(bars.masked(s));
          s += P::kMaskGroups;
          if (s >= static_cast<uint32_t>(kStages)) {
            s -= kStages;
            ph ^= 1u;
          }
        }
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue warps
    epilogue_role<OUT, false, kTok>(g, &tmap_y, tmem_base, smem + P::kEpiOffset + warp * OutTraits<OUT>::kStageBytes,
                                    reinterpret_cast<float*>(smem + P::kSxOffset + warp * kSxBytesPerWarp), warp,
                                    lane, blockIdx.x, gridDim.x, num_tiles, kTileCh, 0, bars.acc_full(0),
                                    bars.acc_empty(0), limit, abort_flag);
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
cudaError_t launch_out(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ty, const GemmArgs& g,
                       int num_sms, cudaStream_t stream) {
  static bool configured[64] = {false};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      e = cudaFuncSetAttribute(masked_gemm_kernel<OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Plan<OUT>::kSmemBytes);
      if (e != cudaSuccess) return e;
      configured[dev] = true;
    }
  }
  const int tiles = g.num_m_tiles * g.num_n_tiles;
  const int grid = tiles < num_sms ? tiles : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads1, 1, 1);
  cfg.dynamicSmemBytes = Plan<OUT>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = use_pdl() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, masked_gemm_kernel<OUT>, tw, tx, ty, g);
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

cudaError_t launch_masked_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const CUtensorMap& tmap_y,
                               const GemmArgs& g, OutKind out, int num_sms, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  switch (out) {
    case OutKind::F16:
      return launch_out<static_cast<int>(OutKind::F16)>(tmap_w, tmap_x, tmap_y, g, num_sms, stream);
    case OutKind::BF16:
      return launch_out<static_cast<int>(OutKind::BF16)>(tmap_w, tmap_x, tmap_y, g, num_sms, stream);
    case OutKind::S32:
      return launch_out<static_cast<int>(OutKind::S32)>(tmap_w, tmap_x, tmap_y, g, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_stuck_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t stream) {
  stuck_wait_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace tasq
