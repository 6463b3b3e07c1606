// Masked INT8 GEMM over CTA pairs (tcgen05 cta_group::2): the same arithmetic as
// masked_gemm.cu (acc = xq . (W & ~(2^k - 1))^T, then y = acc * s_x * s_w), with the work of one
// 256-channel x 256-token tile shared by the two CTAs of a cluster.
//
// Each CTA of the pair holds half of each operand per stage: weight rows
// [256 nt + 128 r, +128) and activation-code rows [256 mt + 128 r, +128) (r = rank in the pair),
// 16 KB + 16 KB. The pair's first CTA issues tcgen05.mma.cta_group::2 with M = 256, N = 256; the
// tensor cores of both SMs read both CTAs' halves, and each CTA's TMEM receives its own 128
// channels x 256 tokens. Per SM and per K stage this moves half the activation bytes of the
// one-CTA tile through shared memory and L2 for the same number of MACs.
//
// Roles per CTA (576 threads), as in the one-CTA kernel but with one group of eight mask warps:
//   warp 8      TMA producer of this CTA's halves, completion on its own `full` barrier.
//   warps 10-17 apply the step's LSB mask to this CTA's weight half in place (when k > 0 and the
//               weights were not masked ahead by the prologue launch) and then arrive on the
//               first CTA's `ready` barrier (one arrival per warp).
//   warp 9      TMEM allocation for the pair (both CTAs); in the first CTA also the MMA thread,
//               which commits stage and accumulator completion to the barriers of both CTAs.
//   warps 0-7   epilogue of this CTA's 128 channels; each warp arrives once on the first CTA's
//               `acc_empty` after reading an accumulator.
// Cross-CTA arrivals are mbarrier arrives on the other CTA's barrier (mapa address). Every wait is bounded; at
// the end the two CTAs meet on a pair barrier (bounded) before TMEM is freed, so that no CTA
// leaves while the other's MMAs may still read its shared memory or write its TMEM.
#include <cstdio>
#include <cstdlib>

#include <mutex>

#include "gemm_common.cuh"

namespace tasq {
namespace {

using namespace gemm;

constexpr int kPairCh = 256;              // output channels per pair tile (MMA M)
constexpr int kPairTok = 256;             // tokens per pair tile (MMA N)
constexpr int kHalf = 128;                // operand rows per CTA
constexpr int kABytes = kHalf * kBlockK;  // 16 KB
constexpr int kBBytes = kHalf * kBlockK;  // 16 KB
constexpr int kStageBytes = kABytes + kBBytes;
static_assert(kPairTok == kAccCols, "accumulator width");
// Eight mask / relay warps (10-17): the in-place pass of a stage, on the path from its landing to
// its MMA, takes half as long as with four (masked CogVideoX GEMMs 4-11 % faster; the one-CTA
// kernel is better served by two alternating groups of four).
constexpr int kPairMaskWarps = 8;
constexpr int kPairThreads = 32 * (kMaskWarp0 + kPairMaskWarps);

template <int OUT>
struct PairPlan {
  static constexpr int kStages = OutTraits<OUT>::kS32 ? 5 : 6;
  static constexpr int kEpiOffset = kStages * kStageBytes;
  static constexpr int kSxOffset = kEpiOffset + kEpiWarps * OutTraits<OUT>::kStageBytes;
  static constexpr int kBarOffset = kSxOffset + kEpiWarps * kSxBytesPerWarp;
  static constexpr int kNumBars = 3 * kStages + 2 * kAccStages + 2;
  static constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOffset + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= kMaxSmem, "shared memory");
};

template <int STAGES>
struct PairBars {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t ready(int s) const { return base + 8u * (STAGES + s); }
  __device__ uint32_t empty(int s) const { return base + 8u * (2 * STAGES + s); }
  __device__ uint32_t acc_full(int i) const { return base + 8u * (3 * STAGES + i); }
  __device__ uint32_t acc_empty(int i) const { return base + 8u * (3 * STAGES + kAccStages + i); }
  __device__ uint32_t drain() const { return base + 8u * (3 * STAGES + 2 * kAccStages); }
  __device__ uint32_t pair_exit() const { return base + 8u * (3 * STAGES + 2 * kAccStages + 1); }
};

template <int OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    masked_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                            const __grid_constant__ CUtensorMap tmap_y, const GemmArgs g) {
  using P = PairPlan<OUT>;
  constexpr int kStages = P::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const PairBars<kStages> bars{sbase + P::kBarOffset};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + P::kBarOffset + P::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the next kernel of the stream may be scheduled; it waits for this one before reading
  ptx::grid_dep_launch_dependents();
  if (gated_out(g.gate, g.bits_table, g.bits_index)) return;   // uniform: both CTAs of a pair leave
  const uint32_t rank = ptx::cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;

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
      ptx::mbar_init(bars.ready(s), 2 * kPairMaskWarps);
      ptx::mbar_init(bars.empty(s), 1);
    }
    for (int i = 0; i < kAccStages; ++i) {
      ptx::mbar_init(bars.acc_full(i), 1);
      ptx::mbar_init(bars.acc_empty(i), 2 * kEpiWarps);
    }
    ptx::mbar_init(bars.drain(), 1);
    ptx::mbar_init(bars.pair_exit(), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_y);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc_pair(ptx::smem_addr(tmem_slot), kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before_sync();
  __syncthreads();
  // both CTAs' barriers are initialised and the pair's TMEM is allocated past this point
  ptx::cluster_sync_all();
  ptx::tc_fence_after_sync();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  const int num_tiles = g.num_m_tiles * g.num_n_tiles;
  const int pair_id = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
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
      for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
        int mt, nt;
        tile_coords(tile, g.num_m_tiles, g.num_n_tiles, g.band_tiles, mt, nt);
        for (int kb = 0; kb < g.num_kb; ++kb) {
          // `empty` is arrived by the first CTA's tensor-core commit
          if (!ptx::wait_bounded(bars.empty(s), ph ^ 1u, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bars.full(s), kStageBytes);
          ptx::tma_load_2d(a_base + s * kABytes, &tmap_w, bars.full(s), kb * kBlockK,
                           nt * kPairCh + static_cast<int>(rank) * kHalf);
          ptx::tma_load_2d(b_base + s * kBBytes, &tmap_x, bars.full(s), kb * kBlockK,
                           mt * kPairTok + static_cast<int>(rank) * kHalf);
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
    if (leader && lane == 0) {
      // ------------------------------------------------------------------ MMA issuer (first CTA)
      constexpr uint32_t idesc = ptx::idesc_i8_s32(kPairCh, kPairTok);
      const uint32_t empty_peer0 = ptx::mapa_shared(bars.empty(0), peer);
      const uint32_t acc_full_peer0 = ptx::mapa_shared(bars.acc_full(0), peer);
      uint32_t s = 0, ph = 0, as = 0, aph = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
        if (!ptx::wait_bounded(bars.acc_empty(as), aph ^ 1u, limit, abort_flag)) {
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
          break;
        }
        ptx::tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + as * kAccCols;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          if (!ptx::wait_bounded(bars.ready(s), ph, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
          const uint64_t a_desc = ptx::smem_desc_k_sw128(a_base + s * kABytes);
          const uint64_t b_desc = ptx::smem_desc_k_sw128(b_base + s * kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBlockK / kUmmaK; ++kk) {
            ptx::mma_i8_ss_pair(d_tmem, a_desc + 2u * kk, b_desc + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          ptx::mma_commit_pair(bars.empty(s));
          ptx::mma_commit_pair(empty_peer0 + 8u * s);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit_pair(bars.acc_full(as));
        ptx::mma_commit_pair(acc_full_peer0 + 8u * as);
        as ^= 1u;
        if (as == 0) aph ^= 1u;
      }
      if (issued_any) {
        ptx::mma_commit_pair(bars.drain());
        if (!ptx::wait_bounded(bars.drain(), 0, limit, nullptr))
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_DRAIN);
      }
    }
  } else if (warp >= kMaskWarp0) {
    // -------------------------------------------------------------------- mask / relay warps
    const int t = threadIdx.x - kMaskWarp0 * 32;
    const uint32_t ready_leader0 = ptx::mapa_shared(bars.ready(0), 0);
    uint32_t s = 0, ph = 0;
    bool ok = true;
    for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
      for (int kb = 0; kb < g.num_kb; ++kb) {
        if (!ptx::wait_bounded(bars.full(s), ph, limit, abort_flag)) {
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MASK);
          ok = false;
          break;
        }
        if (masking) {
          mask_stage<kABytes, 32 * kPairMaskWarps>(smem + s * kABytes, t, mask32);
          ptx::fence_proxy_async_smem();
        }
        // one arrival per warp on the first CTA's barrier (remote arrivals are not free)
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(ready_leader0 + 8u * s);
        if (++s == kStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue warps
    epilogue_role<OUT, true, kPairTok>(g, &tmap_y, tmem_base, smem + P::kEpiOffset + warp * OutTraits<OUT>::kStageBytes,
                             reinterpret_cast<float*>(smem + P::kSxOffset + warp * kSxBytesPerWarp), warp, lane,
                             pair_id, num_pairs, num_tiles, kPairCh, static_cast<int>(rank) * kHalf,
                             bars.acc_full(0), ptx::mapa_shared(bars.acc_empty(0), 0), limit, abort_flag);
  }

  __syncwarp();
  ptx::tc_fence_before_sync();
  __syncthreads();
  // pair barrier: the first CTA arrives after its MMAs drained, the second after all its remote
  // arrivals; neither frees TMEM or exits before the other is done with it
  if (threadIdx.x == 0) {
    ptx::mbar_arrive_cluster(ptx::mapa_shared(bars.pair_exit(), peer));
    if (!ptx::wait_bounded(bars.pair_exit(), 0, limit, nullptr))
      raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_DRAIN);
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int OUT>
cudaError_t launch_pair_out(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ty, const GemmArgs& g,
                            int num_sms, cudaStream_t stream) {
  static bool configured[64] = {false};
  static int max_pairs[64] = {0};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int resident_pairs = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      e = cudaFuncSetAttribute(masked_gemm_pair_kernel<OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PairPlan<OUT>::kSmemBytes);
      if (e != cudaSuccess) return e;
      // how many CTA pairs can be resident at once on this device
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
      cfg.blockDim = dim3(kPairThreads, 1, 1);
      cfg.dynamicSmemBytes = PairPlan<OUT>::kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      e = cudaOccupancyMaxActiveClusters(&clusters, masked_gemm_pair_kernel<OUT>, &cfg);
      if (e != cudaSuccess || clusters <= 0) {
        (void)cudaGetLastError();
        clusters = num_sms / 2;
      }
      max_pairs[dev] = clusters;
      configured[dev] = true;
      if (std::getenv("TASQ_VERBOSE") != nullptr)
        std::fprintf(stderr, "tasq: pair GEMM on device %d: %d resident CTA pairs, %d bytes of shared memory\n", dev,
                     clusters, PairPlan<OUT>::kSmemBytes);
    }
    resident_pairs = max_pairs[dev];
  }
  const int tiles = g.num_m_tiles * g.num_n_tiles;
  const int pairs = tiles < resident_pairs ? tiles : resident_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = PairPlan<OUT>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = use_pdl() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, masked_gemm_pair_kernel<OUT>, tw, tx, ty, g);
}

}  // namespace

cudaError_t launch_masked_gemm_pair(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const CUtensorMap& tmap_y,
                                    const GemmArgs& g, OutKind out, int num_sms, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  switch (out) {
    case OutKind::F16:
      return launch_pair_out<static_cast<int>(OutKind::F16)>(tmap_w, tmap_x, tmap_y, g, num_sms, stream);
    case OutKind::BF16:
      return launch_pair_out<static_cast<int>(OutKind::BF16)>(tmap_w, tmap_x, tmap_y, g, num_sms, stream);
    case OutKind::S32:
      return launch_pair_out<static_cast<int>(OutKind::S32)>(tmap_w, tmap_x, tmap_y, g, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tasq
