// Block-scaled NVFP4 GEMM over CTA pairs (tcgen05 cta_group::2): the arithmetic of
// gemm_nvfp4.cu (6Bit-Diffusion technical summary, section 2.A: stable layers in NVFP4, beside
// the INT8 path),
//
//   acc[m, c] = sum over 16-blocks b of  sx4[m, b] * sw4[c, b] * sum_{k in b} ex[m, k] * ew[c, k]
//   y[m, c]   = acc[m, c] * s_x[m] * s_w[c]         (or the raw FP32 acc for the test hook)
//
// with the work of one 256-channel x 192-token tile shared by the two CTAs of a cluster.
//
// Where the time of a block-scaled GEMM goes on sm_100a. Besides its MMAs, every MMA of K = 64
// needs the UE4M3 scales of its rows in TMEM, moved there from shared memory by tcgen05.cp: one
// 512-byte copy per 128 rows of A and per 128 rows of B. Those copies run in the tensor pipe
// beside the MMAs (~45 cycles each, measured), so at 128 x 128 tiles they take about as long as
// the MMAs themselves. This kernel cuts their share three ways:
//   * CTA pairs with M = 256: one tcgen05.cp.cta_group::2 fills both CTAs' TMEM, so the weight
//     scales cost one copy per 256 rows;
//   * N = 192 tokens per MMA: the token scales (two copies per MMA for 192 rows) serve 1.5x the
//     MACs of a 128-token MMA, and wider MMAs run closer to the tensor core's rate (measured:
//     with the copies left out, 192-token tiles ran 1.37x faster than 128-token ones);
//   * the copies are issued by a second thread into two alternating TMEM scale buffers, so the
//     copies of stage s + 1 can overlap the MMAs of stage s (measured: 10 % faster than copies
//     issued in line by the MMA thread).
//
// Per stage (256 elements of K) each CTA holds weight rows [256 nt + 128 r, +128) and token rows
// [192 mt + 96 r, +96) (r = rank in the pair): 16 KB + 12 KB of codes (128-byte swizzle), its
// own 2 KB of weight scales and the 4 KB of scales of the tile's 192 token rows (two 128-row
// groups of the chunked layout). Tiles start every 192 tokens, so an odd tile begins 64 rows
// into a 128-row scale group: for such tiles the relay warp rearranges the landed token scales
// in shared memory (8-byte moves inside each lane's 16-byte row) so that tile row t sits in TMEM
// column t / 32, as the MMA reads it.
//
// Roles per CTA (384 threads):
//   warp 8      producer: two TMA tile loads (codes) and three bulk copies (scales) per stage into
//               this CTA's ring, completion on its own `full` barrier.
//   warp 10     relay: once a stage of this CTA has landed (and, for odd tiles, its token scales
//               are rearranged), one arrival on the first CTA's `ready` barrier.
//   warp 11     in the first CTA, the copy thread: after `ready` it copies the stage's scales into
//               the free TMEM scale buffer of both CTAs and commits to `sf_full`.
//   warp 9      TMEM allocation for the pair (both CTAs); in the first CTA also the MMA thread:
//               per stage it waits for `sf_full`, issues four block-scaled MMAs and commits to
//               the stage's `empty` barriers in both CTAs and to the scale buffer's `sf_free`.
//   warps 0-7   epilogue of this CTA's 128 channels (the INT8 kernels' epilogue on FP32
//               accumulators); each warp arrives once on the first CTA's `acc_empty` after reading
//               an accumulator.
// TMEM (512 columns per CTA): two 192-column FP32 accumulators, then two scale buffers of 48
// columns (16 for the weight scales of four MMAs, 32 for the token scales: 8 per MMA).
// Every wait is bounded; at the end the two CTAs meet on a pair barrier (bounded) before TMEM is
// freed, so that no CTA leaves while the other's MMAs may still read its shared memory or write
// its TMEM.
#include <mutex>

#include "gemm_common.cuh"

namespace tasq {
namespace {

using namespace gemm;

constexpr int kPairCh = 256;                      // output channels per pair tile (MMA M)
constexpr int kPairTok = kGemmNvfp4PairTok;       // tokens per pair tile (MMA N)
constexpr int kHalfCh = 128;                      // weight rows per CTA
constexpr int kHalfTok = kPairTok / 2;            // token rows per CTA
constexpr int kCodeBytes = 128;                   // bytes of codes per row and stage (256 elements)
constexpr int kABytes = kHalfCh * kCodeBytes;     // 16 KB
constexpr int kBBytes = kHalfTok * kCodeBytes;    // 12 KB
constexpr int kSfaBytes = 4 * kNvfp4ChunkBytes;   // weight scales: four K = 64 chunks of 128 rows
constexpr int kSfbGroupBytes = 4 * kNvfp4ChunkBytes;
constexpr int kSfbBytes = 2 * kSfbGroupBytes;     // token scales: two 128-row groups x four chunks
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr int kRelayWarp = 10;
constexpr int kCopyWarp = 11;
constexpr int kThreadsP4 = 32 * (kCopyWarp + 1);
constexpr uint32_t kAccColsP4 = kPairTok;         // one accumulator: 192 FP32 columns
constexpr uint32_t kSfCol = 2 * kAccColsP4;       // first TMEM scale buffer
constexpr uint32_t kSfBufCols = 16 + 32;          // weight scales (4 x 4), token scales (4 x 8)
static_assert(kPairTok == 192, "token-scale groups: a tile spans one 128-row group and half of the next");
static_assert(kEpiWarps == 8 && kProducerWarp == 8 && kMmaWarp == 9, "warp roles");
static_assert(kStageBytes % 1024 == 0 && (kABytes + kBBytes) % 1024 == 0 && kABytes % 1024 == 0,
              "swizzled tiles keep their 1024-byte alignment");
static_assert(kSfCol + 2 * kSfBufCols <= kTmemCols, "TMEM");

template <int OUT>
struct PairPlanF4 {
  static constexpr int kStages = OutTraits<OUT>::kS32 ? 5 : 6;
  static constexpr int kEpiOffset = kStages * kStageBytes;
  static constexpr int kSxOffset = kEpiOffset + kEpiWarps * OutTraits<OUT>::kStageBytes;
  static constexpr int kBarOffset = kSxOffset + kEpiWarps * kSxBytesPerWarp;
  static constexpr int kNumBars = 3 * kStages + 2 * kAccStages + 2 + 4 + 1;
  static constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOffset + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= kMaxSmem, "shared memory");
};

template <int STAGES>
struct PairBarsF4 {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t ready(int s) const { return base + 8u * (STAGES + s); }
  __device__ uint32_t empty(int s) const { return base + 8u * (2 * STAGES + s); }
  __device__ uint32_t acc_full(int i) const { return base + 8u * (3 * STAGES + i); }
  __device__ uint32_t acc_empty(int i) const { return base + 8u * (3 * STAGES + kAccStages + i); }
  __device__ uint32_t drain() const { return base + 8u * (3 * STAGES + 2 * kAccStages); }
  __device__ uint32_t pair_exit() const { return base + 8u * (3 * STAGES + 2 * kAccStages + 1); }
  __device__ uint32_t sf_full(int b) const { return base + 8u * (3 * STAGES + 2 * kAccStages + 2 + b); }
  __device__ uint32_t sf_free(int b) const { return base + 8u * (3 * STAGES + 2 * kAccStages + 4 + b); }
  __device__ uint32_t copy_drain() const { return base + 8u * (3 * STAGES + 2 * kAccStages + 6); }
};

// Tile mt covers token rows [192 mt, 192 mt + 192): 128-row scale groups g0 = floor(1.5 mt) and
// g0 + 1; for odd mt the tile starts at row 64 of g0.
__device__ __forceinline__ int token_group0(int mt) { return (3 * mt) >> 1; }

// Odd tile: in each K = 64 chunk, lane l's 16-byte row holds the scales of rows l, l + 32,
// l + 64, l + 96 of its group (4 bytes each). The tile's rows 0..63 are rows 64..127 of group g0
// (bytes 8..15 of the first chunk), rows 64..191 all of group g0 + 1. Rewrite the two chunks so
// that the first holds tile rows l, l + 32, l + 64, l + 96 and the second tile rows l + 128,
// l + 160 (the rest of the second chunk is never read by an N = 192 MMA).
__device__ __forceinline__ void shift_token_scales(uint8_t* sfb, int lane) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint2* first = reinterpret_cast<uint2*>(sfb + c * kNvfp4ChunkBytes + lane * 16);
    uint2* second = reinterpret_cast<uint2*>(sfb + kSfbGroupBytes + c * kNvfp4ChunkBytes + lane * 16);
    const uint2 a_hi = first[1];
    const uint2 b_lo = second[0];
    const uint2 b_hi = second[1];
    first[0] = a_hi;
    first[1] = b_lo;
    second[0] = b_hi;
  }
}

template <int OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsP4, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                           const __grid_constant__ CUtensorMap tmap_y, const GemmArgs g, const Nvfp4GemmArgs f) {
  using P = PairPlanF4<OUT>;
  constexpr int kStages = P::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_addr(smem);
  const PairBarsF4<kStages> bars{sbase + P::kBarOffset};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + P::kBarOffset + P::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the next kernel of the stream may be scheduled; it waits for this one before reading
  ptx::grid_dep_launch_dependents();
  // uniform over the grid: both CTAs of a pair leave
  if (g.bits_table != nullptr && gated_out(g.gate, g.bits_table, g.bits_index)) return;
  const uint32_t rank = ptx::cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;

  // the schedule entry of an NVFP4 step is 0
  if (threadIdx.x == 0 && g.bits_table != nullptr && g.bits_table[g.bits_index] != 0)
    atomicOr(g.status, TASQ_DEVICE_BAD_BITS);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.ready(s), 2);
      ptx::mbar_init(bars.empty(s), 1);
    }
    for (int i = 0; i < kAccStages; ++i) {
      ptx::mbar_init(bars.acc_full(i), 1);
      ptx::mbar_init(bars.acc_empty(i), 2 * kEpiWarps);
    }
    ptx::mbar_init(bars.drain(), 1);
    ptx::mbar_init(bars.pair_exit(), 1);
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bars.sf_full(b), 1);
      ptx::mbar_init(bars.sf_free(b), 1);
    }
    ptx::mbar_init(bars.copy_drain(), 1);
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
  const int token_groups = (g.M + 127) / 128;   // 128-row groups of the token-scale layout
  // stage s: weight codes, token codes, weight scales, token scales (two groups)
  auto a_smem = [&](int s) { return sbase + static_cast<uint32_t>(s * kStageBytes); };
  auto b_smem = [&](int s) { return a_smem(s) + kABytes; };
  auto sfa_smem = [&](int s) { return b_smem(s) + kBBytes; };
  auto sfb_smem = [&](int s) { return sfa_smem(s) + kSfaBytes; };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------------ producer
      uint32_t s = 0, ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      // the codes and scales come from the prologue kernel just before this one
      ptx::grid_dep_wait();
      for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
        int mt, nt;
        tile_coords(tile, g.num_m_tiles, g.num_n_tiles, g.band_tiles, mt, nt);
        // this CTA's 128 weight rows; a group wholly past N has no scales to load (its rows are
        // zero-filled by the tensor map and its outputs are never stored), and likewise a token
        // group past the last token
        const int w_group = nt * (kPairCh / 128) + static_cast<int>(rank);
        const bool w_rows = w_group * 128 < g.N;
        const int t_group = token_group0(mt);
        const bool t_next = t_group + 1 < token_groups;
        const uint8_t* sfa_src = f.w_sf + (static_cast<int64_t>(w_group) * f.sf_chunks) * kNvfp4ChunkBytes;
        const uint8_t* sfb_src = f.x_sf + (static_cast<int64_t>(t_group) * f.sf_chunks) * kNvfp4ChunkBytes;
        const uint8_t* sfb_src1 = sfb_src + static_cast<int64_t>(f.sf_chunks) * kNvfp4ChunkBytes;
        const uint32_t stage_tx = static_cast<uint32_t>(kABytes + kBBytes + kSfbGroupBytes +
                                                        (t_next ? kSfbGroupBytes : 0) + (w_rows ? kSfaBytes : 0));
        for (int kb = 0; kb < g.num_kb; ++kb) {
          // `empty` is arrived by the first CTA's tensor-core commit
          if (!ptx::wait_bounded(bars.empty(s), ph ^ 1u, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_PRODUCER);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bars.full(s), stage_tx);
          ptx::tma_load_2d(a_smem(s), &tmap_w, bars.full(s), kb * kCodeBytes, w_group * 128);
          ptx::tma_load_2d(b_smem(s), &tmap_x, bars.full(s), kb * kCodeBytes,
                           mt * kPairTok + static_cast<int>(rank) * kHalfTok);
          if (w_rows) ptx::bulk_load(sfa_smem(s), sfa_src + kb * kSfaBytes, kSfaBytes, bars.full(s));
          ptx::bulk_load(sfb_smem(s), sfb_src + kb * kSfbGroupBytes, kSfbGroupBytes, bars.full(s));
          if (t_next)
            ptx::bulk_load(sfb_smem(s) + kSfbGroupBytes, sfb_src1 + kb * kSfbGroupBytes, kSfbGroupBytes, bars.full(s));
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // every copy this thread issued must have landed before the CTA may exit
      for (int i = 0; i < kStages; ++i) {
        if ((issued >> i) & 1u) {
          if (!ptx::wait_bounded(bars.full(i), (issued_par >> i) & 1u, limit, nullptr))
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (leader && lane == 0) {
      // ------------------------------------------------------------------ MMA thread (first CTA)
      constexpr uint32_t idesc = ptx::idesc_nvfp4(kPairCh, kPairTok);
      const uint32_t empty_peer0 = ptx::mapa_shared(bars.empty(0), peer);
      const uint32_t acc_full_peer0 = ptx::mapa_shared(bars.acc_full(0), peer);
      uint32_t s = 0, as = 0, aph = 0, sb = 0, sbph = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
        if (!ptx::wait_bounded(bars.acc_empty(as), aph ^ 1u, limit, abort_flag)) {
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
          break;
        }
        ptx::tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + as * kAccColsP4;
        for (int kb = 0; kb < g.num_kb; ++kb) {
          // the stage's codes have landed in both CTAs and its scales are in TMEM buffer sb
          if (!ptx::wait_bounded(bars.sf_full(sb), sbph, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MMA);
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
          const uint32_t sfa_t = tmem_base + kSfCol + kSfBufCols * sb;
          const uint32_t sfb_t = sfa_t + 16u;
          const uint64_t a_desc = ptx::smem_desc_k_sw128(a_smem(s));
          const uint64_t b_desc = ptx::smem_desc_k_sw128(b_smem(s));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // +32 bytes (64 elements) along K inside the 128-byte swizzle row = +2 in the address field
            ptx::mma_nvfp4_ss_pair(d_tmem, a_desc + 2u * kk, b_desc + 2u * kk, idesc, sfa_t + 4u * kk,
                                   sfb_t + 8u * kk, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          ptx::mma_commit_pair(bars.empty(s));
          ptx::mma_commit_pair(empty_peer0 + 8u * s);
          ptx::mma_commit_pair(bars.sf_free(sb));
          sb ^= 1u;
          if (sb == 0) sbph ^= 1u;
          if (++s == kStages) s = 0;
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
  } else if (warp == kRelayWarp) {
    // -------------------------------------------------------------------- relay
    const uint32_t ready_leader0 = ptx::mapa_shared(bars.ready(0), 0);
    uint32_t s = 0, ph = 0;
    bool ok = true;
    for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
      int mt, nt;
      tile_coords(tile, g.num_m_tiles, g.num_n_tiles, g.band_tiles, mt, nt);
      const bool odd = mt & 1;
      for (int kb = 0; kb < g.num_kb; ++kb) {
        const bool got = ptx::wait_bounded(bars.full(s), ph, limit, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MASK);
          ok = false;
          break;
        }
        if (odd) {
          shift_token_scales(smem + (sfb_smem(s) - sbase), lane);
          // generic-proxy writes before the tensor core's copy reads them
          ptx::fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(ready_leader0 + 8u * s);
        if (++s == kStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp == kCopyWarp) {
    if (leader && lane == 0) {
      // ------------------------------------------------------------------ copy thread (first CTA)
      uint32_t s = 0, ph = 0, cb = 0, cbph = 0;
      bool ok = true;
      bool copied = false;
      for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
        for (int kb = 0; kb < g.num_kb; ++kb) {
          // both CTAs' stages are ready and TMEM scale buffer cb is free
          if (!ptx::wait_bounded(bars.ready(s), ph, limit, abort_flag) ||
              !ptx::wait_bounded(bars.sf_free(cb), cbph ^ 1u, limit, abort_flag)) {
            raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_MASK);
            ok = false;
            break;
          }
          ptx::tc_fence_after_sync();
          const uint32_t sfa_t = tmem_base + kSfCol + kSfBufCols * cb;
          const uint32_t sfb_t = sfa_t + 16u;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            ptx::tmem_cp_32x128b_warpx4_pair(sfa_t + 4u * c, ptx::smem_desc_rows16(sfa_smem(s) + c * kNvfp4ChunkBytes));
            ptx::tmem_cp_32x128b_warpx4_pair(sfb_t + 8u * c, ptx::smem_desc_rows16(sfb_smem(s) + c * kNvfp4ChunkBytes));
            ptx::tmem_cp_32x128b_warpx4_pair(sfb_t + 8u * c + 4u,
                                             ptx::smem_desc_rows16(sfb_smem(s) + kSfbGroupBytes + c * kNvfp4ChunkBytes));
          }
          ptx::mma_commit_pair(bars.sf_full(cb));
          copied = true;
          cb ^= 1u;
          if (cb == 0) cbph ^= 1u;
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // the copies this thread issued must have completed before TMEM is freed
      if (copied) {
        ptx::mma_commit_pair(bars.copy_drain());
        if (!ptx::wait_bounded(bars.copy_drain(), 0, limit, nullptr))
          raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_DRAIN);
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue warps
    epilogue_role<OUT, true, kPairTok, true>(g, &tmap_y, tmem_base,
                                             smem + P::kEpiOffset + warp * OutTraits<OUT>::kStageBytes,
                                             reinterpret_cast<float*>(smem + P::kSxOffset + warp * kSxBytesPerWarp),
                                             warp, lane, pair_id, num_pairs, num_tiles, kPairCh,
                                             static_cast<int>(rank) * kHalfCh, bars.acc_full(0),
                                             ptx::mapa_shared(bars.acc_empty(0), 0), limit, abort_flag);
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
cudaError_t launch_pair_f4(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ty, const GemmArgs& g,
                           const Nvfp4GemmArgs& f, int num_sms, cudaStream_t stream) {
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
      e = cudaFuncSetAttribute(gemm_nvfp4_pair_kernel<OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PairPlanF4<OUT>::kSmemBytes);
      if (e != cudaSuccess) return e;
      // how many CTA pairs can be resident at once on this device
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
      cfg.blockDim = dim3(kThreadsP4, 1, 1);
      cfg.dynamicSmemBytes = PairPlanF4<OUT>::kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      e = cudaOccupancyMaxActiveClusters(&clusters, gemm_nvfp4_pair_kernel<OUT>, &cfg);
      if (e != cudaSuccess || clusters <= 0) {
        (void)cudaGetLastError();
        clusters = num_sms / 2;
      }
      max_pairs[dev] = clusters;
      configured[dev] = true;
    }
    resident_pairs = max_pairs[dev];
  }
  const int tiles = g.num_m_tiles * g.num_n_tiles;
  const int pairs = tiles < resident_pairs ? tiles : resident_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kThreadsP4, 1, 1);
  cfg.dynamicSmemBytes = PairPlanF4<OUT>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = use_pdl() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_nvfp4_pair_kernel<OUT>, tw, tx, ty, g, f);
}

}  // namespace

cudaError_t launch_gemm_nvfp4_pair(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const CUtensorMap& tmap_y,
                                   const GemmArgs& g, const Nvfp4GemmArgs& f, OutKind out, int num_sms,
                                   cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (reinterpret_cast<uintptr_t>(f.w_sf) % 16 != 0 || reinterpret_cast<uintptr_t>(f.x_sf) % 16 != 0 ||
      f.sf_chunks != g.num_kb * 4 || g.num_m_tiles != (g.M + kPairTok - 1) / kPairTok ||
      g.num_n_tiles != (g.N + kPairCh - 1) / kPairCh)
    return cudaErrorInvalidValue;
  switch (out) {
    case OutKind::F16:
      return launch_pair_f4<static_cast<int>(OutKind::F16)>(tmap_w, tmap_x, tmap_y, g, f, num_sms, stream);
    case OutKind::BF16:
      return launch_pair_f4<static_cast<int>(OutKind::BF16)>(tmap_w, tmap_x, tmap_y, g, f, num_sms, stream);
    case OutKind::S32:
      return launch_pair_f4<static_cast<int>(OutKind::S32)>(tmap_w, tmap_x, tmap_y, g, f, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tasq
