// Pieces shared by the two masked INT8 GEMM kernels (one CTA per tile, and CTA pairs): warp
// roles, shared-memory plan of the epilogue, and the epilogue role itself.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../../include/tasq.h"
#include "ptx.cuh"
#include "tasq_internal.h"

namespace tasq {
namespace gemm {

constexpr int kBlockK = kGemmBlockK;          // 128 bytes of K per pipeline stage
constexpr int kUmmaK = 32;                    // K of one tcgen05.mma.kind::i8
constexpr int kAccCols = 256;                 // widest tile: tokens = INT32 TMEM columns per accumulator
constexpr int kAccStages = 2;
constexpr uint32_t kTmemCols = 512;           // the whole TMEM of the SM
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kMaskWarp0 = 10;
constexpr int kMaskWarps = 4;
constexpr int kThreads = 32 * (kEpiWarps + 2 + kMaskWarps);
constexpr int kMaskThreads = 32 * kMaskWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kSxBytesPerWarp = (kAccCols / 2) * 4;      // token scales of one epilogue warp
constexpr int kMaxSmem = 232448;

template <int OUT>
struct OutTraits {
  static constexpr bool kS32 = OUT == static_cast<int>(OutKind::S32);
  static constexpr int kBytes = kS32 ? 4 : 2;
  static constexpr int kStageBytes = 32 * 32 * kBytes;   // one 32 x 32 output box per epilogue warp
};

// Order of a launch's tiles: bands of `band` token tiles (GemmArgs::band_tiles); inside a band the
// token tile varies fastest, then the channel tile. The CTAs of one wave then work on a few token
// tiles and a few channel tiles, and a band's codes stay in L2 while its channel tiles go by. With
// the token tile varying fastest over all of M, every wave took all token tiles of one channel
// tile, and once the codes outgrew L2 (CogVideoX fc2: 218 MB) they came from DRAM again for every
// channel tile (2.5 GB read by one launch for 256 MB of operands). Every role of a kernel maps tile
// indices the same way.
__device__ __forceinline__ void tile_coords(int tile, int num_m_tiles, int num_n_tiles, int band, int& mt, int& nt) {
  const int band_tiles = band * num_n_tiles;
  const int b = tile / band_tiles;
  const int within = tile - b * band_tiles;
  const int m0 = b * band;
  const int gm = num_m_tiles - m0 < band ? num_m_tiles - m0 : band;
  mt = m0 + within % gm;
  nt = within / gm;
}

__device__ __forceinline__ void raise_failure(uint32_t* status, volatile int* abort_flag, uint32_t bit) {
  atomicOr(status, bit);
  *abort_flag = 1;
}

// Packed FP32x2 product, each lane rounded once to nearest even.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  const uint64_t ua = *reinterpret_cast<const uint64_t*>(&a);
  const uint64_t ub = *reinterpret_cast<const uint64_t*>(&b);
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ua), "l"(ub));
  return *reinterpret_cast<const float2*>(&r);
}

// Two adjacent tokens of one channel: y = (acc * s_x) * s_w in FP32, then a packed FP16 / BF16
// pair (first token in the low half). The accumulators are INT32 (the INT8 GEMM) or FP32 (the
// block-scaled NVFP4 GEMM, ACC_F32).
template <int OUT, bool ACC_F32 = false>
__device__ __forceinline__ uint32_t out_pair(uint32_t a0, uint32_t a1, float2 sx, float sw) {
  const float2 acc = ACC_F32 ? make_float2(__uint_as_float(a0), __uint_as_float(a1))
                             : make_float2(static_cast<float>(static_cast<int32_t>(a0)),
                                           static_cast<float>(static_cast<int32_t>(a1)));
  const float2 v = mul2(mul2(acc, sx), make_float2(sw, sw));
  if constexpr (OUT == static_cast<int>(OutKind::F16)) {
    const __half2 h = __floats2half2_rn(v.x, v.y);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

// Epilogue role of warps 0..7 for tiles of TOK tokens (256 or 192). Warp w owns TMEM lanes
// 32 (w % 4) .. +31 (32 output channels) and accumulator columns TOK/2 (w / 4) .. +TOK/2 - 1,
// taken in chunks of 32 columns; accumulator i starts at TMEM column i * TOK. Each chunk
// is scaled, converted and written into the warp's private 32 x 32 staging box in output row
// order, then stored with one TMA bulk store. Warps never wait on each other.
//   FP16 / BF16: two 16 x 256-bit TMEM loads give each lane two adjacent tokens of four channels;
//   the packed pairs are exactly 8 x 8 matrix fragments (row = channel, column = token), which
//   stmatrix.trans writes token-major into the box, 16 bytes per row, through a 64-byte swizzle
//   (chunk ^= (row >> 1) & 3) that keeps the eight rows of each matrix on distinct banks; the TMA
//   store undoes the swizzle.
//   INT32 (test hook): 32 x 32-bit TMEM loads, one value per lane per store, no swizzle; the raw
//   accumulator words (FP32 bits when ACC_F32).
//   ACC_F32: the accumulators are FP32 (the NVFP4 GEMM) instead of INT32.
//   ch_per_tile / ch_offset : output channels of tile nt start at nt * ch_per_tile + ch_offset.
//   acc_full + 8 i          : local barrier the MMA side arrives on when accumulator i is ready.
//   acc_empty + 8 i         : barrier (local, or in another CTA of the cluster when CLUSTER) that
//                             each epilogue warp arrives on once, after reading accumulator i.
template <int OUT, bool CLUSTER, int TOK, bool ACC_F32 = false>
__device__ __forceinline__ void epilogue_role(const GemmArgs& g, const CUtensorMap* tmap_y, uint32_t tmem_base,
                                              uint8_t* stage, float* sx_slice, int warp, int lane, int tile0,
                                              int tile_step, int num_tiles, int ch_per_tile, int ch_offset,
                                              uint32_t acc_full, uint32_t acc_empty, uint64_t limit,
                                              volatile int* abort_flag) {
  using O = OutTraits<OUT>;
  constexpr int kEpiCols = TOK / 2;   // tokens of one epilogue warp per tile
  static_assert(TOK % 64 == 0 && TOK <= kAccCols, "tile width");
  const int q = warp & 3;         // TMEM lanes 32 q .. 32 q + 31
  const int h = warp >> 2;        // accumulator columns kEpiCols h .. kEpiCols (h + 1) - 1
  const uint32_t stage_addr = ptx::smem_addr(stage);
  uint32_t as = 0, aph = 0;
  bool store_pending = false;
  // the token scales come from the prologue kernel just before this one
  ptx::grid_dep_wait();
  for (int tile = tile0; tile < num_tiles; tile += tile_step) {
    int mt, nt;
    tile_coords(tile, g.num_m_tiles, g.num_n_tiles, g.band_tiles, mt, nt);
    const int tok0 = mt * TOK + h * kEpiCols;
    const bool got = ptx::wait_bounded(acc_full + 8u * as, aph, limit, abort_flag);
    if (!__all_sync(0xffffffffu, got)) {
      if (lane == 0) raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_EPILOGUE);
      break;
    }
    ptx::tc_fence_after_sync();
    const int c0 = nt * ch_per_tile + ch_offset + q * 32;   // first channel of this warp
    const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + as * TOK + h * kEpiCols;
    if constexpr (O::kS32) {
      const int ch = c0 + lane;
#pragma unroll 1
      for (int j = 0; j < kEpiCols / 32; ++j) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(tacc + j * 32, r);
        ptx::tmem_ld_wait(r);
        if (j == kEpiCols / 32 - 1) {
          ptx::tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            if constexpr (CLUSTER) ptx::mbar_arrive_cluster(acc_empty + 8u * as);
            else ptx::mbar_arrive(acc_empty + 8u * as);
          }
        }
        const int t0 = tok0 + j * 32;
        if (t0 >= g.M || c0 >= g.N) continue;
        if (c0 + 32 > g.N && (g.N * O::kBytes) % 16 != 0) {
          // a TMA store writes whole 16-byte granules, so a box whose right edge is not 16-byte
          // aligned would write past column N: store this one with plain predicated stores
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            if (ch < g.N && t0 + t < g.M)
              static_cast<int32_t*>(g.y)[static_cast<int64_t>(t0 + t) * g.ldy + ch] = static_cast<int32_t>(r[t]);
          }
          continue;
        }
        if (store_pending) {
          if (lane == 0) ptx::bulk_wait_read0();
          __syncwarp();
        }
        uint32_t* st = reinterpret_cast<uint32_t*>(stage);
#pragma unroll
        for (int t = 0; t < 32; ++t) st[t * 32 + lane] = r[t];
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::tma_store_2d(tmap_y, stage_addr, c0, t0);
          ptx::bulk_commit();
        }
        store_pending = true;
      }
    } else {
      // this lane's four channels: c0 + 16 g + 8 o + lane / 4 for lane half g and octet o
      float sw[2][2];
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
#pragma unroll
        for (int o = 0; o < 2; ++o) {
          const int ch = c0 + 16 * gg + 8 * o + (lane >> 2);
          sw[gg][o] = ch < g.N ? g.s_w[ch] : 0.0f;
        }
      }
      // this warp's token scales, read once per tile into its private slice
      if (4 * lane < kEpiCols) {
        float4 v4;
        const int m = tok0 + 4 * lane;
        v4.x = m < g.M ? g.s_x[m] : 0.0f;
        v4.y = m + 1 < g.M ? g.s_x[m + 1] : 0.0f;
        v4.z = m + 2 < g.M ? g.s_x[m + 2] : 0.0f;
        v4.w = m + 3 < g.M ? g.s_x[m + 3] : 0.0f;
        reinterpret_cast<float4*>(sx_slice)[lane] = v4;
      }
      __syncwarp();
#pragma unroll 1
      for (int j = 0; j < kEpiCols / 32; ++j) {
        uint32_t ra[16], rb[16];   // lanes 32 q + 0 .. 15 and 32 q + 16 .. 31
        ptx::tmem_ld_16x256b_x4(tacc + j * 32, ra);
        ptx::tmem_ld_16x256b_x4(tacc + (16u << 16) + j * 32, rb);
        ptx::tmem_ld_wait(ra, rb);
        if (j == kEpiCols / 32 - 1) {
          // the accumulator has been read: hand it back to the MMA before storing (one arrival
          // per warp, after every lane's TMEM reads are ordered before the warp barrier)
          ptx::tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            if constexpr (CLUSTER) ptx::mbar_arrive_cluster(acc_empty + 8u * as);
            else ptx::mbar_arrive(acc_empty + 8u * as);
          }
        }
        const int t0 = tok0 + j * 32;
        // boxes wholly past the last token or channel have nothing to store (warp-uniform)
        if (t0 >= g.M || c0 >= g.N) continue;
        const float* sxc = sx_slice + j * 32;
        if (c0 + 32 > g.N && (g.N * O::kBytes) % 16 != 0) {
          // ragged last box whose edge is not 16-byte aligned: plain predicated stores
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const uint32_t* rr = gg == 0 ? ra : rb;
#pragma unroll
            for (int o = 0; o < 2; ++o) {
              const int ch = c0 + 16 * gg + 8 * o + (lane >> 2);
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const int tl = 8 * r + 2 * (lane & 3);
                const uint32_t pr = out_pair<OUT, ACC_F32>(rr[4 * r + 2 * o], rr[4 * r + 2 * o + 1],
                                                  make_float2(sxc[tl], sxc[tl + 1]), sw[gg][o]);
                if (ch < g.N) {
                  uint16_t* y = static_cast<uint16_t*>(g.y);
                  if (t0 + tl < g.M) y[static_cast<int64_t>(t0 + tl) * g.ldy + ch] = static_cast<uint16_t>(pr & 0xFFFFu);
                  if (t0 + tl + 1 < g.M) y[static_cast<int64_t>(t0 + tl + 1) * g.ldy + ch] = static_cast<uint16_t>(pr >> 16);
                }
              }
            }
          }
          continue;
        }
        if (store_pending) {
          // the previous bulk store of this warp must have finished reading the staging box
          if (lane == 0) ptx::bulk_wait_read0();
          __syncwarp();
        }
        float2 sx2[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) sx2[r] = *reinterpret_cast<const float2*>(sxc + 8 * r + 2 * (lane & 3));
        // row `lane` of the box is token t0 + lane; its 16-byte chunk c holds channels 8c .. 8c + 7
        const uint32_t row_addr = stage_addr + 64u * lane;
        const uint32_t swz = (static_cast<uint32_t>(lane) >> 1) & 3u;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const uint32_t* rr = gg == 0 ? ra : rb;
#pragma unroll
          for (int o = 0; o < 2; ++o) {
            uint32_t p[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) p[r] = out_pair<OUT, ACC_F32>(rr[4 * r + 2 * o], rr[4 * r + 2 * o + 1], sx2[r], sw[gg][o]);
            const uint32_t chunk = static_cast<uint32_t>(2 * gg + o);
            ptx::stmatrix_x4_trans(row_addr + 16u * (chunk ^ swz), p[0], p[1], p[2], p[3]);
          }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::tma_store_2d(tmap_y, stage_addr, c0, t0);
          ptx::bulk_commit();
        }
        store_pending = true;
      }
    }
    as ^= 1u;
    if (as == 0) aph ^= 1u;
  }
  if (lane == 0) ptx::bulk_wait0();
}

// In-place LSB mask of one landed weight stage by THREADS threads (thread t of them): every byte
// AND (0xFF << k), 16 bytes at a time.
template <int A_BYTES, int THREADS = kMaskThreads>
__device__ __forceinline__ void mask_stage(uint8_t* a_stage, int t, uint32_t mask32) {
  static_assert(A_BYTES % (16 * THREADS) == 0, "mask pass must tile the weight stage");
  uint4* wt = reinterpret_cast<uint4*>(a_stage);
#pragma unroll
  for (int i = 0; i < A_BYTES / 16 / THREADS; ++i) {
    uint4 w = wt[i * THREADS + t];
    w.x &= mask32;
    w.y &= mask32;
    w.z &= mask32;
    w.w &= mask32;
    wt[i * THREADS + t] = w;
  }
}

}  // namespace gemm
}  // namespace tasq
