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
constexpr int kAccCols = 256;                 // tokens per tile = INT32 TMEM columns per accumulator
constexpr int kAccStages = 2;
constexpr uint32_t kTmemCols = kAccCols * kAccStages;   // 512: the whole TMEM of the SM
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kMaskWarp0 = 10;
constexpr int kMaskWarps = 4;
constexpr int kThreads = 32 * (kEpiWarps + 2 + kMaskWarps);
constexpr int kMaskThreads = 32 * kMaskWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kEpiCols = kAccCols / (kEpiWarps / 4);     // 128 tokens per epilogue warp
constexpr int kSxBytesPerWarp = kEpiCols * 4;
constexpr int kMaxSmem = 232448;

template <int OUT>
struct OutTraits {
  static constexpr bool kS32 = OUT == static_cast<int>(OutKind::S32);
  static constexpr int kBytes = kS32 ? 4 : 2;
  static constexpr int kStageBytes = 32 * 32 * kBytes;   // one 32 x 32 output box per epilogue warp
};

__device__ __forceinline__ void raise_failure(uint32_t* status, volatile int* abort_flag, uint32_t bit) {
  atomicOr(status, bit);
  *abort_flag = 1;
}

// y = (acc * s_x) * s_w, each product rounded once in FP32, then rounded to the output type.
template <int OUT>
__device__ __forceinline__ uint16_t out_bits(uint32_t acc, float sx, float sw) {
  const float v = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(acc)), sx), sw);
  if constexpr (OUT == static_cast<int>(OutKind::F16)) {
    return __half_as_ushort(__float2half_rn(v));
  } else {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

// Epilogue role of warps 0..7. Warp w reads TMEM lanes 32 (w % 4) .. +31 (its 32 output channels)
// and accumulator columns 128 (w / 4) .. +127 (its 128 tokens) in chunks of 32 columns, scales,
// converts, writes the 32 x 32 box into its private staging buffer in output row order and
// stores it with one TMA bulk store. Warps never wait on each other.
//   ch_per_tile / ch_offset : output channels of tile nt start at nt * ch_per_tile + ch_offset.
//   acc_full + 8 i          : local barrier the MMA side arrives on when accumulator i is ready.
//   acc_empty + 8 i         : barrier (local, or in another CTA of the cluster when CLUSTER) that
//                             each epilogue warp arrives on once, after reading accumulator i.
template <int OUT, bool CLUSTER>
__device__ __forceinline__ void epilogue_role(const GemmArgs& g, const CUtensorMap* tmap_y, uint32_t tmem_base,
                                              uint8_t* stage, float* sx_slice, int warp, int lane, int tile0,
                                              int tile_step, int num_tiles, int ch_per_tile, int ch_offset,
                                              uint32_t acc_full, uint32_t acc_empty, uint64_t limit,
                                              volatile int* abort_flag) {
  using O = OutTraits<OUT>;
  const int q = warp & 3;         // TMEM lanes 32 q .. 32 q + 31
  const int h = warp >> 2;        // accumulator columns 128 h .. 128 h + 127
  const uint32_t stage_addr = ptx::smem_addr(stage);
  uint32_t as = 0, aph = 0;
  bool store_pending = false;
  // the token scales come from the prologue kernel just before this one
  ptx::grid_dep_wait();
  for (int tile = tile0; tile < num_tiles; tile += tile_step) {
    const int mt = tile % g.num_m_tiles;
    const int nt = tile / g.num_m_tiles;
    const int tok0 = mt * kAccCols + h * kEpiCols;
    const bool got = ptx::wait_bounded(acc_full + 8u * as, aph, limit, abort_flag);
    if (!__all_sync(0xffffffffu, got)) {
      if (lane == 0) raise_failure(g.status, abort_flag, TASQ_DEVICE_TIMEOUT_EPILOGUE);
      break;
    }
    ptx::tc_fence_after_sync();
    const int c0 = nt * ch_per_tile + ch_offset + q * 32;
    const int ch = c0 + lane;
    float sw = 0.0f;
    if constexpr (!O::kS32) {
      if (ch < g.N) sw = g.s_w[ch];
      // this warp's 128 token scales, read once per tile into its private slice
      float4 v4;
      const int m = tok0 + 4 * lane;
      v4.x = m < g.M ? g.s_x[m] : 0.0f;
      v4.y = m + 1 < g.M ? g.s_x[m + 1] : 0.0f;
      v4.z = m + 2 < g.M ? g.s_x[m + 2] : 0.0f;
      v4.w = m + 3 < g.M ? g.s_x[m + 3] : 0.0f;
      reinterpret_cast<float4*>(sx_slice)[lane] = v4;
      __syncwarp();
    }
    const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + as * kAccCols + h * kEpiCols;
#pragma unroll 1
    for (int j = 0; j < kEpiCols / 32; ++j) {
      uint32_t r[32];
      ptx::tmem_ld_32x32b_x32(tacc + j * 32, r);
      ptx::tmem_ld_wait(r);
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
      if (c0 + 32 > g.N && (g.N * O::kBytes) % 16 != 0) {
        // a TMA store writes whole 16-byte granules, so a box whose right edge is not 16-byte
        // aligned would write past column N: store this one with plain predicated stores
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          if (ch < g.N && t0 + t < g.M) {
            const int64_t idx = static_cast<int64_t>(t0 + t) * g.ldy + ch;
            if constexpr (O::kS32) {
              static_cast<int32_t*>(g.y)[idx] = static_cast<int32_t>(r[t]);
            } else {
              static_cast<uint16_t*>(g.y)[idx] = out_bits<OUT>(r[t], sx_slice[j * 32 + t], sw);
            }
          }
        }
        continue;
      }
      if (store_pending) {
        // the previous bulk store of this warp must have finished reading the staging tile
        if (lane == 0) ptx::bulk_wait_read0();
        __syncwarp();
      }
      if constexpr (O::kS32) {
        uint32_t* st = reinterpret_cast<uint32_t*>(stage);
#pragma unroll
        for (int t = 0; t < 32; ++t) st[t * 32 + lane] = r[t];
      } else {
        const float4* sx4 = reinterpret_cast<const float4*>(sx_slice + j * 32);
        uint16_t* st = reinterpret_cast<uint16_t*>(stage);
#pragma unroll
        for (int t4 = 0; t4 < 8; ++t4) {
          const float4 sx = sx4[t4];
          const float sxv[4] = {sx.x, sx.y, sx.z, sx.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) st[(4 * t4 + i) * 32 + lane] = out_bits<OUT>(r[4 * t4 + i], sxv[i], sw);
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
    as ^= 1u;
    if (as == 0) aph ^= 1u;
  }
  if (lane == 0) ptx::bulk_wait0();
}

// In-place LSB mask of one landed weight stage: every byte AND (0xFF << k), 16 bytes at a time.
template <int A_BYTES>
__device__ __forceinline__ void mask_stage(uint8_t* a_stage, int t, uint32_t mask32) {
  uint4* wt = reinterpret_cast<uint4*>(a_stage);
#pragma unroll
  for (int i = 0; i < A_BYTES / 16 / kMaskThreads; ++i) {
    uint4 w = wt[i * kMaskThreads + t];
    w.x &= mask32;
    w.y &= mask32;
    w.z &= mask32;
    w.w &= mask32;
    wt[i * kMaskThreads + t] = w;
  }
}

}  // namespace gemm
}  // namespace tasq
