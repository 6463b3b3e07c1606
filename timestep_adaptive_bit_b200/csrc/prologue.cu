// Activation prologue of the masked INT8 linear (one kernel, one pass over HBM):
//   z = x_pad . blockdiag(H_n)          block Hadamard along K, Sylvester H_n, n = 64 or 128
//                                       (HQ-DM technical summary, section 2.1 "Mecanismo";
//                                        6Bit-Diffusion section 2.A, Block Hadamard Transform)
//   a = max |z| over the padded row      per-token dynamic scale
//   q = clamp(RNE(z * (127 / a)), +-127) symmetric codes (HQ-DM section 2.2)
//   s_x = a / (127 sqrt(n))              the 2^(-k/2) normalisation folded into the scale
//                                        (HQ-DM section 2.1, "Eficiencia de Hardware")
//
// One CTA of 128 threads owns one token row. Thread t holds chunks c = j * 128 + t of 8
// consecutive channels (one 16-byte load each), so every warp load is 512 contiguous bytes.
// A Hadamard block of n channels is n / 8 consecutive chunks, i.e. n / 8 consecutive lanes of
// one warp: butterfly strides 1, 2, 4 run inside a thread's registers, strides 8 ... n/2 run
// across lanes with xor shuffles. The row never leaves registers between load and store.
// All arithmetic is FP32 round-to-nearest (no contraction: adds, subtracts and one multiply).
#include <cuda_fp16.h>

#include "tasq_internal.h"

namespace tasq {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ uint4 ld_stream_16B(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_8B(void* p, uint32_t lo, uint32_t hi) {
  asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(lo), "r"(hi) : "memory");
}

__device__ __forceinline__ uint32_t quant_byte(float z, float inv) {
  int q = __float2int_rn(__fmul_rn(z, inv));
  q = max(-127, min(127, q));
  return static_cast<uint32_t>(q) & 0xFFu;
}

template <int CHUNKS, int LANES_PER_BLOCK>
__global__ void __launch_bounds__(kThreads) prologue_kernel(const PrologueArgs a) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t row = blockIdx.x;
  const int real_chunks = a.K >> 3;
  const int all_chunks = a.Kp >> 3;
  const __half* xr = static_cast<const __half*>(a.x) + row * a.ldx;

  float v[CHUNKS][8];
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
    const int c = j * kThreads + tid;
    if (c < real_chunks) {
      const uint4 u = ld_stream_16B(xr + static_cast<int64_t>(c) * 8);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __half2 h2;
        *reinterpret_cast<uint32_t*>(&h2) = w[i];
        const float2 f = __half22float2(h2);
        v[j][2 * i] = f.x;
        v[j][2 * i + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[j][i] = 0.0f;
    }
  }

  // butterfly stages with element stride 1, 2, 4: inside the thread
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if ((i & h) == 0) {
          const float lo = v[j][i];
          const float hi = v[j][i + h];
          v[j][i] = __fadd_rn(lo, hi);
          v[j][i + h] = __fsub_rn(lo, hi);
        }
      }
    }
  }
  // stages with element stride 8 m (m = 1, 2, 4 [, 8]): partner chunk sits in lane ^ m
#pragma unroll
  for (int m = 1; m < LANES_PER_BLOCK; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int j = 0; j < CHUNKS; ++j) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float mine = v[j][i];
        const float other = __shfl_xor_sync(0xffffffffu, mine, m);
        v[j][i] = upper ? __fsub_rn(other, mine) : __fadd_rn(mine, other);
      }
    }
  }

  // per-token absmax over the padded row (chunks past Kp are zero and do not matter)
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[j][i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float red[kThreads / 32];
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));

  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  int8_t* qr = a.xq + row * a.Kp;
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
    const int c = j * kThreads + tid;
    if (c < all_chunks) {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) lo |= quant_byte(v[j][i], inv) << (8 * i);
#pragma unroll
      for (int i = 0; i < 4; ++i) hi |= quant_byte(v[j][4 + i], inv) << (8 * i);
      st_8B(qr + static_cast<int64_t>(c) * 8, lo, hi);
    }
  }
  if (tid == 0) a.s_x[row] = __fmul_rn(amax, a.sx_factor);
}

template <int LPB>
cudaError_t launch_for_chunks(int chunks, const PrologueArgs& a, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(a.M)), block(kThreads);
  switch (chunks) {
    case 1: prologue_kernel<1, LPB><<<grid, block, 0, s>>>(a); break;
    case 2: prologue_kernel<2, LPB><<<grid, block, 0, s>>>(a); break;
    case 3: prologue_kernel<3, LPB><<<grid, block, 0, s>>>(a); break;
    case 4: prologue_kernel<4, LPB><<<grid, block, 0, s>>>(a); break;
    case 5: case 6: prologue_kernel<6, LPB><<<grid, block, 0, s>>>(a); break;
    case 7: case 8: prologue_kernel<8, LPB><<<grid, block, 0, s>>>(a); break;
    case 9: case 10: case 11: case 12: prologue_kernel<12, LPB><<<grid, block, 0, s>>>(a); break;
    case 13: case 14: case 15: case 16: prologue_kernel<16, LPB><<<grid, block, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t stream) {
  if (a.M <= 0) return cudaSuccess;
  const int chunks = (a.Kp / 8 + kThreads - 1) / kThreads;
  if (a.n == 64) return launch_for_chunks<8>(chunks, a, stream);
  if (a.n == 128) return launch_for_chunks<16>(chunks, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace tasq
