// Activation prologue of the masked INT8 linear (one kernel, one pass over HBM):
//   z = x_pad . blockdiag(H_n)          block Hadamard along K, Sylvester H_n, n = 64 or 128
//                                       (HQ-DM technical summary, section 2.1 "Mecanismo";
//                                        6Bit-Diffusion section 2.A, Block Hadamard Transform)
//   a = max |z| over the padded row      per-token dynamic scale
//   q = clamp(RNE(z * (127 / a)), +-127) symmetric codes (HQ-DM section 2.2)
//   s_x = a / (127 sqrt(n))              the 2^(-k/2) normalisation folded into the scale
//                                        (HQ-DM section 2.1, "Eficiencia de Hardware")
//
// Work split: a CTA owns R consecutive token rows and R * C threads, C = Kp / 64. Thread i owns
// the 64 consecutive channels [64 (i % C), 64 (i % C) + 64) of row i / C: 128 contiguous bytes
// in, 64 contiguous bytes out, all 64 values in registers. R is chosen on the host so that R * C
// fills whole warps, which keeps every lane busy for any K (the kernel is issue-bound otherwise).
//
// The 64 values sit in 32 register pairs, pair p = (z_p, z_(p+32)), so the butterfly stages with
// stride 1, 2, 4, 8, 16 are packed FP32x2 add / fma (two independent IEEE round-to-nearest
// operations each), the stride-32 stage runs inside each pair, and for n = 128 the stride-64
// stage pairs the chunks of lanes 2j and 2j + 1 through one xor shuffle. The stages run in
// increasing stride, each butterfly (a, b) -> (a + b, a - b) rounded once in FP32, so the codes
// are the same bits as a textbook FP32 fast Walsh-Hadamard transform produces.
// The per-row absmax is combined through a shared-memory atomicMax on the float bits (all values
// are non-negative). No FMA contraction happens anywhere on the path.
#include <cuda_fp16.h>

#include "tasq_internal.h"

namespace tasq {
namespace {

constexpr int kMaxRowsPerCta = 64;
constexpr int kMaxThreads = 512;

__device__ __forceinline__ uint4 ld_16B(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void st_16B(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// (a + b) and (a - b), lane-wise on FP32 pairs; each result rounded once to nearest even.
__device__ __forceinline__ void butterfly2(float2& a, float2& b) {
  const uint64_t ua = *reinterpret_cast<const uint64_t*>(&a);
  const uint64_t ub = *reinterpret_cast<const uint64_t*>(&b);
  const float2 minus_one = make_float2(-1.0f, -1.0f);
  const uint64_t um = *reinterpret_cast<const uint64_t*>(&minus_one);
  uint64_t s, d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(s) : "l"(ua), "l"(ub));
  // b * (-1) + a is exact in the product, so the single rounding is that of a - b
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(ub), "l"(um), "l"(ua));
  a = *reinterpret_cast<const float2*>(&s);
  b = *reinterpret_cast<const float2*>(&d);
}

__device__ __forceinline__ float2 mul2(float2 a, float s) {
  const float2 ss = make_float2(s, s);
  const uint64_t ua = *reinterpret_cast<const uint64_t*>(&a);
  const uint64_t us = *reinterpret_cast<const uint64_t*>(&ss);
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ua), "l"(us));
  return *reinterpret_cast<const float2*>(&r);
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(b), 0x0040);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(c), static_cast<uint32_t>(d), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

__device__ __forceinline__ int code(float t) {
  int q = __float2int_rn(t);
  return max(-127, min(127, q));
}

template <int LANES_PER_BLOCK>
__global__ void __launch_bounds__(kMaxThreads) prologue_kernel(const PrologueArgs a, const int rows_per_cta) {
  const int C = a.Kp >> 6;                       // 64-channel chunks per row
  const int tid = threadIdx.x;
  const int r_local = tid / C;
  const int chunk = tid - r_local * C;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + r_local;
  const bool active = r_local < rows_per_cta && row < a.M;

  __shared__ unsigned int row_max[kMaxRowsPerCta];
  if (tid < rows_per_cta) row_max[tid] = 0u;
  __syncthreads();

  const int c0 = chunk * 64;
  float2 v[32];
  {
    uint4 u[8];
    const __half* src = static_cast<const __half*>(a.x) + row * a.ldx + c0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      u[j] = (active && c0 + 8 * j < a.K) ? ld_16B(src + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
      const uint32_t hi[4] = {u[j + 4].x, u[j + 4].y, u[j + 4].z, u[j + 4].w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        __half2 hl, hh;
        *reinterpret_cast<uint32_t*>(&hl) = lo[t];
        *reinterpret_cast<uint32_t*>(&hh) = hi[t];
        const float2 fl = __half22float2(hl);   // channels 8j + 2t, 8j + 2t + 1
        const float2 fh = __half22float2(hh);   // the same + 32
        v[8 * j + 2 * t] = make_float2(fl.x, fh.x);
        v[8 * j + 2 * t + 1] = make_float2(fl.y, fh.y);
      }
    }
  }

  // strides 1, 2, 4, 8, 16: pairs p and p + h, both halves at once
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int p = 0; p < 32; ++p) {
      if ((p & h) == 0) butterfly2(v[p], v[p + h]);
    }
  }
  // stride 32: inside each pair
#pragma unroll
  for (int p = 0; p < 32; ++p) {
    const float lo = v[p].x, hi = v[p].y;
    v[p].x = __fadd_rn(lo, hi);
    v[p].y = __fsub_rn(lo, hi);
  }
  // stride 64 (n = 128): the other half of the block is the chunk of lane ^ 1
  if constexpr (LANES_PER_BLOCK == 2) {
    const bool upper = (tid & 1) != 0;
#pragma unroll
    for (int p = 0; p < 32; ++p) {
      const float ox = __shfl_xor_sync(0xffffffffu, v[p].x, 1);
      const float oy = __shfl_xor_sync(0xffffffffu, v[p].y, 1);
      v[p].x = upper ? __fsub_rn(ox, v[p].x) : __fadd_rn(v[p].x, ox);
      v[p].y = upper ? __fsub_rn(oy, v[p].y) : __fadd_rn(v[p].y, oy);
    }
  }

  float m = 0.0f;
#pragma unroll
  for (int p = 0; p < 32; ++p) m = fmaxf(m, fmaxf(fabsf(v[p].x), fabsf(v[p].y)));
  if (active) atomicMax(&row_max[r_local], __float_as_uint(m));
  __syncthreads();
  if (!active) return;
  const float amax = __uint_as_float(row_max[r_local]);
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;

#pragma unroll
  for (int p = 0; p < 32; ++p) v[p] = mul2(v[p], inv);
  uint32_t w[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {   // bytes 4j .. 4j + 3 are channels 4j .. 4j + 3 (low half)
    w[j] = pack4(code(v[4 * j].x), code(v[4 * j + 1].x), code(v[4 * j + 2].x), code(v[4 * j + 3].x));
    w[8 + j] = pack4(code(v[4 * j].y), code(v[4 * j + 1].y), code(v[4 * j + 2].y), code(v[4 * j + 3].y));
  }
  int8_t* dst = a.xq + row * a.Kp + c0;
#pragma unroll
  for (int j = 0; j < 4; ++j) st_16B(dst + 16 * j, w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  if (chunk == 0) a.s_x[row] = __fmul_rn(amax, a.sx_factor);
}

// rows per CTA: fill whole warps (R * C a multiple of 32) with 128..512 threads where possible
int pick_rows(int C) {
  int best_r = 1;
  double best_score = -1.0;
  for (int r = 1; r <= kMaxRowsPerCta && r * C <= kMaxThreads; ++r) {
    const int t = r * C;
    const double util = static_cast<double>(t) / (((t + 31) / 32) * 32);
    double score = util;
    if (t < 128) score -= 0.05 * (128 - t) / 128.0;
    if (score > best_score + 1e-9) {
      best_score = score;
      best_r = r;
    }
  }
  return best_r;
}

}  // namespace

cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t stream) {
  if (a.M <= 0) return cudaSuccess;
  if (a.Kp % 64 != 0 || (a.n != 64 && a.n != 128)) return cudaErrorInvalidValue;
  const int C = a.Kp / 64;
  if (C > kMaxThreads) return cudaErrorInvalidValue;
  const int R = pick_rows(C);
  const int threads = ((R * C + 31) / 32) * 32;
  const int64_t grid = (a.M + R - 1) / R;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (a.n == 64)
    prologue_kernel<1><<<static_cast<unsigned>(grid), threads, 0, stream>>>(a, R);
  else
    prologue_kernel<2><<<static_cast<unsigned>(grid), threads, 0, stream>>>(a, R);
  return cudaGetLastError();
}

}  // namespace tasq
