// Activation prologue of the masked INT8 linear (one kernel, one pass over HBM):
//   z = x_pad . blockdiag(H_n)          block Hadamard along K, Sylvester H_n, n = 64 or 128
//                                       (HQ-DM technical summary, section 2.1 "Mecanismo";
//                                        6Bit-Diffusion section 2.A, Block Hadamard Transform)
//   a = max |z| over the padded row      per-token dynamic scale
//   q = clamp(RNE(z * (127 / a)), +-127) symmetric codes (HQ-DM section 2.2)
//   s_x = a / (127 sqrt(n))              the 2^(-k/2) normalisation folded into the scale
//                                        (HQ-DM section 2.1, "Eficiencia de Hardware")
//
// Work split: a CTA owns R consecutive token rows and R * L threads, L = Kp / 32. Thread i owns
// the 32 consecutive channels [32 (i % L), 32 (i % L) + 32) of row i / L: 64 contiguous bytes in
// (two full 32-byte sectors), 32 contiguous bytes out (one sector), all values in registers. A
// Hadamard block of n channels is n / 32 neighbouring lanes. R is chosen on the host so that R * L
// fills whole warps, which keeps every lane busy for any K.
//
// The 32 values sit in 16 register pairs, pair p = (z_p, z_(p+16)), so the butterfly stages with
// stride 1, 2, 4, 8 are packed FP32x2 add / fma (two independent IEEE round-to-nearest operations
// each), the stride-16 stage runs inside each pair, and the stride-32 (and, for n = 128,
// stride-64) stage pairs lane i with lane i ^ 1 (and i ^ 2) through xor shuffles and one packed
// fma by +-1 (exact product, one rounding). The stages run in increasing stride, each butterfly (a, b) -> (a + b, a - b) rounded once in FP32, so the codes
// are the same bits as a textbook FP32 fast Walsh-Hadamard transform produces.
// The per-row absmax is combined through a shared-memory atomicMax on the float bits (all values
// are non-negative). No FMA contraction happens anywhere on the path.
//
// The same launch can also truncate a layer's weights for the step (TASQ's LSB mask,
// w AND (0xFF << k) with k = 8 - bits): CTAs past the activation rows stream the layer's INT8
// weights once, 32 bytes per thread and load, into a masked copy that the GEMM then reads as its
// weight operand. Masking once per forward costs 2 N Kp bytes of HBM traffic; masking inside the
// GEMM costs a shared-memory read and write of every weight tile for every token tile.
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

// 32-byte load (one full sector); the address must be 32-byte aligned.
__device__ __forceinline__ void ld_32B(const void* p, uint32_t (&u)[8]) {
  float f[8];
  asm volatile("ld.global.L1::no_allocate.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3]), "=f"(f[4]), "=f"(f[5]), "=f"(f[6]), "=f"(f[7])
               : "l"(p));
#pragma unroll
  for (int i = 0; i < 8; ++i) u[i] = __float_as_uint(f[i]);
}

__device__ __forceinline__ void st_16B(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// 32-byte store (one full sector); the address must be 32-byte aligned.
__device__ __forceinline__ void st_32B(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.L1::no_allocate.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
               "f"(__uint_as_float(w[0])), "f"(__uint_as_float(w[1])), "f"(__uint_as_float(w[2])),
               "f"(__uint_as_float(w[3])), "f"(__uint_as_float(w[4])), "f"(__uint_as_float(w[5])),
               "f"(__uint_as_float(w[6])), "f"(__uint_as_float(w[7]))
               : "memory");
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

// Four INT32 codes to four signed bytes (a in the lowest byte), saturating to [-128, 127].
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  uint32_t hi, out;
  asm("cvt.pack.sat.s8.s32.b32 %0, %2, %1, 0;" : "=r"(hi) : "r"(c), "r"(d));
  asm("cvt.pack.sat.s8.s32.b32 %0, %2, %1, %3;" : "=r"(out) : "r"(a), "r"(b), "r"(hi));
  return out;
}

// RNE code of t = z * fp32(127 / a). With |z| <= a the two roundings keep |t| <= 127 (1 + 2^-23)
// < 127.5, so the code is always in [-127, 127]; the saturating pack is never reached.
__device__ __forceinline__ int code(float t) { return __float2int_rn(t); }

// other + s * mine on FP32 pairs with one rounding: s = +1 gives RN(mine + other), s = -1 gives
// RN(other - mine), the two outputs of a butterfly whose partner value sits in another lane.
__device__ __forceinline__ float2 fma2_sign(float2 mine, float s, float2 other) {
  const float2 ss = make_float2(s, s);
  const uint64_t um = *reinterpret_cast<const uint64_t*>(&mine);
  const uint64_t us = *reinterpret_cast<const uint64_t*>(&ss);
  const uint64_t uo = *reinterpret_cast<const uint64_t*>(&other);
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(um), "l"(us), "l"(uo));
  return *reinterpret_cast<const float2*>(&r);
}

constexpr int kWeightUnroll = 4;         // 32-byte loads in flight per thread in the weight pass
constexpr int64_t kMaxWeightCtas = 592;  // four CTAs for each of a B200's 148 SMs

// Weight pass of CTA `cta` of `num_ctas`: w_dst = w_src AND the step's byte mask.
__device__ __forceinline__ void weight_pass(const PrologueArgs& a, int64_t cta, int64_t num_ctas) {
  // the previous GEMM may still read w_dst: wait for it, then let the next kernel start its setup
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  int bits = a.bits_table[a.bits_index];
  if (bits < 1 || bits > 8) {
    if (cta == 0 && threadIdx.x == 0) atomicOr(a.status, TASQ_DEVICE_BAD_BITS);
    bits = 8;
  }
  const uint32_t m = 0x01010101u * ((0xFFu << (8 - bits)) & 0xFFu);
  const int64_t n32 = a.w_bytes >> 5;
  const int64_t stride = num_ctas * blockDim.x;
  for (int64_t i0 = cta * blockDim.x + threadIdx.x; i0 < n32; i0 += kWeightUnroll * stride) {
    uint32_t u[kWeightUnroll][8];
#pragma unroll
    for (int j = 0; j < kWeightUnroll; ++j) {
      const int64_t i = i0 + j * stride;
      if (i < n32) ld_32B(a.w_src + 32 * i, u[j]);
    }
#pragma unroll
    for (int j = 0; j < kWeightUnroll; ++j) {
      const int64_t i = i0 + j * stride;
      if (i < n32) {
#pragma unroll
        for (int e = 0; e < 8; ++e) u[j][e] &= m;
        st_32B(a.w_dst + 32 * i, u[j]);
      }
    }
  }
}

// LANES = n / 32 lanes per Hadamard block; VEC32: row starts of x and xq are 32-byte aligned.
// CTAs [0, row_ctas) quantize activation rows, the rest run the weight pass.
template <int LANES, bool VEC32>
__global__ void __launch_bounds__(kMaxThreads)
    prologue_kernel(const PrologueArgs a, const int rows_per_cta, const int row_ctas) {
  if (static_cast<int>(blockIdx.x) >= row_ctas) {
    weight_pass(a, blockIdx.x - row_ctas, gridDim.x - row_ctas);
    return;
  }
  const int L = a.Kp >> 5;                       // 32-channel segments per row
  const int tid = threadIdx.x;
  const int r_local = tid / L;
  const int seg = tid - r_local * L;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + r_local;
  const bool active = r_local < rows_per_cta && row < a.M;

  // x may be the previous kernel's output: wait for it, then let the GEMM start its setup
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  __shared__ unsigned int row_max[kMaxRowsPerCta];
  if (tid < rows_per_cta) row_max[tid] = 0u;
  __syncthreads();

  const int c0 = seg * 32;
  float2 v[16];
  {
    uint32_t u[16];   // u[i] holds channels c0 + 2i, c0 + 2i + 1
    const __half* src = static_cast<const __half*>(a.x) + row * a.ldx + c0;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      uint32_t* ug = u + 8 * g;
      const int e0 = c0 + 16 * g;
      if (active && e0 + 16 <= a.K) {
        if constexpr (VEC32) {
          uint32_t t[8];
          ld_32B(src + 16 * g, t);
#pragma unroll
          for (int i = 0; i < 8; ++i) ug[i] = t[i];
        } else {
          const uint4 p0 = ld_16B(src + 16 * g), p1 = ld_16B(src + 16 * g + 8);
          ug[0] = p0.x; ug[1] = p0.y; ug[2] = p0.z; ug[3] = p0.w;
          ug[4] = p1.x; ug[5] = p1.y; ug[6] = p1.z; ug[7] = p1.w;
        }
      } else if (active && e0 + 8 <= a.K) {
        const uint4 p0 = ld_16B(src + 16 * g);
        ug[0] = p0.x; ug[1] = p0.y; ug[2] = p0.z; ug[3] = p0.w;
        ug[4] = 0u; ug[5] = 0u; ug[6] = 0u; ug[7] = 0u;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) ug[i] = 0u;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      __half2 hl, hh;
      *reinterpret_cast<uint32_t*>(&hl) = u[i];       // channels 2i, 2i + 1
      *reinterpret_cast<uint32_t*>(&hh) = u[i + 8];   // channels 16 + 2i, 17 + 2i
      const float2 fl = __half22float2(hl);
      const float2 fh = __half22float2(hh);
      v[2 * i] = make_float2(fl.x, fh.x);
      v[2 * i + 1] = make_float2(fl.y, fh.y);
    }
  }

  // strides 1, 2, 4, 8: pairs p and p + h, both halves at once
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      if ((p & h) == 0) butterfly2(v[p], v[p + h]);
    }
  }
  // stride 16: inside each pair
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const float lo = v[p].x, hi = v[p].y;
    v[p].x = __fadd_rn(lo, hi);
    v[p].y = __fsub_rn(lo, hi);
  }
  // strides 32 (and 64): the partner segment of the block sits in lane ^ m; the lower lane keeps
  // mine + other, the upper lane other - mine
#pragma unroll
  for (int m = 1; m < LANES; m <<= 1) {
    const float sgn = (seg & m) != 0 ? -1.0f : 1.0f;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      float2 o;
      o.x = __shfl_xor_sync(0xffffffffu, v[p].x, m);
      o.y = __shfl_xor_sync(0xffffffffu, v[p].y, m);
      v[p] = fma2_sign(v[p], sgn, o);
    }
  }

  float mx = 0.0f;
#pragma unroll
  for (int p = 0; p < 16; ++p) mx = fmaxf(mx, fmaxf(fabsf(v[p].x), fabsf(v[p].y)));
  if (active) atomicMax(&row_max[r_local], __float_as_uint(mx));
  __syncthreads();
  if (!active) return;
  const float amax = __uint_as_float(row_max[r_local]);
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;

#pragma unroll
  for (int p = 0; p < 16; ++p) v[p] = mul2(v[p], inv);
  uint32_t w[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {   // bytes 4j .. 4j + 3 are channels 4j .. 4j + 3
    w[j] = pack4(code(v[4 * j].x), code(v[4 * j + 1].x), code(v[4 * j + 2].x), code(v[4 * j + 3].x));
    w[4 + j] = pack4(code(v[4 * j].y), code(v[4 * j + 1].y), code(v[4 * j + 2].y), code(v[4 * j + 3].y));
  }
  int8_t* dst = a.xq + row * a.Kp + c0;
  if constexpr (VEC32) {
    st_32B(dst, w);
  } else {
    st_16B(dst, w[0], w[1], w[2], w[3]);
    st_16B(dst + 16, w[4], w[5], w[6], w[7]);
  }
  if (seg == 0) a.s_x[row] = __fmul_rn(amax, a.sx_factor);
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
  const bool weights = a.w_bytes > 0;
  if (a.M <= 0 && !weights) return cudaSuccess;
  if (a.Kp % a.n != 0 || (a.n != 64 && a.n != 128)) return cudaErrorInvalidValue;
  if (weights && (a.w_bytes % 32 != 0 || reinterpret_cast<uintptr_t>(a.w_src) % 32 != 0 ||
                  reinterpret_cast<uintptr_t>(a.w_dst) % 32 != 0 || a.bits_table == nullptr || a.status == nullptr))
    return cudaErrorInvalidValue;
  const int L = a.Kp / 32;
  if (L > kMaxThreads) return cudaErrorInvalidValue;
  int R = 1, threads = 256;
  int64_t row_ctas = 0;
  if (a.M > 0) {
    R = pick_rows(L);
    threads = ((R * L + 31) / 32) * 32;
    row_ctas = (a.M + R - 1) / R;
  }
  int64_t weight_ctas = 0;
  if (weights) {
    // about kWeightUnroll 32-byte loads per thread; larger layers loop
    const int64_t per_cta = static_cast<int64_t>(threads) * 32 * kWeightUnroll;
    weight_ctas = (a.w_bytes + per_cta - 1) / per_cta;
    if (weight_ctas > kMaxWeightCtas) weight_ctas = kMaxWeightCtas;
  }
  const int64_t grid = row_ctas + weight_ctas;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  const bool vec32 = a.M > 0 && (reinterpret_cast<uintptr_t>(a.x) % 32 == 0) && (a.ldx % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(a.xq) % 32 == 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = use_pdl() ? 1 : 0;
  const int rc = static_cast<int>(row_ctas);
  if (a.n == 64) {
    if (vec32) return cudaLaunchKernelEx(&cfg, prologue_kernel<2, true>, a, R, rc);
    return cudaLaunchKernelEx(&cfg, prologue_kernel<2, false>, a, R, rc);
  }
  if (vec32) return cudaLaunchKernelEx(&cfg, prologue_kernel<4, true>, a, R, rc);
  return cudaLaunchKernelEx(&cfg, prologue_kernel<4, false>, a, R, rc);
}

}  // namespace tasq
