// Activation prologue of the masked INT8 linear (one kernel, one pass over HBM):
//   z = x_pad . blockdiag(H_n)          block Hadamard along K, Sylvester H_n, n = 64 or 128
//                                       (HQ-DM technical summary, section 2.1 "Mecanismo";
//                                        6Bit-Diffusion section 2.A, Block Hadamard Transform)
//   a = max |z| over the padded row      per-token dynamic scale
//   q = clamp(RNE(z * (127 / a)), +-127) symmetric codes (HQ-DM section 2.2)
//   s_x = a / (127 sqrt(n))              the 2^(-k/2) normalisation folded into the scale
//                                        (HQ-DM section 2.1, "Eficiencia de Hardware")
//
// Every thread owns 32 consecutive channels of one row, all values in registers; a Hadamard
// block of n channels is n / 32 threads of one warp. The 32 values sit in 16 register pairs,
// pair p = (z_p, z_(p+16)), so the butterfly stages with stride 1, 2, 4, 8 are packed FP32x2 add /
// fma (two independent IEEE round-to-nearest operations each), the stride-16 stage runs inside
// each pair, and the stride-32 (and, for n = 128, stride-64) stage pairs the thread with the one
// holding the partner segment through xor shuffles and one packed fma by +-1 (exact product, one
// rounding). The stages run in increasing stride, each butterfly (a, b) -> (a + b, a - b) rounded
// once in FP32, so the codes are the same bits as a textbook FP32 fast Walsh-Hadamard transform
// produces. The per-row absmax is combined through a shared-memory atomicMax on the float bits
// (all values are non-negative). No FMA contraction happens anywhere on the path.
//
// Three variants compute the same bits:
//   bulk-fed  one persistent CTA per SM; a producer warp streams blocks of rows into a ring of
//             shared-memory stages, one 1-D bulk copy per row, so that many bytes stay in flight
//             while up to 31 compute warps work on the stages already landed (any K % 8 == 0).
//   direct    a CTA owns R consecutive rows and R * Kp / 32 threads that load their 64 bytes
//             straight from global memory (two full sectors) and store 32 (one sector); it
//             serves the weight-only launch and arguments the bulk-fed layout does not fit.
//   direct64  the same with 64 channels (128 bytes) a thread, R * Kp / 64 threads a CTA: for
//             n = 64 a whole Hadamard block in one thread; taken for rows longer than 9216.
//
// The same launch can also truncate a layer's weights for the step (TASQ's LSB mask,
// w AND (0xFF << k) with k = 8 - bits) into a masked copy that the GEMM then reads as its weight
// operand: the bulk-fed CTAs do it after their rows, the direct variant in extra CTAs. Masking once
// per forward costs 2 N Kp bytes of HBM traffic; masking inside the GEMM costs a shared-memory
// read and write of every weight tile for every token tile.
#include <cuda_fp16.h>

#include <mutex>

#include "ptx.cuh"
#include "tasq_internal.h"

namespace tasq {
namespace {

constexpr int kMaxRowsPerCta = 64;
constexpr int kMaxThreads = 512;
constexpr int kSmallThreads = 288;   // CTAs up to this size get 56 registers: 4 CTAs per SM
constexpr int kMidThreads = 384;     // NVFP4 prologue: CTAs up to this size get 56 registers, 3 per SM

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

// ------------------------------------------------------------------------------ one segment
// The arithmetic of one thread's 32-channel segment, shared by both variants.

// u[i] holds channels 2i, 2i + 1 (FP16) -> v[p] = (z_p, z_(p+16)) in FP32 (exact).
__device__ __forceinline__ void to_pairs(const uint32_t (&u)[16], float2 (&v)[16]) {
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

// The block Hadamard butterflies of one segment, strides 1, 2, ..., n / 2 in that order, each
// (a, b) -> (a + b, a - b) rounded once in FP32. LANES = n / 32 segments per Hadamard block; the
// partner of segment `seg` for stride 32 m (m = 1, 2) is the thread `lane_unit * m` lanes away
// (xor), in the same warp.
template <int LANES>
__device__ __forceinline__ void fwht_segment(float2 (&v)[16], int seg, int lane_unit) {
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
  // strides 32 (and 64): the lower segment keeps mine + other, the upper one other - mine
#pragma unroll
  for (int m = 1; m < LANES; m <<= 1) {
    const float sgn = (seg & m) != 0 ? -1.0f : 1.0f;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      float2 o;
      o.x = __shfl_xor_sync(0xffffffffu, v[p].x, m * lane_unit);
      o.y = __shfl_xor_sync(0xffffffffu, v[p].y, m * lane_unit);
      v[p] = fma2_sign(v[p], sgn, o);
    }
  }
}

__device__ __forceinline__ float absmax_segment(const float2 (&v)[16]) {
  float mx = 0.0f;
#pragma unroll
  for (int p = 0; p < 16; ++p) mx = fmaxf(mx, fmaxf(fabsf(v[p].x), fabsf(v[p].y)));
  return mx;
}

// Codes RNE(fp32(z * inv)) of the segment; w[j] = channels 4j .. 4j + 3, lowest channel in the
// lowest byte.
__device__ __forceinline__ void codes_segment(float2 (&v)[16], float inv, uint32_t (&w)[8]) {
#pragma unroll
  for (int p = 0; p < 16; ++p) v[p] = mul2(v[p], inv);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[j] = pack4(code(v[4 * j].x), code(v[4 * j + 1].x), code(v[4 * j + 2].x), code(v[4 * j + 3].x));
    w[4 + j] = pack4(code(v[4 * j].y), code(v[4 * j + 1].y), code(v[4 * j + 2].y), code(v[4 * j + 3].y));
  }
}

constexpr int kWeightUnroll = 4;         // 32-byte loads in flight per thread in the weight pass
constexpr int64_t kMaxWeightCtas = 592;  // four CTAs for each of a B200's 148 SMs

// A thread's row within its CTA is tid / L for the L segment threads of a row. The kernels take
// it as (tid * row_mul) >> kRowShift with row_mul = ceil(2^20 / L). For tid < 2^10 and L <= 2^9
// the product stays below 2^30 and exceeds tid * 2^20 / L by less than tid < 2^10, while
// tid * 2^20 / L lies at least 2^20 / L >= 2^11 below the next multiple of 2^20, so the shift
// gives the exact quotient. It replaces a runtime integer division (a reciprocal, two conversions
// and corrections) that every thread paid once.
constexpr int kRowShift = 20;

int row_multiplier(int L) { return static_cast<int>(((1 << kRowShift) + L - 1) / L); }

// Weight pass over `count` cooperating threads, thread `idx` of them.
__device__ __forceinline__ void weight_pass_threads(const PrologueArgs& a, int64_t idx, int64_t count) {
  for (int seg = 0; seg < a.num_w; ++seg) {
    const PrologueArgs::WeightSegment& ws = a.w[seg];
    int bits = a.bits_table[ws.bits_index];
    if (bits < 1 || bits > 8) {
      if (idx == 0) atomicOr(a.status, TASQ_DEVICE_BAD_BITS);
      bits = 8;
    }
    const uint32_t m = 0x01010101u * ((0xFFu << (8 - bits)) & 0xFFu);
    const int64_t n32 = ws.bytes >> 5;
    for (int64_t i0 = idx; i0 < n32; i0 += kWeightUnroll * count) {
      uint32_t u[kWeightUnroll][8];
#pragma unroll
      for (int jj = 0; jj < kWeightUnroll; ++jj) {
        const int64_t i = i0 + jj * count;
        if (i < n32) ld_32B(ws.src + 32 * i, u[jj]);
      }
#pragma unroll
      for (int jj = 0; jj < kWeightUnroll; ++jj) {
        const int64_t i = i0 + jj * count;
        if (i < n32) {
#pragma unroll
          for (int e = 0; e < 8; ++e) u[jj][e] &= m;
          st_32B(ws.dst + 32 * i, u[jj]);
        }
      }
    }
  }
}

// Weight pass of CTA `cta` of `num_ctas` of the direct variant: w_dst = w_src AND the step's
// byte mask.
__device__ __forceinline__ void weight_pass(const PrologueArgs& a, int64_t cta, int64_t num_ctas) {
  // the previous GEMM may still read w_dst: wait for it, then let the next kernel start its setup
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  weight_pass_threads(a, cta * blockDim.x + threadIdx.x, num_ctas * blockDim.x);
}

// LANES = n / 32 lanes per Hadamard block; VEC32: row starts of x and xq are 32-byte aligned.
// CTAs [0, row_ctas) quantize activation rows, the rest run the weight pass.
template <int LANES, bool VEC32, int MAXT, int MINB>
__global__ void __launch_bounds__(MAXT, MINB)
    prologue_kernel(const PrologueArgs a, const int rows_per_cta, const int row_ctas, const int row_mul) {
  if (gated_out(a.gate, a.bits_table, a.gate_index)) return;
  if (static_cast<int>(blockIdx.x) >= row_ctas) {
    weight_pass(a, blockIdx.x - row_ctas, gridDim.x - row_ctas);
    return;
  }
  const int L = a.Kp >> 5;                       // 32-channel segments per row
  const int tid = threadIdx.x;
  const int r_local = (tid * row_mul) >> kRowShift;   // tid / L (see row_multiplier)
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
    to_pairs(u, v);
  }
  fwht_segment<LANES>(v, seg, 1);
  const float mx = absmax_segment(v);
  if (active) atomicMax(&row_max[r_local], __float_as_uint(mx));
  __syncthreads();
  if (!active) return;
  const float amax = __uint_as_float(row_max[r_local]);
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  uint32_t w[8];
  codes_segment(v, inv, w);
  int8_t* dst = a.xq + row * a.Kp + c0;
  if constexpr (VEC32) {
    st_32B(dst, w);
  } else {
    st_16B(dst, w[0], w[1], w[2], w[3]);
    st_16B(dst + 16, w[4], w[5], w[6], w[7]);
  }
  if (seg == 0) a.s_x[row] = __fmul_rn(amax, a.sx_factor);
}

// ------------------------------------------------------------------------------ 64 channels a thread
// The same arithmetic with 64 consecutive channels per thread: for n = 64 a thread holds a whole
// Hadamard block, so every butterfly stage stays in registers (no shuffle), and the per-thread
// costs (addressing, the row's absmax, the division) are spread over twice the elements. The 64
// values sit in 32 register pairs, pair p = (z_p, z_(p+32)): strides 1 .. 16 are packed FP32x2
// add / fma between pairs, stride 32 runs inside each pair; for n = 128 the stride-64 stage pairs
// the two threads of a block through one xor shuffle. The stages run in increasing stride, each
// butterfly rounded once in FP32, exactly as in the 32-channel kernel.

// u[i] holds channels 2i, 2i + 1 (FP16) -> v[p] = (z_p, z_(p+32)) in FP32 (exact).
__device__ __forceinline__ void to_pairs64(const uint32_t (&u)[32], float2 (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    __half2 hl, hh;
    *reinterpret_cast<uint32_t*>(&hl) = u[i];        // channels 2i, 2i + 1
    *reinterpret_cast<uint32_t*>(&hh) = u[i + 16];   // channels 32 + 2i, 33 + 2i
    const float2 fl = __half22float2(hl);
    const float2 fh = __half22float2(hh);
    v[2 * i] = make_float2(fl.x, fh.x);
    v[2 * i + 1] = make_float2(fl.y, fh.y);
  }
}

template <bool N128>
__device__ __forceinline__ void fwht_segment64(float2 (&v)[32], int seg) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int p = 0; p < 32; ++p) {
      if ((p & h) == 0) butterfly2(v[p], v[p + h]);
    }
  }
#pragma unroll
  for (int p = 0; p < 32; ++p) {
    const float lo = v[p].x, hi = v[p].y;
    v[p].x = __fadd_rn(lo, hi);
    v[p].y = __fsub_rn(lo, hi);
  }
  if constexpr (N128) {
    // stride 64: the lower segment of the block keeps mine + other, the upper one other - mine
    const float sgn = (seg & 1) != 0 ? -1.0f : 1.0f;
#pragma unroll
    for (int p = 0; p < 32; ++p) {
      float2 o;
      o.x = __shfl_xor_sync(0xffffffffu, v[p].x, 1);
      o.y = __shfl_xor_sync(0xffffffffu, v[p].y, 1);
      v[p] = fma2_sign(v[p], sgn, o);
    }
  }
}

__device__ __forceinline__ float absmax_segment64(const float2 (&v)[32]) {
  float mx = 0.0f;
#pragma unroll
  for (int p = 0; p < 32; ++p) mx = fmaxf(mx, fmaxf(fabsf(v[p].x), fabsf(v[p].y)));
  return mx;
}

// Codes of the 64 channels: w[j] = channels 4j .. 4j + 3 (j < 8 from the .x halves, j >= 8 the
// .y halves), the lowest channel in the lowest byte.
__device__ __forceinline__ void codes_segment64(float2 (&v)[32], float inv, uint32_t (&w)[16]) {
#pragma unroll
  for (int p = 0; p < 32; ++p) v[p] = mul2(v[p], inv);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    w[j] = pack4(code(v[4 * j].x), code(v[4 * j + 1].x), code(v[4 * j + 2].x), code(v[4 * j + 3].x));
    w[8 + j] = pack4(code(v[4 * j].y), code(v[4 * j + 1].y), code(v[4 * j + 2].y), code(v[4 * j + 3].y));
  }
}

// N128: n = 128 (two threads per Hadamard block); VEC32: rows of x and xq 32-byte aligned. A CTA
// owns rows_per_cta rows of Kp / 64 threads each; CTAs [row_ctas, gridDim) run the weight pass.
template <bool N128, bool VEC32, int MAXT, int MINB>
__global__ void __launch_bounds__(MAXT, MINB)
    prologue64_kernel(const PrologueArgs a, const int rows_per_cta, const int row_ctas, const int row_mul) {
  if (gated_out(a.gate, a.bits_table, a.gate_index)) return;
  if (static_cast<int>(blockIdx.x) >= row_ctas) {
    weight_pass(a, blockIdx.x - row_ctas, gridDim.x - row_ctas);
    return;
  }
  const int L = a.Kp >> 6;                       // 64-channel segments per row
  const int tid = threadIdx.x;
  const int r_local = (tid * row_mul) >> kRowShift;   // tid / L (see row_multiplier)
  const int seg = tid - r_local * L;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_cta + r_local;
  const bool active = r_local < rows_per_cta && row < a.M;

  // x may be the previous kernel's output: wait for it, then let the GEMM start its setup
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  __shared__ unsigned int row_max[kMaxRowsPerCta];
  if (tid < rows_per_cta) row_max[tid] = 0u;
  __syncthreads();

  const int c0 = seg * 64;
  float2 v[32];
  {
    uint32_t u[32];   // u[i] holds channels c0 + 2i, c0 + 2i + 1
    const __half* src = static_cast<const __half*>(a.x) + row * a.ldx + c0;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
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
    to_pairs64(u, v);
  }
  fwht_segment64<N128>(v, seg);
  const float mx = absmax_segment64(v);
  if (active) atomicMax(&row_max[r_local], __float_as_uint(mx));
  __syncthreads();
  if (!active) return;
  const float amax = __uint_as_float(row_max[r_local]);
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  uint32_t w[16];
  codes_segment64(v, inv, w);
  int8_t* dst = a.xq + row * a.Kp + c0;
  if constexpr (VEC32) {
    uint32_t w0[8], w1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w0[i] = w[i];
      w1[i] = w[8 + i];
    }
    st_32B(dst, w0);
    st_32B(dst + 32, w1);
  } else {
    st_16B(dst, w[0], w[1], w[2], w[3]);
    st_16B(dst + 16, w[4], w[5], w[6], w[7]);
    st_16B(dst + 32, w[8], w[9], w[10], w[11]);
    st_16B(dst + 48, w[12], w[13], w[14], w[15]);
  }
  if (seg == 0) a.s_x[row] = __fmul_rn(amax, a.sx_factor);
}

// ------------------------------------------------------------------------------ NVFP4 variant
// The NVFP4 step of 6Bit-Diffusion (technical summary, section 2.A: the stable layers of a step
// in NVFP4, Blackwell's 4-bit format, after the same block Hadamard). The thread layout, loads and
// transform are those of the direct INT8 kernel; then per token u = z * fp32(2688 / a), and per
// 16-block of a row b = max |u|, the UE4M3 scale sb = RNE(fp32(b / 6)) and the E2M1 codes
// RNE(fp32(u * fp32(1 / sb))), both saturating; a block whose scale is 0 gets zero codes. The
// thread's 32 channels are two whole 16-blocks: the .x halves of its register pairs and the .y
// halves.

// UE4M3 code of s >= 0, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_code(float s) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(s), "f"(s));
  return h & 0xFFu;
}

// Value of a UE4M3 code, exact (every E4M3 value is an FP16 value). The code sits in both bytes,
// so either half of the FP16 pair holds it.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h2;
  const uint16_t both = static_cast<uint16_t>(code | (code << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(both));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// E2M1 codes of eight values (round to nearest even, saturating at 6), t[0] in the lowest nibble.
__device__ __forceinline__ uint32_t e2m1_x8(const float (&t)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(t[0]), "f"(t[1]), "f"(t[2]), "f"(t[3]), "f"(t[4]), "f"(t[5]), "f"(t[6]), "f"(t[7]));
  return r;
}

__device__ __forceinline__ float2 mul2v(float2 a, float2 b) {
  const uint64_t ua = *reinterpret_cast<const uint64_t*>(&a);
  const uint64_t ub = *reinterpret_cast<const uint64_t*>(&b);
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ua), "l"(ub));
  return *reinterpret_cast<const float2*>(&r);
}

// Byte of row r, 16-block j in the chunked scale layout (see Nvfp4PrologueArgs).
__device__ __forceinline__ int64_t nvfp4_sf_offset(int64_t r, int64_t j, int64_t chunks_per_group) {
  return ((r >> 7) * chunks_per_group + (j >> 2)) * kNvfp4ChunkBytes + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3);
}

// NVFP4 codes and scale of 16 INT8 weights (one block of one output channel), given as the four
// 32-bit words that hold them: 8 bytes of E2M1 codes (lower-indexed element in the low nibble)
// and the UE4M3 scale byte.
__device__ __forceinline__ uint32_t nvfp4_weight_block(const uint4 q, uint2* codes) {
  const uint32_t words[4] = {q.x, q.y, q.z, q.w};
  float f[16];
  int m = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int v = static_cast<int8_t>((words[i >> 2] >> (8 * (i & 3))) & 0xFFu);
    f[i] = static_cast<float>(v);
    m = max(m, abs(v));
  }
  const uint32_t sc = e4m3_code(__fdiv_rn(static_cast<float>(m), 6.0f));
  const float d = e4m3_value(sc);
  const float r = d > 0.0f ? __frcp_rn(d) : 0.0f;
  float t0[8], t1[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    t0[i] = __fmul_rn(f[i], r);
    t1[i] = __fmul_rn(f[8 + i], r);
  }
  *codes = d == 0.0f ? make_uint2(0u, 0u) : make_uint2(e2m1_x8(t0), e2m1_x8(t1));
  return sc;
}

// Weight conversion of CTA `cta` of `num_ctas`. One thread per four consecutive 16-blocks of a
// row: 64 INT8 weights in (four independent 16-byte loads), 32 bytes of codes and one 32-bit word
// of scales out (the four blocks' scales are adjacent bytes of the chunked layout). Quads past Kp
// (Kp is a multiple of 64, so a quad is wholly inside or outside) get zero scales, so that the
// GEMM's last stage multiplies zero codes by zero.
__device__ __forceinline__ void nvfp4_weight_pass(const Nvfp4PrologueArgs& a, int cta, int num_ctas) {
  // the previous GEMM may still read the converted weights: wait for it
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (cta == 0 && threadIdx.x == 0 && a.bits_table != nullptr && a.bits_table[a.bits_index] != 0)
    atomicOr(a.status, TASQ_DEVICE_BAD_BITS);
  const int nb = a.Kp / kNvfp4Block;
  const int quads = static_cast<int>(nvfp4_kp4(a.Kp) / 64);   // per row; = scale chunks per row group
  const int total = a.N * quads;
  const int stride = num_ctas * static_cast<int>(blockDim.x);
  for (int qd = cta * static_cast<int>(blockDim.x) + static_cast<int>(threadIdx.x); qd < total; qd += stride) {
    const int row = qd / quads;
    const int j0 = 4 * (qd - row * quads);
    uint32_t* sf = reinterpret_cast<uint32_t*>(a.w_sf + nvfp4_sf_offset(row, j0, quads));
    if (j0 >= nb) {
      *sf = 0u;
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(a.w + static_cast<int64_t>(row) * a.Kp + 16 * j0);
    uint4 q[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) q[b] = __ldg(src + b);
    uint2 c[4];
    uint32_t scales = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) scales |= nvfp4_weight_block(q[b], &c[b]) << (8 * b);
    uint4* dst = reinterpret_cast<uint4*>(a.w_codes + static_cast<int64_t>(row) * (a.Kp / 2) + 8 * j0);
    dst[0] = make_uint4(c[0].x, c[0].y, c[1].x, c[1].y);
    dst[1] = make_uint4(c[2].x, c[2].y, c[3].x, c[3].y);
    *sf = scales;
  }
}

template <int LANES, int MAXT, int MINB>
__global__ void __launch_bounds__(MAXT, MINB)
    prologue_nvfp4_kernel(const Nvfp4PrologueArgs a, const int rows_per_cta, const int row_ctas, const int row_mul) {
  if (gated_out(a.gate, a.gate_table, a.gate_index)) return;
  // CTAs [0, weight_ctas) convert the weights (each loops over several quads, so they start
  // first), the rest quantize activation rows
  const int weight_ctas = static_cast<int>(gridDim.x) - row_ctas;
  if (static_cast<int>(blockIdx.x) < weight_ctas) {
    nvfp4_weight_pass(a, blockIdx.x, weight_ctas);
    return;
  }
  const int row_block = static_cast<int>(blockIdx.x) - weight_ctas;
  const int L = a.Kp >> 5;
  const int tid = threadIdx.x;
  const int r_local = (tid * row_mul) >> kRowShift;   // tid / L (see row_multiplier)
  const int seg = tid - r_local * L;
  const int64_t row = static_cast<int64_t>(row_block) * rows_per_cta + r_local;
  const bool active = r_local < rows_per_cta && row < a.M;

  // x may be the previous kernel's output, and the previous GEMM may still read the codes
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  __shared__ unsigned int row_max[kMaxRowsPerCta];
  if (tid < rows_per_cta) row_max[tid] = 0u;
  __syncthreads();

  const int c0 = seg * 32;
  float2 v[16];
  {
    uint32_t u[16];
    const __half* src = static_cast<const __half*>(a.x) + row * a.ldx + c0;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      uint32_t* ug = u + 8 * g;
      const int e0 = c0 + 16 * g;
      if (active && e0 + 16 <= a.K) {
        const uint4 p0 = ld_16B(src + 16 * g), p1 = ld_16B(src + 16 * g + 8);
        ug[0] = p0.x; ug[1] = p0.y; ug[2] = p0.z; ug[3] = p0.w;
        ug[4] = p1.x; ug[5] = p1.y; ug[6] = p1.z; ug[7] = p1.w;
      } else if (active && e0 + 8 <= a.K) {
        const uint4 p0 = ld_16B(src + 16 * g);
        ug[0] = p0.x; ug[1] = p0.y; ug[2] = p0.z; ug[3] = p0.w;
        ug[4] = 0u; ug[5] = 0u; ug[6] = 0u; ug[7] = 0u;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) ug[i] = 0u;
      }
    }
    to_pairs(u, v);
  }
  fwht_segment<LANES>(v, seg, 1);
  const float mx = absmax_segment(v);
  if (active) atomicMax(&row_max[r_local], __float_as_uint(mx));
  __syncthreads();
  if (!active) return;
  const float amax = __uint_as_float(row_max[r_local]);
  const float g = amax > 0.0f ? __fdiv_rn(kNvfp4Range, amax) : 0.0f;
  float b0 = 0.0f, b1 = 0.0f;
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    v[p] = mul2(v[p], g);
    b0 = fmaxf(b0, fabsf(v[p].x));
    b1 = fmaxf(b1, fabsf(v[p].y));
  }
  const uint32_t s0 = e4m3_code(__fdiv_rn(b0, 6.0f)), s1 = e4m3_code(__fdiv_rn(b1, 6.0f));
  const float d0 = e4m3_value(s0), d1 = e4m3_value(s1);
  const float2 r = make_float2(d0 > 0.0f ? __frcp_rn(d0) : 0.0f, d1 > 0.0f ? __frcp_rn(d1) : 0.0f);
  float t0[8], t1[8], t2[8], t3[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const float2 lo = mul2v(v[p], r), hi = mul2v(v[p + 8], r);
    t0[p] = lo.x;   // block 0: channels c0 .. c0 + 7
    t1[p] = hi.x;   //          c0 + 8 .. c0 + 15
    t2[p] = lo.y;   // block 1: c0 + 16 .. c0 + 23
    t3[p] = hi.y;   //          c0 + 24 .. c0 + 31
  }
  uint32_t w0 = e2m1_x8(t0), w1 = e2m1_x8(t1), w2 = e2m1_x8(t2), w3 = e2m1_x8(t3);
  if (d0 == 0.0f) w0 = w1 = 0u;
  if (d1 == 0.0f) w2 = w3 = 0u;
  st_16B(a.codes + row * (a.Kp / 2) + c0 / 2, w0, w1, w2, w3);
  const int64_t chunks = nvfp4_kp4(a.Kp) / 64;
  *reinterpret_cast<uint16_t*>(a.sf + nvfp4_sf_offset(row, c0 >> 4, chunks)) = static_cast<uint16_t>(s0 | (s1 << 8));
  if (seg == 0) a.s_x[row] = __fmul_rn(amax, a.sx_factor);
}

// ------------------------------------------------------------------------------ bulk-fed variant
constexpr int kFedMaxCompute = 992;           // compute threads per CTA (one CTA per SM)
constexpr int kFedMaxStageBytes = 50 * 1024;
constexpr int kFedSmemBudget = 200 * 1024;    // stage ring
constexpr int kFedMaxStages = 8;

struct FedGeom {
  int32_t RG;           // rows per group (power of two); a row's segments sit RG lanes apart
  int32_t R;            // rows per block, a multiple of RG
  int32_t L;            // 32-channel segments per padded row = Kp / 32
  int32_t T;            // compute threads = R * L; RG * L is a multiple of 32
  int32_t row_stride;   // bytes between rows in a stage: round_up(2 K, 128) + 16
  int32_t stages;
  int32_t stage_bytes;  // R * row_stride rounded up to 128
  int64_t num_blocks;   // ceil(M / R)
  int32_t vec32;        // xq rows are 32-byte aligned
};

// AND of `p` over the T compute threads, which all wait at named barrier 1 (the barrier also
// orders their shared-memory accesses).
__device__ __forceinline__ bool all_compute(bool p, int T) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred q, r;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "barrier.cta.red.and.pred r, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, r;\n\t}"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(p)), "r"(T)
      : "memory");
  return out != 0;
}

// One persistent CTA per SM. Warp T / 32 streams blocks of R rows into a ring of stages, one
// 1-D bulk copy of 2 K bytes per row (its 32 lanes issue them), rows 16 bytes apart modulo 128 so
// that the compute threads' 16-byte reads hit distinct banks. Compute thread t owns row
// (t / (RG L)) RG + t % RG and segment (t / RG) % L of the block: the RG threads of a warp that
// share a segment read RG consecutive rows, and the segments of one Hadamard block sit RG (and
// 2 RG) lanes apart.
template <int LANES>
__global__ void __launch_bounds__(kFedMaxCompute + 32, 1)
    prologue_fed_kernel(const PrologueArgs a, const FedGeom geo) {
  if (gated_out(a.gate, a.bits_table, a.gate_index)) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const uint32_t sbase = ptx::smem_addr(smem);
  const int S = geo.stages;
  const int R = geo.R;
  const int T = geo.T;
  const uint32_t full0 = sbase + S * geo.stage_bytes;
  const uint32_t empty0 = full0 + 8 * S;
  unsigned int* row_max = reinterpret_cast<unsigned int*>(smem + S * geo.stage_bytes + 16 * S);   // [3][R]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(row_max + 3 * R);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const uint64_t limit = a.wait_limit_ns;

  // x may be the previous kernel's output and the previous GEMM may still read the workspace:
  // wait for it, then let the next kernel start its setup
  ptx::grid_dep_wait();
  ptx::grid_dep_launch_dependents();

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(full0 + 8 * i, 1);
      ptx::mbar_init(empty0 + 8 * i, T / 32);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  for (int i = tid; i < 3 * R; i += blockDim.x) row_max[i] = 0u;
  __syncthreads();

  const uint32_t row_bytes = static_cast<uint32_t>(a.K) * 2u;
  if (tid >= T) {
    // ------------------------------------------------------------------ producer warp
    const char* x = static_cast<const char*>(a.x);
    uint32_t s = 0, ph = 0, issued = 0, issued_par = 0;
    for (int64_t rb = blockIdx.x; rb < geo.num_blocks; rb += gridDim.x) {
      bool ok = true;
      if (lane == 0) ok = ptx::wait_bounded(empty0 + 8 * s, ph ^ 1u, limit, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) {
          atomicOr(a.status, TASQ_DEVICE_TIMEOUT_PROLOGUE);
          *abort_flag = 1;
        }
        break;
      }
      const int64_t left = a.M - rb * R;
      const int rows = left < R ? static_cast<int>(left) : R;
      if (lane == 0) ptx::mbar_arrive_expect_tx(full0 + 8 * s, static_cast<uint32_t>(rows) * row_bytes);
      __syncwarp();
      for (int i = lane; i < rows; i += 32) {
        ptx::bulk_load(sbase + s * geo.stage_bytes + i * geo.row_stride, x + (rb * R + i) * a.ldx * 2, row_bytes,
                       full0 + 8 * s);
      }
      issued |= 1u << s;
      issued_par = (issued_par & ~(1u << s)) | (ph << s);
      if (++s == static_cast<uint32_t>(S)) {
        s = 0;
        ph ^= 1u;
      }
    }
    // every copy this warp issued must have landed before the CTA may exit
    if (lane == 0) {
      for (int i = 0; i < S; ++i) {
        if ((issued >> i) & 1u) {
          if (!ptx::wait_bounded(full0 + 8 * i, (issued_par >> i) & 1u, limit, nullptr))
            atomicOr(a.status, TASQ_DEVICE_TIMEOUT_PROLOGUE);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------------- compute threads
  const int RG = geo.RG;
  const int r_in = tid & (RG - 1);
  const int q = tid / RG;
  const int seg = q % geo.L;
  const int rl = (q / geo.L) * RG + r_in;         // row of the block
  const int c0 = 32 * seg;                        // first channel of the segment
  uint32_t s = 0, ph = 0;
  int buf = 0;
  bool ok = true;
  for (int64_t rb = blockIdx.x; rb < geo.num_blocks; rb += gridDim.x) {
    const bool got = ptx::wait_bounded(full0 + 8 * s, ph, limit, abort_flag);
    const int64_t row = rb * R + rl;
    const bool valid = row < a.M;
    float2 v[16];
    {
      uint32_t u[16];
      const uint8_t* src = smem + s * geo.stage_bytes + rl * geo.row_stride + 2 * c0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {   // 8 channels per 16-byte chunk; K % 8 == 0
        if (got && valid && c0 + 8 * c + 8 <= a.K) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(src + 16 * c);
          u[4 * c] = q4.x;
          u[4 * c + 1] = q4.y;
          u[4 * c + 2] = q4.z;
          u[4 * c + 3] = q4.w;
        } else {
          u[4 * c] = 0u;
          u[4 * c + 1] = 0u;
          u[4 * c + 2] = 0u;
          u[4 * c + 3] = 0u;
        }
      }
      // the stage is in registers: hand it back to the producer (one arrival per warp)
      if (__all_sync(0xffffffffu, got) && lane == 0) ptx::mbar_arrive(empty0 + 8 * s);
      to_pairs(u, v);
    }
    fwht_segment<LANES>(v, seg, RG);
    float mx = absmax_segment(v);
    // the lanes of this warp that hold the same row are RG apart
    for (int off = RG; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (got && lane < RG) atomicMax(&row_max[buf * R + rl], __float_as_uint(mx));
    if (!all_compute(got, T)) {
      if (tid == 0) {
        atomicOr(a.status, TASQ_DEVICE_TIMEOUT_PROLOGUE);
        *abort_flag = 1;
      }
      ok = false;
      break;
    }
    // the buffer of the previous block was read before the barrier just passed: clear it for
    // the block after next
    const int prev = buf == 0 ? 2 : buf - 1;
    if (seg == 0) row_max[prev * R + rl] = 0u;
    const float amax = __uint_as_float(row_max[buf * R + rl]);
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    if (valid) {
      uint32_t w[8];
      codes_segment(v, inv, w);
      int8_t* dst = a.xq + row * a.Kp + c0;
      if (geo.vec32) {
        st_32B(dst, w);
      } else {
        st_16B(dst, w[0], w[1], w[2], w[3]);
        st_16B(dst + 16, w[4], w[5], w[6], w[7]);
      }
      if (seg == 0) a.s_x[row] = __fmul_rn(amax, a.sx_factor);
    }
    buf = buf == 2 ? 0 : buf + 1;
    if (++s == static_cast<uint32_t>(S)) {
      s = 0;
      ph ^= 1u;
    }
  }
  if (ok && a.num_w > 0)
    weight_pass_threads(a, static_cast<int64_t>(blockIdx.x) * T + tid, static_cast<int64_t>(gridDim.x) * T);
}

// Geometry of the bulk-fed variant for (n, K, Kp), or R = 0 when no layout fits.
FedGeom fed_geometry(int n, int K, int Kp) {
  FedGeom g{};
  g.L = Kp / 32;
  g.row_stride = static_cast<int32_t>(round_up(static_cast<size_t>(K) * 2, 128) + 16);
  // the segments of a Hadamard block must sit in one warp: RG * (n / 32) <= 32
  const int rg_max = n == 64 ? 16 : 8;
  for (int rg = rg_max; rg >= 1; rg >>= 1) {
    if ((rg * g.L) % 32 == 0 && rg * g.L <= kFedMaxCompute) {
      g.RG = rg;
      break;
    }
  }
  if (g.RG == 0) return g;
  int groups = kFedMaxCompute / (g.RG * g.L);
  while (groups > 1 && static_cast<int64_t>(groups) * g.RG * g.row_stride > kFedMaxStageBytes) --groups;
  g.R = groups * g.RG;
  g.T = g.R * g.L;
  g.stage_bytes = static_cast<int32_t>(round_up(static_cast<size_t>(g.R) * g.row_stride, 128));
  g.stages = kFedSmemBudget / g.stage_bytes;
  if (g.stages > kFedMaxStages) g.stages = kFedMaxStages;
  if (g.stages < 2) g.R = 0;
  return g;
}

// rows per CTA: fill whole warps (R * C a multiple of 32) with 128..cap threads where possible
int pick_rows(int C, int cap) {
  int best_r = 1;
  double best_score = -1.0;
  for (int r = 1; r <= kMaxRowsPerCta && r * C <= cap; ++r) {
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

namespace {

template <int LANES>
cudaError_t launch_fed(const PrologueArgs& a, const FedGeom& geo, int grid, int smem, cudaStream_t stream) {
  static bool configured[64] = {false};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      e = cudaFuncSetAttribute(prologue_fed_kernel<LANES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               128 + kFedSmemBudget + 16 * kFedMaxStages + 12 * 1024 + 64);
      if (e != cudaSuccess) return e;
      configured[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(geo.T + 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = use_pdl() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, prologue_fed_kernel<LANES>, a, geo);
}

// The bulk-fed variant, if it applies to these arguments (returns false otherwise). In automatic
// mode it is taken only when each CTA streams many blocks: on B200 it beats the direct variant
// in steady state (4.4 vs 4.0 TB/s on 17776 x 12288 rows) but loses on launches of a few blocks
// per SM, where its ring never fills (1.9 vs 2.2 TB/s on 8192 x 1152).
constexpr int64_t kFedMinBlocksPerSm = 32;

bool try_launch_fed(const PrologueArgs& a, cudaStream_t stream, cudaError_t* err) {
  if (a.M <= 0 || a.num_sms <= 0 || a.status == nullptr) return false;
  if (reinterpret_cast<uintptr_t>(a.x) % 16 != 0 || a.ldx % 8 != 0 || a.K % 8 != 0 ||
      reinterpret_cast<uintptr_t>(a.xq) % 16 != 0)
    return false;
  FedGeom geo = fed_geometry(a.n, a.K, a.Kp);
  if (geo.R == 0) return false;
  geo.num_blocks = (a.M + geo.R - 1) / geo.R;
  if (a.variant == 0 && geo.num_blocks < kFedMinBlocksPerSm * a.num_sms) return false;
  geo.vec32 = (reinterpret_cast<uintptr_t>(a.xq) % 32 == 0) ? 1 : 0;
  const int64_t grid = geo.num_blocks < a.num_sms ? geo.num_blocks : a.num_sms;
  const int smem = 128 + geo.stages * geo.stage_bytes + 16 * geo.stages + 12 * geo.R + 16;
  *err = a.n == 64 ? launch_fed<2>(a, geo, static_cast<int>(grid), smem, stream)
                   : launch_fed<4>(a, geo, static_cast<int>(grid), smem, stream);
  return true;
}

}  // namespace

namespace {

// The 64-channel direct kernel: rows of Kp / 64 threads, CTAs of up to k64Threads threads.
constexpr int k64Threads = 256;
constexpr int k64MinBlocks = 3;

cudaError_t launch_prologue64(const PrologueArgs& a, int64_t w_bytes, cudaStream_t stream) {
  const bool weights = a.num_w > 0;
  const int L = a.Kp / 64;
  if (L > k64Threads) return cudaErrorInvalidValue;
  int R = 1, threads = 128;
  int64_t row_ctas = 0;
  if (a.M > 0) {
    R = pick_rows(L, k64Threads);
    threads = ((R * L + 31) / 32) * 32;
    row_ctas = (a.M + R - 1) / R;
  }
  int64_t weight_ctas = 0;
  if (weights) {
    const int64_t per_cta = static_cast<int64_t>(threads) * 32 * kWeightUnroll;
    weight_ctas = (w_bytes + per_cta - 1) / per_cta;
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
    if (vec32) return cudaLaunchKernelEx(&cfg, prologue64_kernel<false, true, k64Threads, k64MinBlocks>, a, R, rc, row_multiplier(L));
    return cudaLaunchKernelEx(&cfg, prologue64_kernel<false, false, k64Threads, k64MinBlocks>, a, R, rc, row_multiplier(L));
  }
  if (vec32) return cudaLaunchKernelEx(&cfg, prologue64_kernel<true, true, k64Threads, k64MinBlocks>, a, R, rc, row_multiplier(L));
  return cudaLaunchKernelEx(&cfg, prologue64_kernel<true, false, k64Threads, k64MinBlocks>, a, R, rc, row_multiplier(L));
}

}  // namespace

cudaError_t launch_prologue_nvfp4(const Nvfp4PrologueArgs& a, cudaStream_t stream) {
  const bool weights = a.w != nullptr;
  if (a.M <= 0 && !weights) return cudaSuccess;
  if (a.Kp % a.n != 0 || (a.n != 64 && a.n != 128) || a.K % 8 != 0) return cudaErrorInvalidValue;
  if (a.M > 0 && (reinterpret_cast<uintptr_t>(a.x) % 16 != 0 || a.ldx % 8 != 0 ||
                  reinterpret_cast<uintptr_t>(a.codes) % 16 != 0 || reinterpret_cast<uintptr_t>(a.sf) % 2 != 0))
    return cudaErrorInvalidValue;
  if (weights && (reinterpret_cast<uintptr_t>(a.w) % 16 != 0 || reinterpret_cast<uintptr_t>(a.w_codes) % 8 != 0 ||
                  a.status == nullptr || a.N <= 0))
    return cudaErrorInvalidValue;
  const int L = a.Kp / 32;
  if (L > kMaxThreads) return cudaErrorInvalidValue;
  // rows of up to 288 threads run in CTAs of at most 288 threads, four per SM; rows of up to
  // 384 threads (K = 12288) one per CTA, three per SM; longer rows take the 512-thread instance
  const bool small = L <= kSmallThreads;
  const bool mid = !small && L <= kMidThreads;
  int R = 1, threads = 256;
  int64_t row_ctas = 0;
  if (a.M > 0) {
    R = pick_rows(L, small ? kSmallThreads : mid ? kMidThreads : kMaxThreads);
    threads = ((R * L + 31) / 32) * 32;
    row_ctas = (a.M + R - 1) / R;
  }
  int64_t weight_ctas = 0;
  if (weights) {
    // one thread per four 16-blocks of a row
    const int64_t quads = static_cast<int64_t>(a.N) * (nvfp4_kp4(a.Kp) / 64);
    if (quads > 0x7fffffffLL) return cudaErrorInvalidValue;
    weight_ctas = (quads + threads - 1) / threads;
    if (weight_ctas > kMaxWeightCtas) weight_ctas = kMaxWeightCtas;
  }
  const int64_t grid = row_ctas + weight_ctas;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
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
  if (small) {
    if (a.n == 64) return cudaLaunchKernelEx(&cfg, prologue_nvfp4_kernel<2, kSmallThreads, 4>, a, R, rc, row_multiplier(L));
    return cudaLaunchKernelEx(&cfg, prologue_nvfp4_kernel<4, kSmallThreads, 4>, a, R, rc, row_multiplier(L));
  }
  if (mid) {
    if (a.n == 64) return cudaLaunchKernelEx(&cfg, prologue_nvfp4_kernel<2, kMidThreads, 3>, a, R, rc, row_multiplier(L));
    return cudaLaunchKernelEx(&cfg, prologue_nvfp4_kernel<4, kMidThreads, 3>, a, R, rc, row_multiplier(L));
  }
  if (a.n == 64) return cudaLaunchKernelEx(&cfg, prologue_nvfp4_kernel<2, kMaxThreads, 1>, a, R, rc, row_multiplier(L));
  return cudaLaunchKernelEx(&cfg, prologue_nvfp4_kernel<4, kMaxThreads, 1>, a, R, rc, row_multiplier(L));
}

cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t stream) {
  const bool weights = a.num_w > 0;
  if (a.M <= 0 && !weights) return cudaSuccess;
  if (a.Kp % a.n != 0 || (a.n != 64 && a.n != 128)) return cudaErrorInvalidValue;
  if (a.num_w < 0 || a.num_w > kMaxWeightSegments) return cudaErrorInvalidValue;
  int64_t w_bytes = 0;
  for (int i = 0; i < a.num_w; ++i) {
    const PrologueArgs::WeightSegment& ws = a.w[i];
    if (ws.bytes % 32 != 0 || reinterpret_cast<uintptr_t>(ws.src) % 32 != 0 ||
        reinterpret_cast<uintptr_t>(ws.dst) % 32 != 0)
      return cudaErrorInvalidValue;
    w_bytes += ws.bytes;
  }
  if (weights && (a.bits_table == nullptr || a.status == nullptr)) return cudaErrorInvalidValue;
  // Rows longer than kSmallThreads 32-channel segments (Kp > 9216) take the 64-channel kernel:
  // with 32 channels a thread a row needs the 512-thread instance at one CTA per SM, with 64 it is
  // 192 threads for K = 12288 and four CTAs share an SM (CogVideoX fc2, 17776 x 12288: 123-132 us
  // against 150-164 for the bulk-fed kernel and 159-173 for the 32-channel one). On shorter rows
  // the 64-channel kernel ran level with the 32-channel one or behind it.
  if (a.variant == 3 || (a.variant == 0 && a.M > 0 && a.Kp / 32 > kSmallThreads))
    return launch_prologue64(a, w_bytes, stream);
  if (a.variant == 0 || a.variant == 2) {
    cudaError_t e = cudaSuccess;
    if (try_launch_fed(a, stream, &e)) return e;
  }
  const int L = a.Kp / 32;
  if (L > kMaxThreads) return cudaErrorInvalidValue;
  int R = 1, threads = 256;
  int64_t row_ctas = 0;
  // rows of up to 384 threads run in CTAs of at most 384 threads with 56 registers each, so four
  // CTAs share an SM; longer rows take the 512-thread instance
  const bool small = L <= kSmallThreads;
  if (a.M > 0) {
    R = pick_rows(L, small ? kSmallThreads : kMaxThreads);
    threads = ((R * L + 31) / 32) * 32;
    row_ctas = (a.M + R - 1) / R;
  }
  int64_t weight_ctas = 0;
  if (weights) {
    // about kWeightUnroll 32-byte loads per thread; larger layers loop
    const int64_t per_cta = static_cast<int64_t>(threads) * 32 * kWeightUnroll;
    weight_ctas = (w_bytes + per_cta - 1) / per_cta;
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
  if (small) {
    if (a.n == 64) {
      if (vec32) return cudaLaunchKernelEx(&cfg, prologue_kernel<2, true, kSmallThreads, 4>, a, R, rc, row_multiplier(L));
      return cudaLaunchKernelEx(&cfg, prologue_kernel<2, false, kSmallThreads, 4>, a, R, rc, row_multiplier(L));
    }
    if (vec32) return cudaLaunchKernelEx(&cfg, prologue_kernel<4, true, kSmallThreads, 4>, a, R, rc, row_multiplier(L));
    return cudaLaunchKernelEx(&cfg, prologue_kernel<4, false, kSmallThreads, 4>, a, R, rc, row_multiplier(L));
  }
  if (a.n == 64) {
    if (vec32) return cudaLaunchKernelEx(&cfg, prologue_kernel<2, true, kMaxThreads, 1>, a, R, rc, row_multiplier(L));
    return cudaLaunchKernelEx(&cfg, prologue_kernel<2, false, kMaxThreads, 1>, a, R, rc, row_multiplier(L));
  }
  if (vec32) return cudaLaunchKernelEx(&cfg, prologue_kernel<4, true, kMaxThreads, 1>, a, R, rc, row_multiplier(L));
  return cudaLaunchKernelEx(&cfg, prologue_kernel<4, false, kMaxThreads, 1>, a, R, rc, row_multiplier(L));
}

}  // namespace tasq
