// On-device DMPQ precision predictor (6Bit-Diffusion technical summary, section 2.A,
// "Quantizacao de Precisao Mista Dinamica (DMPQ)"): the relative L1 distance between a block's
// input and output at step t-1, Gamma = ||out - in||_1 / ||in||_1, decides the bit width of the
// block's linears at step t. Unstable blocks (Gamma > tau) keep the wide width, stable ones get
// the narrow one. The decision is written straight into the device schedule table, with no
// host round trip.
//
// Every FP16 value is an integer number of 2^-24 units (the smallest subnormal), so both L1
// sums can be taken exactly. Each thread adds its terms in FP64, which is exact here: every
// term and every partial sum is a multiple of 2^-24, and a thread flushes after at most 4096
// terms, so no sum reaches 4096 * 131008 < 2^29 (53 - 24 bits). Each flush converts the FP64
// sum to an integer count of 2^-24 units and adds it to a 64-bit integer (at most 2^21 terms of
// below 2^41 units per thread). CTAs and the final sum add in 128-bit integers. The result does not
// depend on the grid or on the order of the additions. Gamma is the IEEE double quotient of the two
// sums, each rounded once to nearest-even, which is what the CPU oracle computes.
//
// One launch: every CTA streams its share of the two tensors once (HBM-bound, 4 bytes per
// element) into a 128-bit partial sum; the last CTA to finish adds the partials, divides, and
// writes the bits for every listed table entry (and Gamma, if asked).
#include <cuda_runtime.h>

#include <cuda_fp16.h>

#include <cstdint>

#include "tasq_internal.h"

namespace tasq {
namespace {

typedef unsigned __int128 u128;

constexpr int kPartialThreads = 256;

__device__ __forceinline__ uint4 ld_nc_16B(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 32 bytes in one load (rows and pointers 32-byte aligned).
__device__ __forceinline__ void ld_nc_32B(const void* p, uint32_t (&u)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
               : "l"(p));
}

template <int VE>
__device__ __forceinline__ void ld_vec(const void* p, uint32_t (&u)[VE / 2]) {
  if constexpr (VE == 16) {
    ld_nc_32B(p, u);
  } else {
    const uint4 v = ld_nc_16B(p);
    u[0] = v.x;
    u[1] = v.y;
    u[2] = v.z;
    u[3] = v.w;
  }
}

__device__ __forceinline__ u128 shfl_down_u128(u128 v, int off) {
  const uint64_t lo = __shfl_down_sync(0xffffffffu, static_cast<uint64_t>(v), off);
  const uint64_t hi = __shfl_down_sync(0xffffffffu, static_cast<uint64_t>(v >> 64), off);
  return (static_cast<u128>(hi) << 64) | lo;
}

// FP16 bit pattern (low 16 bits) to FP64, exact.
__device__ __forceinline__ double f16_to_f64(uint32_t bits) {
  double d;
  const unsigned short h = static_cast<unsigned short>(bits);
  asm("cvt.f64.f16 %0, %1;" : "=d"(d) : "h"(h));
  return d;
}

constexpr int kFlushElems = 4096;    // terms a thread adds in FP64 between integer flushes
// 32-byte vectors of each tensor per batch (16-byte vectors: twice as many), two batches in flight
// per thread, two 256-thread CTAs per SM: 128 bytes of each tensor in registers per thread. Timed
// against 32-byte batches at four CTAs per SM and the single-batch loop: fastest on 8192 x 1152
// (12.7 vs 13.9 and 14.7 us), within 4 % on 17776 x 3072, and fastest inside the CogVideoX step.
constexpr int kBatch16 = 2;

__device__ __forceinline__ void add_units(uint64_t& acc, double sum) {
  acc += static_cast<uint64_t>(__double2ll_rn(sum * 16777216.0));   // exact: an integer of units
}

// One pass over in and out ([M, D] FP16, row strides ld_in / ld_out elements, D % VE == 0, VE
// elements a load): partial[cta] = {num lo, num hi, den lo, den hi} in 2^-24 units,
// num = sum |out - in|, den = sum |in|.
__device__ void finish(const DmpqArgs& a, const uint64_t* partial, int num_partials);

// NB vectors of each tensor per batch; two batches alternate, so that the loads of the next
// batch are in flight while the current one is summed.
template <int VE, int NB>
struct Batch {
  uint32_t wi[NB][VE / 2], wo[NB][VE / 2];
};

// This thread's walk over the vectors (row, col), vector index thread, thread + stride, ...;
// it ends at row M. M < 2^31 is checked on the host, and a row passes M by at most stride_rows + 1
// < 2^18, so the unsigned row never wraps; vector columns stay below 2 * D / 8.
struct Cursor {
  uint32_t row, M;
  int32_t col, vpr, stride_rows, stride_cols;
  __device__ __forceinline__ bool more() const { return row < M; }
  __device__ __forceinline__ void advance() {
    row += stride_rows;
    col += stride_cols;
    if (col >= vpr) {
      col -= vpr;
      ++row;
    }
  }
};

template <int VE, int NB>
__device__ __forceinline__ void load_batch(const DmpqArgs& a, Cursor& c, Batch<VE, NB>& b) {
#pragma unroll
  for (int u = 0; u < NB; ++u) {
    if (c.more()) {
      ld_vec<VE>(static_cast<const __half*>(a.in) + static_cast<int64_t>(c.row) * a.ld_in + VE * c.col, b.wi[u]);
      ld_vec<VE>(static_cast<const __half*>(a.out) + static_cast<int64_t>(c.row) * a.ld_out + VE * c.col, b.wo[u]);
      c.advance();
    } else {
#pragma unroll
      for (int i = 0; i < VE / 2; ++i) b.wi[u][i] = b.wo[u][i] = 0u;   // zero terms add nothing
    }
  }
}

template <int VE, int NB>
__device__ __forceinline__ void add_batch(const Batch<VE, NB>& b, double& fnum, double& fden) {
#pragma unroll
  for (int u = 0; u < NB; ++u) {
#pragma unroll
    for (int i = 0; i < VE / 2; ++i) {
      const double i0 = f16_to_f64(b.wi[u][i] & 0xFFFFu), i1 = f16_to_f64(b.wi[u][i] >> 16);
      const double o0 = f16_to_f64(b.wo[u][i] & 0xFFFFu), o1 = f16_to_f64(b.wo[u][i] >> 16);
      fnum += fabs(o0 - i0) + fabs(o1 - i1);   // every step exact (see the header)
      fden += fabs(i0) + fabs(i1);
    }
  }
}

template <int VE, int NB, int MINB>
__global__ void __launch_bounds__(kPartialThreads, MINB)
    dmpq_partial_kernel(const DmpqArgs a, uint64_t* __restrict__ partial, unsigned int* __restrict__ arrived) {
  constexpr int kBatchElems = NB * VE;
  static_assert(kFlushElems % kBatchElems == 0, "flush on a batch boundary");
  Cursor c;
  c.M = static_cast<uint32_t>(a.M);
  c.vpr = a.D / VE;                                     // vectors per row
  const int32_t stride = static_cast<int32_t>(gridDim.x * blockDim.x);
  c.stride_rows = stride / c.vpr;
  c.stride_cols = stride - c.stride_rows * c.vpr;
  const int32_t v = static_cast<int32_t>(blockIdx.x * blockDim.x + threadIdx.x);
  c.row = static_cast<uint32_t>(v / c.vpr);             // advanced incrementally below
  c.col = v - static_cast<int32_t>(c.row) * c.vpr;
  uint64_t num = 0, den = 0;
  double fnum = 0.0, fden = 0.0;
  int since_flush = 0;                                  // terms since the last flush
  auto count = [&]() {
    since_flush += kBatchElems;
    if (since_flush >= kFlushElems) {
      add_units(num, fnum);
      add_units(den, fden);
      fnum = fden = 0.0;
      since_flush = 0;
    }
  };
  Batch<VE, NB> b0, b1;
  load_batch(a, c, b0);
  for (;;) {
    const bool more0 = c.more();
    if (more0) load_batch(a, c, b1);
    add_batch(b0, fnum, fden);
    count();
    if (!more0) break;
    const bool more1 = c.more();
    if (more1) load_batch(a, c, b0);
    add_batch(b1, fnum, fden);
    count();
    if (!more1) break;
  }
  add_units(num, fnum);
  add_units(den, fden);
  u128 n = num, dd = den;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    n += shfl_down_u128(n, off);
    dd += shfl_down_u128(dd, off);
  }
  __shared__ u128 warp_num[kPartialThreads / 32], warp_den[kPartialThreads / 32];
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    warp_num[warp] = n;
    warp_den[warp] = dd;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    u128 tn = 0, td = 0;
    for (int w = 0; w < kPartialThreads / 32; ++w) {
      tn += warp_num[w];
      td += warp_den[w];
    }
    uint64_t* p = partial + 4 * static_cast<int64_t>(blockIdx.x);
    p[0] = static_cast<uint64_t>(tn);
    p[1] = static_cast<uint64_t>(tn >> 64);
    p[2] = static_cast<uint64_t>(td);
    p[3] = static_cast<uint64_t>(td >> 64);
  }
  // the last CTA to arrive adds the partials (the others' writes are visible after their fence
  // and the counter's atomic order) and resets the counter for the next call on the stream
  __shared__ bool last;
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(arrived, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (threadIdx.x < 32) finish(a, partial, gridDim.x);
  if (threadIdx.x == 0) *arrived = 0u;
}

// Round a 128-bit unsigned integer to the nearest double, ties to even.
__device__ __forceinline__ double u128_to_double_rn(u128 v) {
  const uint64_t hi = static_cast<uint64_t>(v >> 64);
  const uint64_t lo = static_cast<uint64_t>(v);
  if (hi == 0 && lo < (1ull << 53)) return static_cast<double>(lo);   // exact
  const int msb = hi != 0 ? 127 - __clzll(static_cast<long long>(hi)) : 63 - __clzll(static_cast<long long>(lo));
  const int shift = msb - 52;                       // bits below the 53-bit significand
  u128 mant = v >> shift;
  const u128 rem = v & ((static_cast<u128>(1) << shift) - 1);
  const u128 half = static_cast<u128>(1) << (shift - 1);
  if (rem > half || (rem == half && (mant & 1))) mant += 1;   // mant <= 2^53: still exact below
  return scalbn(static_cast<double>(static_cast<uint64_t>(mant)), shift);
}

// Run by the 32 threads of warp 0 of the last CTA.
__device__ void finish(const DmpqArgs& a, const uint64_t* partial, int num_partials) {
  u128 n = 0, d = 0;
  for (int i = threadIdx.x; i < num_partials; i += 32) {
    const volatile uint64_t* p = partial + 4 * static_cast<int64_t>(i);
    n += (static_cast<u128>(p[1]) << 64) | p[0];
    d += (static_cast<u128>(p[3]) << 64) | p[2];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    n += shfl_down_u128(n, off);
    d += shfl_down_u128(d, off);
  }
  if (threadIdx.x != 0) return;
  double gamma;
  bool unstable;
  if (d == 0) {
    // no input magnitude: no information, keep the wide width
    gamma = n > 0 ? __longlong_as_double(0x7FF0000000000000ll) : 0.0;
    unstable = true;
  } else {
    gamma = __ddiv_rn(u128_to_double_rn(n), u128_to_double_rn(d));
    unstable = gamma > a.tau;
  }
  const uint8_t bits = static_cast<uint8_t>(unstable ? a.bits_unstable : a.bits_stable);
  for (int i = 0; i < a.num_entries; ++i) a.table[a.entries[i]] = bits;
  if (a.gamma_out != nullptr) *a.gamma_out = gamma;
}

}  // namespace

int dmpq_partial_ctas(int64_t M, int32_t D, int num_sms) {
  const int64_t vecs = M * (D / 8);
  int64_t ctas = (vecs + kPartialThreads * 4 - 1) / (kPartialThreads * 4);
  const int64_t cap = static_cast<int64_t>(num_sms) * kDmpqCtasPerSm;
  if (ctas > cap) ctas = cap;
  if (ctas < 1) ctas = 1;
  return static_cast<int>(ctas);
}

cudaError_t launch_dmpq(const DmpqArgs& a, uint64_t* partial, unsigned int* arrived, int num_sms,
                        cudaStream_t stream) {
  const int ctas = dmpq_partial_ctas(a.M, a.D, num_sms);
  // 32-byte loads where every row starts on a 32-byte boundary, else 16-byte ones
  const bool vec32 = a.D % 16 == 0 && a.ld_in % 16 == 0 && a.ld_out % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(a.in) % 32 == 0 && reinterpret_cast<uintptr_t>(a.out) % 32 == 0;
  if (vec32)
    dmpq_partial_kernel<16, kBatch16, kDmpqCtasPerSm><<<ctas, kPartialThreads, 0, stream>>>(a, partial, arrived);
  else
    dmpq_partial_kernel<8, 2 * kBatch16, kDmpqCtasPerSm><<<ctas, kPartialThreads, 0, stream>>>(a, partial, arrived);
  return cudaGetLastError();
}

}  // namespace tasq
