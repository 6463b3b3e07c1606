// Launch interfaces shared by the C-ABI layer and the kernel translation units.
#pragma once

#include <cstdint>
#include <string>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/tasq.h"

namespace tasq {

// Activation prologue: block Hadamard along K, per-token absmax, RNE INT8 codes.
constexpr int kMaxWeightSegments = 4;   // layers one prologue launch can mask (= TASQ_GROUP_MAX)

struct PrologueArgs {
  const void* x;      // FP16 [M, K], row stride ldx elements
  int64_t ldx;
  int32_t K;          // multiple of 8
  int32_t Kp;         // ceil(K / n) * n
  int64_t M;
  int8_t* xq;         // [M, Kp]
  float* s_x;         // [M]
  int32_t n;          // 64 or 128
  float sx_factor;    // fp32(1 / (127 sqrt(n)))
  // Optional weight pass in the same launch (num_w > 0): for each segment, dst = src AND the
  // byte mask 0xFF << (8 - bits), bits = bits_table[bits_index]; out-of-range bits set
  // TASQ_DEVICE_BAD_BITS in *status and are read as 8. Buffers 32-byte aligned, bytes a
  // multiple of 32.
  struct WeightSegment {
    const int8_t* src;
    int8_t* dst;
    int64_t bytes;
    int32_t bits_index;
  };
  int32_t num_w;
  WeightSegment w[kMaxWeightSegments];
  const uint8_t* bits_table;
  // Always set: receives TASQ_DEVICE_BAD_BITS and, when a bounded wait of the bulk-fed variant
  // gives up after wait_limit_ns, TASQ_DEVICE_TIMEOUT_PROLOGUE.
  uint32_t* status;
  uint64_t wait_limit_ns;
  int32_t num_sms;
  int32_t variant;    // 0: bulk-fed for long launches, else direct; 1: always direct;
                      // 2: bulk-fed wherever its layout fits
  int32_t gate;       // kGateNone, or kGateInt8: the launch steps aside when the schedule entry
  int32_t gate_index; //   bits_table[gate_index] is 0 (an NVFP4 step decided on the device)
};
// Launches the activation rows (M > 0) and the weight pass (num_w > 0) as one grid; either
// part may be empty.
cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t stream);

// Gated launches. When the on-device predictor may pick either format for a (layer, step), a
// forward launches both the INT8 and the NVFP4 kernels; each reads the schedule entry first and,
// if the step is not its format, waits for the kernel before it (so the launches after it still
// see that kernel's results) and returns without touching memory.
constexpr int32_t kGateNone = 0;
constexpr int32_t kGateInt8 = 1;    // run only if the entry is 1..8
constexpr int32_t kGateNvfp4 = 2;   // run only if the entry is 0
__device__ __forceinline__ bool gated_out(int32_t gate, const uint8_t* table, int32_t index) {
  if (gate == kGateNone) return false;
  const bool nvfp4 = table[index] == 0;
  const bool skip = gate == kGateInt8 ? nvfp4 : !nvfp4;
  if (skip) asm volatile("griddepcontrol.wait;" ::: "memory");
  return skip;
}

// NVFP4 step (6Bit-Diffusion's stable layers): E2M1 codes with one UE4M3 scale per 16 elements
// along K. Block scales live in 512-byte chunks, one per 128 rows x 64 elements of K; chunk
// (row / 128) * sf_chunks + k / 64 holds the scale of row r, 16-block j of those 64 at byte
// (r % 32) * 16 + ((r % 128) / 32) * 4 + j (the layout tcgen05.cp 32x128b.warpx4 moves into the
// tensor memory the block-scaled MMA reads). sf_chunks = Kp4 / 64 with Kp4 = Kp rounded up to
// 256, the K of one GEMM stage; chunks past Kp hold zero scales.
constexpr int kNvfp4Block = 16;
constexpr int kNvfp4Kp4 = 256;
constexpr int kNvfp4ChunkBytes = 512;
constexpr float kNvfp4Range = 2688.0f;   // 6 (largest E2M1) * 448 (largest E4M3)
__host__ __device__ inline int64_t nvfp4_kp4(int64_t Kp) { return (Kp + kNvfp4Kp4 - 1) / kNvfp4Kp4 * kNvfp4Kp4; }
__host__ __device__ inline int64_t nvfp4_sf_bytes(int64_t rows, int64_t Kp) {
  return (rows + 127) / 128 * (nvfp4_kp4(Kp) / 64) * kNvfp4ChunkBytes;
}
struct Nvfp4PrologueArgs {
  // activations: x FP16 [M, K] (row stride ldx) -> codes [M, Kp / 2], scales, s_x [M]
  const void* x;
  int64_t ldx;
  int32_t K, Kp, n;
  int64_t M;
  uint8_t* codes;
  uint8_t* sf;
  float* s_x;
  float sx_factor;     // fp32(1 / (2688 sqrt(n)))
  // optional weight conversion in the same launch: the shared INT8 weights [N, Kp] of one layer
  // -> NVFP4 codes [N, Kp / 2] and scales; the schedule entry bits_table[bits_index] must be 0
  // (no check when bits_table is null)
  const int8_t* w;
  uint8_t* w_codes;
  uint8_t* w_sf;
  int32_t N;
  const uint8_t* bits_table;
  int32_t bits_index;
  uint32_t* status;
  // gating (see gated_out): kGateNvfp4 makes the whole launch step aside unless
  // gate_table[gate_index] is 0
  int32_t gate;
  const uint8_t* gate_table;
  int32_t gate_index;
};
cudaError_t launch_prologue_nvfp4(const Nvfp4PrologueArgs& a, cudaStream_t stream);


enum class OutKind : int { F16 = 0, BF16 = 1, S32 = 2 };

// DMPQ precision predictor: Gamma = ||out - in||_1 / ||in||_1 over FP16 [M, D] (D % 8 == 0,
// rows 16-byte aligned), then table[entries[i]] = Gamma > tau ? bits_unstable : bits_stable.
constexpr int kDmpqMaxEntries = 32;
constexpr int kDmpqCtasPerSm = 2;
struct DmpqArgs {
  const void* in;
  const void* out;
  int64_t ld_in, ld_out;   // row strides in elements
  int64_t M;
  int32_t D;
  double tau;
  int32_t bits_unstable, bits_stable;
  uint8_t* table;
  int32_t num_entries;
  int32_t entries[kDmpqMaxEntries];   // indices into the schedule table
  double* gamma_out;                  // optional
};
int dmpq_partial_ctas(int64_t M, int32_t D, int num_sms);
// One launch on `stream`; `partial` holds 4 * dmpq_partial_ctas(...) uint64 values, and
// `arrived` is a zeroed counter that the launch leaves zeroed again.
cudaError_t launch_dmpq(const DmpqArgs& a, uint64_t* partial, unsigned int* arrived, int num_sms,
                        cudaStream_t stream);

// Masked INT8 GEMM: y[m, c] = sum_k xq[m, k] * mask(w[c, k]) (* s_x[m] * s_w[c]).
struct GemmArgs {
  int32_t M;
  int32_t N;
  int32_t num_kb;          // ceil(Kp / 128)
  int32_t num_m_tiles;     // ceil(M / 256)
  int32_t num_n_tiles;     // ceil(N / 128)
  const uint8_t* bits_table;
  int32_t bits_index;      // layer * num_steps + step
  const float* s_x;
  const float* s_w;
  void* y;
  int64_t ldy;
  uint32_t* status;
  uint64_t wait_limit_ns;
  int32_t premasked;       // 1: the weight operand already holds mask(w) for this bit width
  int32_t gate;            // kGateNone, kGateInt8 or kGateNvfp4 (see gated_out), on bits_table[bits_index]
  int32_t band_tiles;      // token tiles per band of the tile order (gemm_band_tiles), >= 1
};
// Token tiles per band of a GEMM's tile order (tile_coords): 8, or all token tiles when fewer, and
// never 0.
int32_t gemm_band_tiles(int64_t num_m_tiles, int64_t tile_tok, int64_t code_row_bytes);
cudaError_t launch_masked_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const CUtensorMap& tmap_y,
                               const GemmArgs& g, OutKind out, int num_sms, cudaStream_t stream);

// Block-scaled NVFP4 GEMM (tcgen05 kind::mxf4nvf4), tiles of 128 channels x 128 tokens; tmap_w and
// tmap_x cover the E2M1 codes as bytes ([N, Kp / 2] and [M, Kp / 2], boxes of 128 x 128 bytes),
// g.num_kb = Kp4 / 256 stages, the scales in the chunked layout above (16-byte aligned). The
// accumulators are FP32; OutKind::S32 writes their raw bits. g.bits_table may be null (no check).
struct Nvfp4GemmArgs {
  const uint8_t* w_sf;
  const uint8_t* x_sf;
  int32_t sf_chunks;   // Kp4 / 64 = 4 * g.num_kb
};
cudaError_t launch_gemm_nvfp4(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const CUtensorMap& tmap_y,
                              const GemmArgs& g, const Nvfp4GemmArgs& f, OutKind out, int num_sms,
                              cudaStream_t stream);

// The NVFP4 GEMM over CTA pairs (tcgen05 cta_group::2): tiles of 256 channels x 192 tokens, each
// CTA holding 128 weight rows and 96 token rows per stage (tensor-map boxes of 128 x 128 and
// 96 x 128 bytes), g.num_m_tiles = ceil(M / 192), g.num_n_tiles = ceil(N / 256); the scales in
// the same chunked layout as launch_gemm_nvfp4.
constexpr int kGemmNvfp4PairTok = 192;   // tokens per NVFP4 pair tile
cudaError_t launch_gemm_nvfp4_pair(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const CUtensorMap& tmap_y,
                                   const GemmArgs& g, const Nvfp4GemmArgs& f, OutKind out, int num_sms,
                                   cudaStream_t stream);
// Whether the automatic choice runs an NVFP4 GEMM of M tokens and N channels on CTA pairs
// (defined in tasq_api.cu).
bool nvfp4_use_pair(int64_t M, int64_t N, int num_sms);

// The same GEMM over CTA pairs (tcgen05 cta_group::2): tiles of 256 channels x 256 tokens, each
// CTA holding 128 rows of each operand (tensor-map boxes of 128 x 128 bytes for both).
cudaError_t launch_masked_gemm_pair(const CUtensorMap& tmap_w, const CUtensorMap& tmap_x, const CUtensorMap& tmap_y,
                                    const GemmArgs& g, OutKind out, int num_sms, cudaStream_t stream);
constexpr int kGemmPairTile = 256;  // channels and tokens per pair tile
constexpr int kGemmPairHalf = 128;  // operand rows per CTA of a pair

// Geometry of the GEMM tiles (for the host's tensor maps).
constexpr int kGemmTileCh = 128;    // weight rows per tile
constexpr int kGemmTileTok = 256;   // activation rows per tile
constexpr int kGemmBlockK = 128;    // K bytes per pipeline stage
constexpr int kGemmStoreBox = 32;   // outputs leave in 32 x 32 TMA store boxes

// Whether the automatic choice runs a GEMM of M tokens and N channels on CTA pairs rather than
// one CTA per tile (defined in tasq_api.cu, with the measurements behind it).
bool gemm_use_pair(int64_t M, int64_t N, int num_sms);

cudaError_t launch_stuck_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t stream);

// Whether kernels are launched with programmatic dependent launch, so that a kernel's setup
// overlaps the tail of the previous kernel on the stream (environment TASQ_PDL=0 turns it off).
bool use_pdl();

// Host helpers shared by the entry points (defined in tasq_api.cu).
extern thread_local std::string g_last_error;
void set_last_error(const std::string& msg);
tasq_status fail(tasq_status st, const std::string& msg);
tasq_status fail_cuda(cudaError_t e, const char* what);
bool aligned16(const void* p);
size_t round_up(size_t v, size_t a);
// UINT8 [rows, cols] tensor (row stride cols bytes) read in 128-byte-swizzled boxes.
tasq_status make_tmap_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                         uint32_t box_rows);
// Output tensor [rows, cols] (row stride ld elements) written in 32 x 32 boxes (64-byte swizzled
// staging for 2-byte elements, plain for 4-byte ones).
tasq_status make_tmap_out(CUtensorMap* m, void* base, CUtensorMapDataType dt, uint32_t elem_bytes, uint64_t cols,
                          uint64_t rows, uint64_t ld);

}  // namespace tasq
