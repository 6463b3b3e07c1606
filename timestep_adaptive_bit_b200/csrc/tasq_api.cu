// C ABI of the masked INT8 linear: context (one shared weight buffer, device schedule table,
// activation workspace), argument validation, TMA descriptors and kernel launches.
#include <cudaTypedefs.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/tasq.h"
#include "tasq_internal.h"

namespace tasq {

thread_local std::string g_last_error;

void set_last_error(const std::string& msg) { g_last_error = msg; }


tasq_status fail(tasq_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

tasq_status fail_cuda(cudaError_t e, const char* what) {
  std::string m = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return fail(TASQ_ERR_CUDA, m);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool use_pdl() {
  static const bool on = [] {
    const char* v = std::getenv("TASQ_PDL");
    return v == nullptr || std::string(v) != "0";
  }();
  return on;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D UINT8 tensor [rows, cols] with row stride `cols` bytes, loaded in boxes of
// box_cols x box_rows with 128-byte swizzle; out-of-range elements read as zero.
tasq_status make_tmap_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                         uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(TASQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TASQ_ERR_CUDA, "cuTensorMapEncodeTiled failed with CUresult " + std::to_string(r));
  return TASQ_OK;
}

// 2-D output tensor [rows, cols] (element type `dt`, row stride `ld` elements) written in
// boxes of 32 x 32 by TMA stores; elements outside [rows, cols] are never written. 16-bit boxes
// are read from shared memory with the 64-byte swizzle the epilogue writes them in.
tasq_status make_tmap_out(CUtensorMap* m, void* base, CUtensorMapDataType dt, uint32_t elem_bytes, uint64_t cols,
                          uint64_t rows, uint64_t ld) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(TASQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * elem_bytes};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(tasq::kGemmStoreBox), static_cast<cuuint32_t>(tasq::kGemmStoreBox)};
  const cuuint32_t estr[2] = {1, 1};
  // 16-bit outputs are staged in 64-byte swizzled boxes (32 channels x 2 bytes per row), 32-bit
  // outputs in plain ones
  const CUtensorMapSwizzle sw = elem_bytes == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(m, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(TASQ_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed with CUresult " + std::to_string(r));
  return TASQ_OK;
}

}  // namespace tasq

namespace {

using tasq::fail;
using tasq::fail_cuda;
using tasq::aligned16;
using tasq::round_up;
using tasq::make_tmap_u8;
using tasq::make_tmap_out;
using tasq::g_last_error;

struct LayerInfo {
  int32_t N, K, Kp;
  size_t w_off;    // bytes into the weight buffer
  size_t sw_off;   // floats into the scale buffer
};

struct TraceRec {
  cudaEvent_t e0, e1, e2;
  double ops, bytes, wbytes;   // GEMM ops, prologue activation bytes, weight-pass bytes
};

}  // namespace

struct tasq_ctx {
  int device = -1;
  int num_sms = 0;
  int32_t num_layers = 0, num_steps = 0, n = 0, out_dtype = 0;
  int64_t max_tokens = 0;
  int32_t kp_max = 0;
  std::vector<LayerInfo> layers;
  std::vector<CUtensorMap> tmap_w;
  int8_t* d_w = nullptr;
  float* d_sw = nullptr;
  uint8_t* d_bits = nullptr;
  int8_t* d_xq = nullptr;               // INT8 codes [M, Kp], or NVFP4 codes [M, Kp / 2]
  uint8_t* d_sf4 = nullptr;             // NVFP4 block scales of the activations (chunked layout)
  float* d_sx = nullptr;
  uint32_t* d_status = nullptr;
  uint64_t* d_dmpq = nullptr;          // per-CTA partial sums of the DMPQ predictor
  unsigned int* d_dmpq_arrived = nullptr;   // its CTA arrival counter (zero between calls)
  uint64_t wait_limit_ns = 1000000000ull;
  float sx_factor = 0.0f;
  float sx_factor4 = 0.0f;              // NVFP4: fp32(1 / (2688 sqrt(n)))
  int32_t gemm_mode = 0;   // 0 automatic, 1 one CTA per tile, 2 CTA pairs
  int32_t mask_mode = 0;   // 0 and 1: in the GEMM, in shared memory; 2: ahead in the prologue launch,
                           // into a masked copy
  int32_t prologue_mode = 0;   // 0 automatic, 1 direct-load prologue, 2 bulk-fed prologue where it fits,
                               // 3 direct-load prologue with 64 channels a thread
  // host copy of the last schedule given, used only to choose where the mask is applied: both
  // places read the device table and give the same result for every bit width, so a device table
  // that is newer or older than this copy changes no result
  std::vector<uint8_t> bits_host;
  // entries the on-device predictor may have set to either an INT8 width (kept in bits_host) or
  // NVFP4: forwards of such an entry launch both paths, gated on the device table
  std::vector<uint8_t> maybe_nvfp4;
  int8_t* d_wk = nullptr;              // masked copies: wk_slots slots of wk_slot_bytes each
  size_t wk_slot_bytes = 0;            // largest N x Kp, rounded up to 1024
  int32_t wk_slots = 0;                // min(num_layers, TASQ_GROUP_MAX)
  std::vector<CUtensorMap> tmap_wk;    // per layer, over slot 0
  // trace
  int32_t trace_cap = 0, trace_count = 0;
  std::vector<TraceRec> trace;
};

namespace {

void free_ctx(tasq_ctx* c) {
  if (c == nullptr) return;
  if (c->device >= 0) cudaSetDevice(c->device);
  cudaDeviceSynchronize();
  cudaFree(c->d_w);
  cudaFree(c->d_wk);
  cudaFree(c->d_sw);
  cudaFree(c->d_bits);
  cudaFree(c->d_xq);
  cudaFree(c->d_sf4);
  cudaFree(c->d_sx);
  cudaFree(c->d_status);
  cudaFree(c->d_dmpq);
  cudaFree(c->d_dmpq_arrived);
  for (auto& t : c->trace) {
    cudaEventDestroy(t.e0);
    cudaEventDestroy(t.e1);
    cudaEventDestroy(t.e2);
  }
  delete c;
}

tasq_status check_device(const tasq_ctx* c) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  if (dev != c->device)
    return fail(TASQ_ERR_INVALID_ARG, "current device " + std::to_string(dev) + " is not the context's device " +
                                          std::to_string(c->device));
  return TASQ_OK;
}

tasq_status check_layer(const tasq_ctx* c, int32_t layer) {
  if (layer < 0 || layer >= c->num_layers)
    return fail(TASQ_ERR_INVALID_ARG, "layer " + std::to_string(layer) + " out of range [0, " +
                                          std::to_string(c->num_layers) + ")");
  return TASQ_OK;
}

tasq_status check_step(const tasq_ctx* c, int32_t step) {
  if (step < 0 || step >= c->num_steps)
    return fail(TASQ_ERR_INVALID_ARG,
                "step " + std::to_string(step) + " out of range [0, " + std::to_string(c->num_steps) + ")");
  return TASQ_OK;
}

tasq_status check_tokens(const tasq_ctx* c, int64_t M) {
  if (M < 0) return fail(TASQ_ERR_INVALID_ARG, "M must be >= 0");
  if (M > c->max_tokens)
    return fail(TASQ_ERR_WORKSPACE,
                "M = " + std::to_string(M) + " exceeds max_tokens = " + std::to_string(c->max_tokens));
  return TASQ_OK;
}

tasq_status check_rows(const void* p, int64_t ld, int64_t width, const char* name) {
  if (p == nullptr) return fail(TASQ_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (!aligned16(p)) return fail(TASQ_ERR_INVALID_ARG, std::string(name) + " is not 16-byte aligned");
  if (ld < width || ld % 8 != 0)
    return fail(TASQ_ERR_INVALID_ARG, std::string("row stride of ") + name + " must be >= " + std::to_string(width) +
                                          " and a multiple of 8, got " + std::to_string(ld));
  return TASQ_OK;
}

// Whether this forward masks the layer's weights once in the prologue launch, into a masked copy
// that the GEMM then loads (mask mode 2, kept to measure against). Otherwise the GEMM's mask warps
// clear the step's low bit planes of every weight tile of the one stored buffer in shared memory, as
// it lands, whenever the device table drops bits, and no copy of the weights exists.
bool mask_ahead(const tasq_ctx* c, int32_t /*layer*/, int32_t /*step*/) { return c->mask_mode == 2; }

int8_t* wk_slot(const tasq_ctx* c, int32_t slot) { return c->d_wk + static_cast<size_t>(slot) * c->wk_slot_bytes; }

// Add (layer, step) to the prologue launch's weight pass, masked into slot `slot`.
void add_weight_pass(tasq::PrologueArgs& a, const tasq_ctx* c, int32_t layer, int32_t step, int32_t slot) {
  const LayerInfo& L = c->layers[layer];
  tasq::PrologueArgs::WeightSegment& ws = a.w[a.num_w++];
  ws.src = c->d_w + L.w_off;
  ws.dst = wk_slot(c, slot);
  ws.bytes = static_cast<int64_t>(L.N) * L.Kp;
  ws.bits_index = layer * c->num_steps + step;
  a.bits_table = c->d_bits;
  a.status = c->d_status;
}

// Activation prologue of (layer, step) over M rows (M may be 0), with the weight pass when
// `weights` is set.
// `masked` lists up to kMaxWeightSegments layers whose weights the same launch masks, layer
// masked[i] into masked-weight slot i.
tasq_status run_prologue(tasq_ctx* c, int32_t layer, int32_t step, const std::vector<int32_t>& masked, const void* x,
                         int64_t M, int64_t ldx, int8_t* xq, float* sx, cudaStream_t s,
                         int32_t gate = tasq::kGateNone) {
  const LayerInfo& L = c->layers[layer];
  tasq::PrologueArgs a{};
  for (size_t i = 0; i < masked.size(); ++i) add_weight_pass(a, c, masked[i], step, static_cast<int32_t>(i));
  a.x = x;
  a.ldx = ldx;
  a.K = L.K;
  a.Kp = L.Kp;
  a.M = M;
  a.xq = xq;
  a.s_x = sx;
  a.n = c->n;
  a.sx_factor = c->sx_factor;
  a.status = c->d_status;
  a.wait_limit_ns = c->wait_limit_ns;
  a.num_sms = c->num_sms;
  a.variant = c->prologue_mode;
  a.bits_table = c->d_bits;
  a.gate = gate;
  a.gate_index = layer * c->num_steps + step;
  g_last_error.clear();
  cudaError_t e = tasq::launch_prologue(a, s);
  if (e != cudaSuccess) {
    if (!g_last_error.empty()) return fail(TASQ_ERR_CUDA, "prologue launch: " + g_last_error);
    return fail_cuda(e, "prologue launch");
  }
  return TASQ_OK;
}

// ---------------------------------------------------------------- NVFP4 step
bool nvfp4_step(const tasq_ctx* c, int32_t layer, int32_t step) {
  return c->bits_host[static_cast<size_t>(layer) * c->num_steps + step] == 0;
}

// Whether the device may have chosen either format for this entry (see maybe_nvfp4).
bool either_format(const tasq_ctx* c, int32_t layer, int32_t step) {
  return c->maybe_nvfp4[static_cast<size_t>(layer) * c->num_steps + step] != 0;
}

// The NVFP4 weights of a layer live in masked-weight slot `slot`: codes [N, Kp / 2] at its start,
// block scales from the next 512-byte boundary.
uint8_t* nvfp4_w_codes(const tasq_ctx* c, int32_t slot) { return reinterpret_cast<uint8_t*>(wk_slot(c, slot)); }
uint8_t* nvfp4_w_sf(const tasq_ctx* c, int32_t layer, int32_t slot) {
  const LayerInfo& L = c->layers[layer];
  return nvfp4_w_codes(c, slot) + round_up(static_cast<size_t>(L.N) * L.Kp / 2, 512);
}

// NVFP4 prologue launch: activations (M > 0) into codes / sf / sx, and, when w_codes is set, the
// layer's weights converted into w_codes / w_sf. step < 0: no schedule check.
tasq_status run_prologue_nvfp4(tasq_ctx* c, int32_t layer, int32_t step, const void* x, int64_t M, int64_t ldx,
                               uint8_t* codes, uint8_t* sf, float* sx, uint8_t* w_codes, uint8_t* w_sf,
                               cudaStream_t s, int32_t gate = tasq::kGateNone) {
  const LayerInfo& L = c->layers[layer];
  tasq::Nvfp4PrologueArgs a{};
  a.x = x;
  a.ldx = ldx;
  a.K = L.K;
  a.Kp = L.Kp;
  a.n = c->n;
  a.M = M;
  a.codes = codes;
  a.sf = sf;
  a.s_x = sx;
  a.sx_factor = c->sx_factor4;
  if (w_codes != nullptr) {
    a.w = c->d_w + L.w_off;
    a.w_codes = w_codes;
    a.w_sf = w_sf;
    a.N = L.N;
    a.bits_table = c->d_bits;
    a.bits_index = layer * c->num_steps + (step < 0 ? 0 : step);
    if (step < 0) a.bits_table = nullptr;
  }
  a.status = c->d_status;
  if (step >= 0 && gate != tasq::kGateNone) {
    a.gate = gate;
    a.gate_table = c->d_bits;
    a.gate_index = layer * c->num_steps + step;
  }
  cudaError_t e = tasq::launch_prologue_nvfp4(a, s);
  if (e != cudaSuccess) return fail_cuda(e, "NVFP4 prologue launch");
  return TASQ_OK;
}

// NVFP4 GEMM of (layer, step) on the given activation codes and the weights in slot `slot`.
// step < 0: no schedule check. out S32 writes the raw FP32 accumulators.
tasq_status run_gemm_nvfp4(tasq_ctx* c, int32_t layer, int32_t step, const uint8_t* codes, const uint8_t* sf,
                           const float* sx, int64_t M, void* y, int64_t ldy, tasq::OutKind out, int32_t slot,
                           cudaStream_t s, int32_t gate = tasq::kGateNone) {
  const LayerInfo& L = c->layers[layer];
  const int64_t kp4 = tasq::nvfp4_kp4(L.Kp);
  const bool pair = c->gemm_mode == 2 || (c->gemm_mode == 0 && tasq::nvfp4_use_pair(M, L.N, c->num_sms));
  const int tile_tok = pair ? tasq::kGemmNvfp4PairTok : 128;
  const int tile_ch = pair ? 256 : 128;
  CUtensorMap tw, tx, ty;
  tasq_status st = make_tmap_u8(&tw, nvfp4_w_codes(c, slot), static_cast<uint64_t>(L.Kp / 2),
                                static_cast<uint64_t>(L.N), 128, 128);
  if (st == TASQ_OK)
    st = make_tmap_u8(&tx, codes, static_cast<uint64_t>(L.Kp / 2), static_cast<uint64_t>(M), 128,
                      static_cast<uint32_t>(pair ? tile_tok / 2 : tile_tok));
  if (st != TASQ_OK) return st;
  const CUtensorMapDataType dt = out == tasq::OutKind::S32    ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                 : out == tasq::OutKind::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  st = make_tmap_out(&ty, y, dt, out == tasq::OutKind::S32 ? 4u : 2u, static_cast<uint64_t>(L.N),
                     static_cast<uint64_t>(M), static_cast<uint64_t>(ldy));
  if (st != TASQ_OK) return st;
  tasq::GemmArgs g{};
  g.M = static_cast<int32_t>(M);
  g.N = L.N;
  g.num_kb = static_cast<int32_t>(kp4 / 256);
  g.num_m_tiles = static_cast<int32_t>((M + tile_tok - 1) / tile_tok);
  g.num_n_tiles = (L.N + tile_ch - 1) / tile_ch;
  g.bits_table = step < 0 ? nullptr : c->d_bits;
  g.bits_index = layer * c->num_steps + (step < 0 ? 0 : step);
  g.s_x = sx;
  g.s_w = c->d_sw + L.sw_off;
  g.y = y;
  g.ldy = ldy;
  g.status = c->d_status;
  g.wait_limit_ns = c->wait_limit_ns;
  g.gate = step < 0 ? tasq::kGateNone : gate;
  g.band_tiles = tasq::gemm_band_tiles(g.num_m_tiles, tile_tok, L.Kp / 2);
  tasq::Nvfp4GemmArgs f{};
  f.w_sf = nvfp4_w_sf(c, layer, slot);
  f.x_sf = sf;
  f.sf_chunks = static_cast<int32_t>(kp4 / 64);
  cudaError_t e = pair ? tasq::launch_gemm_nvfp4_pair(tw, tx, ty, g, f, out, c->num_sms, s)
                       : tasq::launch_gemm_nvfp4(tw, tx, ty, g, f, out, c->num_sms, s);
  if (e != cudaSuccess) return fail_cuda(e, pair ? "NVFP4 pair GEMM launch" : "NVFP4 GEMM launch");
  return TASQ_OK;
}

}  // namespace

namespace tasq {

// Which GEMM kernel finishes first. Both kernels are persistent, so a launch takes (waves of
// tiles) x (time per tile). CUDA-event timings of single launches on B200, over both kernels on
// the PixArt-Sigma, SANA, SDXL and CogVideoX shapes, fixed the rule:
//   * with fewer waves the CTA pair (256 x 256 tiles) wins outright, with more it loses;
//   * with equal waves the pair wins from four waves up (6 % on PixArt-Sigma fc1 and SDXL ff1,
//     3-9 % on CogVideoX) and loses up to 9 % at one or two waves (SANA proj and fc2), where its
//     cluster set-up and exit handshake are not amortised; at three it is level or behind.
// Narrower token tiles (64 .. 224 tokens, both kernels) were measured as well: a tile's time
// shrinks much less than its width, so they lost everywhere but on a few wave-quantised shapes,
// and won there by 3 % at most.
// Bands of 8 token tiles. Measured on CogVideoX block 0 (DRAM bytes read per GEMM launch, ncu in
// place): the token tile varying fastest over all of M read 228 / 84 / 299 / 2534 MB (qkv, proj,
// fc1, fc2); bands of 8 read 170 / 63 / 351 / 654 MB; bands sized to keep 48 MB of codes in L2
// (16 to 64 tiles) read 265 / 94 / 358 / 821 MB, the output stream evicting their codes.
int32_t gemm_band_tiles(int64_t num_m_tiles, int64_t /*tile_tok*/, int64_t /*code_row_bytes*/) {
  constexpr int64_t kBand = 8;
  const int64_t band = num_m_tiles < kBand ? num_m_tiles : kBand;
  return static_cast<int32_t>(band < 1 ? 1 : band);   // never 0: the kernels divide by it
}

bool gemm_use_pair(int64_t M, int64_t N, int num_sms) {
  const int64_t m_tiles = (M + kGemmTileTok - 1) / kGemmTileTok;
  const int64_t t1 = m_tiles * ((N + kGemmTileCh - 1) / kGemmTileCh);
  const int64_t t2 = m_tiles * ((N + kGemmPairTile - 1) / kGemmPairTile);
  const int64_t slots1 = num_sms, slots2 = num_sms / 2;
  const int64_t w1 = (t1 + slots1 - 1) / slots1;
  const int64_t w2 = (t2 + slots2 - 1) / slots2;
  return w2 < w1 || (w2 == w1 && w1 >= 4);
}

// The NVFP4 kernels by estimated time, waves x time per tile: a pair tile (256 x 192 on two SMs)
// holds 1.5x the MACs per SM of a one-CTA tile (128 x 128) and runs them 1.37x faster (CogVideoX
// qkv, 17776 x 3072 -> 9216, CUDA events), so it takes about 1.1x as long.
bool nvfp4_use_pair(int64_t M, int64_t N, int num_sms) {
  const int64_t t1 = ((M + 127) / 128) * ((N + 127) / 128);
  const int64_t t2 = ((M + kGemmNvfp4PairTok - 1) / kGemmNvfp4PairTok) * ((N + 255) / 256);
  const int64_t slots1 = num_sms, slots2 = num_sms / 2;
  const int64_t w1 = (t1 + slots1 - 1) / slots1;
  const int64_t w2 = (t2 + slots2 - 1) / slots2;
  return 110 * w2 <= 100 * w1;
}

}  // namespace tasq

namespace {

// GEMM of (layer, step). premasked: the weights come masked from masked-weight slot `slot`.
tasq_status run_gemm(tasq_ctx* c, int32_t layer, int32_t step, const int8_t* xq, const float* sx, int64_t M,
                     void* y, int64_t ldy, tasq::OutKind out, bool premasked, cudaStream_t s, int32_t slot = 0,
                     int32_t gate = tasq::kGateNone) {
  const LayerInfo& L = c->layers[layer];
  const bool pair = c->gemm_mode == 2 || (c->gemm_mode == 0 && tasq::gemm_use_pair(M, L.N, c->num_sms));
  const int tile_tok = pair ? tasq::kGemmPairTile : tasq::kGemmTileTok;
  const int tile_ch = pair ? tasq::kGemmPairTile : tasq::kGemmTileCh;
  CUtensorMap tx;
  tasq_status st = make_tmap_u8(&tx, xq, static_cast<uint64_t>(L.Kp), static_cast<uint64_t>(M), tasq::kGemmBlockK,
                                pair ? tasq::kGemmPairHalf : tile_tok);
  if (st != TASQ_OK) return st;
  CUtensorMap ty;
  const CUtensorMapDataType dt = out == tasq::OutKind::S32    ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                 : out == tasq::OutKind::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint32_t eb = out == tasq::OutKind::S32 ? 4u : 2u;
  st = make_tmap_out(&ty, y, dt, eb, static_cast<uint64_t>(L.N), static_cast<uint64_t>(M), static_cast<uint64_t>(ldy));
  if (st != TASQ_OK) return st;
  tasq::GemmArgs g{};
  g.M = static_cast<int32_t>(M);
  g.N = L.N;
  g.num_kb = (L.Kp + tasq::kGemmBlockK - 1) / tasq::kGemmBlockK;
  g.num_m_tiles = static_cast<int32_t>((M + tile_tok - 1) / tile_tok);
  g.num_n_tiles = (L.N + tile_ch - 1) / tile_ch;
  g.bits_table = c->d_bits;
  g.bits_index = layer * c->num_steps + step;
  g.s_x = sx;
  g.s_w = c->d_sw + L.sw_off;
  g.y = y;
  g.ldy = ldy;
  g.status = c->d_status;
  g.wait_limit_ns = c->wait_limit_ns;
  g.premasked = premasked ? 1 : 0;
  g.gate = gate;
  g.band_tiles = tasq::gemm_band_tiles(g.num_m_tiles, tile_tok, L.Kp);
  CUtensorMap tw = premasked ? c->tmap_wk[layer] : c->tmap_w[layer];
  if (premasked && slot != 0) {
    st = make_tmap_u8(&tw, wk_slot(c, slot), static_cast<uint64_t>(L.Kp), static_cast<uint64_t>(L.N),
                      tasq::kGemmBlockK, tasq::kGemmTileCh);
    if (st != TASQ_OK) return st;
  }
  cudaError_t e = pair ? tasq::launch_masked_gemm_pair(tw, tx, ty, g, out, c->num_sms, s)
                       : tasq::launch_masked_gemm(tw, tx, ty, g, out, c->num_sms, s);
  if (e != cudaSuccess) return fail_cuda(e, "masked GEMM launch");
  return TASQ_OK;
}

// GEMM of given codes, with the weight pass launched alone first when the mask goes ahead.
tasq_status debug_gemm(tasq_ctx* c, int32_t layer, int32_t step, const int8_t* xq, const float* sx, int64_t M, void* y,
                       int64_t ldy, tasq::OutKind out, cudaStream_t s) {
  const bool ahead = mask_ahead(c, layer, step);
  tasq_status st;
  if (ahead && (st = run_prologue(c, layer, step, {layer}, nullptr, 0, 0, nullptr, nullptr, s)) != TASQ_OK) return st;
  return run_gemm(c, layer, step, xq, sx, M, y, ldy, out, ahead, s);
}

}  // namespace

extern "C" {

const char* tasq_last_error(void) { return g_last_error.c_str(); }

tasq_status tasq_linear_create(tasq_ctx** out, const tasq_layer_desc* layers, int32_t num_layers, int32_t num_steps,
                               int32_t hadamard_n, int64_t max_tokens, int32_t out_dtype, void* stream) {
  g_last_error.clear();
  if (out == nullptr) return fail(TASQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (layers == nullptr || num_layers <= 0) return fail(TASQ_ERR_INVALID_ARG, "need at least one layer");
  if (num_steps <= 0) return fail(TASQ_ERR_INVALID_ARG, "num_steps must be >= 1");
  if (hadamard_n != 64 && hadamard_n != 128) return fail(TASQ_ERR_INVALID_ARG, "hadamard_n must be 64 or 128");
  if (max_tokens <= 0 || max_tokens > 0x7fffffffLL)
    return fail(TASQ_ERR_INVALID_ARG, "max_tokens must be in [1, 2^31 - 1]");
  if (out_dtype != TASQ_OUT_F16 && out_dtype != TASQ_OUT_BF16)
    return fail(TASQ_ERR_INVALID_ARG, "out_dtype must be TASQ_OUT_F16 or TASQ_OUT_BF16");
  if (static_cast<int64_t>(num_layers) * num_steps > (1LL << 30))
    return fail(TASQ_ERR_INVALID_ARG, "schedule table too large");

  std::vector<LayerInfo> info(num_layers);
  size_t w_bytes = 0, sw_count = 0, wk_bytes = 0;
  int32_t kp_max = 0;
  for (int32_t l = 0; l < num_layers; ++l) {
    const tasq_layer_desc& d = layers[l];
    if (d.N <= 0 || d.K < 8 || d.K % 8 != 0)
      return fail(TASQ_ERR_INVALID_ARG, "layer " + std::to_string(l) + ": need N >= 1 and K >= 8 with K % 8 == 0");
    if (d.w == nullptr || d.s_w == nullptr)
      return fail(TASQ_ERR_INVALID_ARG, "layer " + std::to_string(l) + ": weights or scales are NULL");
    const int32_t Kp = (d.K + hadamard_n - 1) / hadamard_n * hadamard_n;
    if (Kp > TASQ_MAX_KP)
      return fail(TASQ_ERR_INVALID_ARG, "layer " + std::to_string(l) + ": padded K " + std::to_string(Kp) +
                                            " exceeds " + std::to_string(TASQ_MAX_KP));
    info[l] = LayerInfo{d.N, d.K, Kp, w_bytes, sw_count};
    w_bytes = round_up(w_bytes + static_cast<size_t>(d.N) * Kp, 1024);
    if (static_cast<size_t>(d.N) * Kp > wk_bytes) wk_bytes = static_cast<size_t>(d.N) * Kp;
    // an NVFP4 step keeps the layer's converted weights in the same slot: codes, then scales
    const size_t f4 = round_up(static_cast<size_t>(d.N) * Kp / 2, 512) +
                      static_cast<size_t>(tasq::nvfp4_sf_bytes(d.N, Kp));
    if (f4 > wk_bytes) wk_bytes = f4;
    sw_count = round_up(sw_count + d.N, 64);
    if (Kp > kp_max) kp_max = Kp;
  }

  // every argument is checked on the host before the device is touched
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(TASQ_ERR_UNSUPPORTED_ARCH, std::string("device ") + prop.name + " is sm_" + std::to_string(prop.major) +
                                               std::to_string(prop.minor) + ", this library is built for sm_100a");

  tasq_ctx* c = new tasq_ctx();
  c->device = dev;
  c->num_sms = prop.multiProcessorCount;
  c->num_layers = num_layers;
  c->num_steps = num_steps;
  c->n = hadamard_n;
  c->out_dtype = out_dtype;
  c->max_tokens = max_tokens;
  c->kp_max = kp_max;
  c->layers = info;
  c->sx_factor = static_cast<float>(1.0 / (127.0 * std::sqrt(static_cast<double>(hadamard_n))));
  c->sx_factor4 = static_cast<float>(1.0 / (tasq::kNvfp4Range * std::sqrt(static_cast<double>(hadamard_n))));
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  auto bail = [&](cudaError_t err, const char* what) {
    tasq_status st = fail_cuda(err, what);
    free_ctx(c);
    return st;
  };
  if ((e = cudaMalloc(&c->d_w, w_bytes)) != cudaSuccess) return bail(e, "cudaMalloc(weights)");
  c->wk_slot_bytes = round_up(wk_bytes, 1024);
  c->wk_slots = num_layers < TASQ_GROUP_MAX ? num_layers : TASQ_GROUP_MAX;
  if ((e = cudaMalloc(&c->d_wk, c->wk_slot_bytes * c->wk_slots)) != cudaSuccess)
    return bail(e, "cudaMalloc(masked weights)");
  if ((e = cudaMalloc(&c->d_sw, sw_count * sizeof(float))) != cudaSuccess) return bail(e, "cudaMalloc(scales)");
  const size_t table = static_cast<size_t>(num_layers) * num_steps;
  if ((e = cudaMalloc(&c->d_bits, table)) != cudaSuccess) return bail(e, "cudaMalloc(schedule)");
  if ((e = cudaMalloc(&c->d_xq, static_cast<size_t>(max_tokens) * kp_max)) != cudaSuccess)
    return bail(e, "cudaMalloc(workspace codes)");
  if ((e = cudaMalloc(&c->d_sx, static_cast<size_t>(max_tokens) * sizeof(float))) != cudaSuccess)
    return bail(e, "cudaMalloc(workspace scales)");
  const size_t sf4_bytes = static_cast<size_t>(tasq::nvfp4_sf_bytes(max_tokens, kp_max));
  if ((e = cudaMalloc(&c->d_sf4, sf4_bytes)) != cudaSuccess) return bail(e, "cudaMalloc(NVFP4 block scales)");
  // scales past a layer's Kp and rows past M are read by the NVFP4 GEMM: keep them finite
  if ((e = cudaMemsetAsync(c->d_sf4, 0, sf4_bytes, s)) != cudaSuccess) return bail(e, "cudaMemsetAsync(NVFP4 scales)");
  if ((e = cudaMalloc(&c->d_status, sizeof(uint32_t))) != cudaSuccess) return bail(e, "cudaMalloc(status)");
  if ((e = cudaMalloc(&c->d_dmpq, 4 * sizeof(uint64_t) * static_cast<size_t>(c->num_sms) * tasq::kDmpqCtasPerSm)) !=
      cudaSuccess)
    return bail(e, "cudaMalloc(predictor partial sums)");
  if ((e = cudaMalloc(&c->d_dmpq_arrived, sizeof(unsigned int))) != cudaSuccess) return bail(e, "cudaMalloc(counter)");
  if ((e = cudaMemsetAsync(c->d_dmpq_arrived, 0, sizeof(unsigned int), s)) != cudaSuccess)
    return bail(e, "cudaMemsetAsync(counter)");

  if ((e = cudaMemsetAsync(c->d_bits, 8, table, s)) != cudaSuccess) return bail(e, "cudaMemsetAsync(schedule)");
  c->bits_host.assign(table, 8);
  c->maybe_nvfp4.assign(table, 0);
  if ((e = cudaMemsetAsync(c->d_status, 0, sizeof(uint32_t), s)) != cudaSuccess) return bail(e, "cudaMemsetAsync(status)");
  for (int32_t l = 0; l < num_layers; ++l) {
    const LayerInfo& L = info[l];
    e = cudaMemcpyAsync(c->d_w + L.w_off, layers[l].w, static_cast<size_t>(L.N) * L.Kp, cudaMemcpyDefault, s);
    if (e != cudaSuccess) return bail(e, "copy of weights");
    e = cudaMemcpyAsync(c->d_sw + L.sw_off, layers[l].s_w, static_cast<size_t>(L.N) * sizeof(float),
                        cudaMemcpyDefault, s);
    if (e != cudaSuccess) return bail(e, "copy of weight scales");
  }
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return bail(e, "cudaStreamSynchronize");

  c->tmap_w.resize(num_layers);
  c->tmap_wk.resize(num_layers);
  for (int32_t l = 0; l < num_layers; ++l) {
    const LayerInfo& L = info[l];
    tasq_status st = make_tmap_u8(&c->tmap_w[l], c->d_w + L.w_off, static_cast<uint64_t>(L.Kp),
                                  static_cast<uint64_t>(L.N), tasq::kGemmBlockK, tasq::kGemmTileCh);
    if (st == TASQ_OK)
      st = make_tmap_u8(&c->tmap_wk[l], c->d_wk, static_cast<uint64_t>(L.Kp), static_cast<uint64_t>(L.N),
                        tasq::kGemmBlockK, tasq::kGemmTileCh);
    if (st != TASQ_OK) {
      std::string m = g_last_error;
      free_ctx(c);
      return fail(st, m);
    }
  }
  *out = c;
  return TASQ_OK;
}

tasq_status tasq_set_schedule(tasq_ctx* c, const uint8_t* bits_host, void* stream) {
  g_last_error.clear();
  if (c == nullptr || bits_host == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx or bits is NULL");
  tasq_status st = check_device(c);
  if (st != TASQ_OK) return st;
  const size_t table = static_cast<size_t>(c->num_layers) * c->num_steps;
  for (size_t i = 0; i < table; ++i) {
    if (bits_host[i] > 8)
      return fail(TASQ_ERR_INVALID_ARG, "bits[" + std::to_string(i) + "] = " + std::to_string(bits_host[i]) +
                                            " outside [0, 8] (0: NVFP4, 1..8: INT8 width)");
  }
  cudaError_t e = cudaMemcpyAsync(c->d_bits, bits_host, table, cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "copy of schedule");
  c->bits_host.assign(bits_host, bits_host + table);
  c->maybe_nvfp4.assign(table, 0);
  return TASQ_OK;
}

tasq_status tasq_linear_forward(tasq_ctx* c, const void* x, int64_t M, int64_t ldx, int32_t layer, int32_t step, void* y,
                                int64_t ldy, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st;
  if ((st = check_layer(c, layer)) != TASQ_OK) return st;
  if ((st = check_step(c, step)) != TASQ_OK) return st;
  if ((st = check_tokens(c, M)) != TASQ_OK) return st;
  const LayerInfo& L = c->layers[layer];
  if ((st = check_rows(x, ldx, L.K, "x")) != TASQ_OK) return st;
  if ((st = check_rows(y, ldy, L.N, "y")) != TASQ_OK) return st;
  if ((st = check_device(c)) != TASQ_OK) return st;
  if (M == 0) return TASQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  TraceRec* tr = c->trace_count < c->trace_cap ? &c->trace[c->trace_count] : nullptr;
  const tasq::OutKind out = c->out_dtype == TASQ_OUT_BF16 ? tasq::OutKind::BF16 : tasq::OutKind::F16;
  if (either_format(c, layer, step)) {
    // the predictor decided on the device: both paths are launched, each gated on the table, and
    // exactly one of them runs (the INT8 width the host knows of is bits_host's entry)
    uint8_t* codes4 = reinterpret_cast<uint8_t*>(c->d_xq);
    const bool ahead = mask_ahead(c, layer, step);
    if (tr) cudaEventRecord(tr->e0, s);
    if ((st = run_prologue(c, layer, step, ahead ? std::vector<int32_t>{layer} : std::vector<int32_t>{}, x, M, ldx,
                           c->d_xq, c->d_sx, s, tasq::kGateInt8)) != TASQ_OK)
      return st;
    if ((st = run_prologue_nvfp4(c, layer, step, x, M, ldx, codes4, c->d_sf4, c->d_sx, nvfp4_w_codes(c, 0),
                                 nvfp4_w_sf(c, layer, 0), s, tasq::kGateNvfp4)) != TASQ_OK)
      return st;
    if (tr) cudaEventRecord(tr->e1, s);
    if ((st = run_gemm(c, layer, step, c->d_xq, c->d_sx, M, y, ldy, out, ahead, s, 0, tasq::kGateInt8)) != TASQ_OK)
      return st;
    if ((st = run_gemm_nvfp4(c, layer, step, codes4, c->d_sf4, c->d_sx, M, y, ldy, out, 0, s, tasq::kGateNvfp4)) !=
        TASQ_OK)
      return st;
    if (tr) {
      cudaEventRecord(tr->e2, s);
      tr->ops = 2.0 * static_cast<double>(M) * L.N * L.K;
      tr->bytes = static_cast<double>(M) * (2.0 * L.K + L.Kp + 4.0);
      tr->wbytes = ahead ? 2.0 * L.N * L.Kp : 0.0;
      ++c->trace_count;
    }
    return TASQ_OK;
  }
  if (nvfp4_step(c, layer, step)) {
    // NVFP4 step: the prologue launch also converts the layer's weights, into slot 0
    uint8_t* codes = reinterpret_cast<uint8_t*>(c->d_xq);
    if (tr) cudaEventRecord(tr->e0, s);
    if ((st = run_prologue_nvfp4(c, layer, step, x, M, ldx, codes, c->d_sf4, c->d_sx, nvfp4_w_codes(c, 0),
                                 nvfp4_w_sf(c, layer, 0), s)) != TASQ_OK)
      return st;
    if (tr) cudaEventRecord(tr->e1, s);
    if ((st = run_gemm_nvfp4(c, layer, step, codes, c->d_sf4, c->d_sx, M, y, ldy, out, 0, s)) != TASQ_OK) return st;
    if (tr) {
      cudaEventRecord(tr->e2, s);
      tr->ops = 2.0 * static_cast<double>(M) * L.N * L.K;
      tr->bytes = static_cast<double>(M) * (2.0 * L.K + L.Kp / 2.0 + L.Kp / 16.0 + 4.0);
      tr->wbytes = static_cast<double>(L.N) * L.Kp * (1.0 + 0.5 + 1.0 / 16.0);
      ++c->trace_count;
    }
    return TASQ_OK;
  }
  const bool ahead = mask_ahead(c, layer, step);
  if (tr) cudaEventRecord(tr->e0, s);
  if ((st = run_prologue(c, layer, step, ahead ? std::vector<int32_t>{layer} : std::vector<int32_t>{}, x, M, ldx,
                         c->d_xq, c->d_sx, s)) != TASQ_OK)
    return st;
  if (tr) cudaEventRecord(tr->e1, s);
  if ((st = run_gemm(c, layer, step, c->d_xq, c->d_sx, M, y, ldy, out, ahead, s)) != TASQ_OK) return st;
  if (tr) {
    cudaEventRecord(tr->e2, s);
    tr->ops = 2.0 * static_cast<double>(M) * L.N * L.K;
    tr->bytes = static_cast<double>(M) * (2.0 * L.K + L.Kp + 4.0);
    tr->wbytes = ahead ? 2.0 * L.N * L.Kp : 0.0;
    ++c->trace_count;
  }
  return TASQ_OK;
}

tasq_status tasq_linear_forward_group(tasq_ctx* c, const void* x, int64_t M, int64_t ldx, const int32_t* layers,
                                      int32_t count, int32_t step, void* const* ys, const int64_t* ldys, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  if (layers == nullptr || ys == nullptr || ldys == nullptr) return fail(TASQ_ERR_INVALID_ARG, "NULL array");
  if (count < 1 || count > c->wk_slots)
    return fail(TASQ_ERR_INVALID_ARG, "count must be in [1, min(num_layers, TASQ_GROUP_MAX)]");
  tasq_status st;
  if ((st = check_step(c, step)) != TASQ_OK) return st;
  if ((st = check_tokens(c, M)) != TASQ_OK) return st;
  for (int32_t i = 0; i < count; ++i) {
    if ((st = check_layer(c, layers[i])) != TASQ_OK) return st;
    if (c->layers[layers[i]].K != c->layers[layers[0]].K)
      return fail(TASQ_ERR_INVALID_ARG, "the layers of a group must share K");
    if ((st = check_rows(ys[i], ldys[i], c->layers[layers[i]].N, "y")) != TASQ_OK) return st;
  }
  const LayerInfo& L0 = c->layers[layers[0]];
  if ((st = check_rows(x, ldx, L0.K, "x")) != TASQ_OK) return st;
  if ((st = check_device(c)) != TASQ_OK) return st;
  if (M == 0) return TASQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // an NVFP4 step quantizes the input differently: then every member runs as its own forward
  for (int32_t i = 0; i < count; ++i) {
    if (nvfp4_step(c, layers[i], step) || either_format(c, layers[i], step)) {
      for (int32_t j = 0; j < count; ++j) {
        if ((st = tasq_linear_forward(c, x, M, ldx, layers[j], step, ys[j], ldys[j], stream)) != TASQ_OK) return st;
      }
      return TASQ_OK;
    }
  }

  // one prologue for the shared input; it also masks, each into its own slot, the weights of
  // every member whose step drops bits
  std::vector<int32_t> masked;
  std::vector<int32_t> slot_of(count, -1);
  for (int32_t i = 0; i < count; ++i) {
    if (mask_ahead(c, layers[i], step)) {
      slot_of[i] = static_cast<int32_t>(masked.size());
      masked.push_back(layers[i]);
    }
  }
  TraceRec* tr = c->trace_count < c->trace_cap ? &c->trace[c->trace_count] : nullptr;
  if (tr) cudaEventRecord(tr->e0, s);
  if ((st = run_prologue(c, layers[0], step, masked, x, M, ldx, c->d_xq, c->d_sx, s)) != TASQ_OK) return st;
  if (tr) cudaEventRecord(tr->e1, s);
  const tasq::OutKind out = c->out_dtype == TASQ_OUT_BF16 ? tasq::OutKind::BF16 : tasq::OutKind::F16;
  double ops = 0.0, wbytes = 0.0;
  for (int32_t i = 0; i < count; ++i) {
    const LayerInfo& L = c->layers[layers[i]];
    const bool ahead = slot_of[i] >= 0;
    if ((st = run_gemm(c, layers[i], step, c->d_xq, c->d_sx, M, ys[i], ldys[i], out, ahead, s,
                       ahead ? slot_of[i] : 0)) != TASQ_OK)
      return st;
    ops += 2.0 * static_cast<double>(M) * L.N * L.K;
    if (ahead) wbytes += 2.0 * L.N * L.Kp;
  }
  if (tr) {
    cudaEventRecord(tr->e2, s);
    tr->ops = ops;
    tr->bytes = static_cast<double>(M) * (2.0 * L0.K + L0.Kp + 4.0);
    tr->wbytes = wbytes;
    ++c->trace_count;
  }
  return TASQ_OK;
}

tasq_status tasq_linear_destroy(tasq_ctx* c) {
  g_last_error.clear();
  free_ctx(c);
  return TASQ_OK;
}

tasq_status tasq_get_device_status(tasq_ctx* c, uint32_t* status_out, int32_t clear, void* stream) {
  g_last_error.clear();
  if (c == nullptr || status_out == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx or status_out is NULL");
  tasq_status st = check_device(c);
  if (st != TASQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, c->d_status, sizeof(v), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail_cuda(e, "read of device status");
  if (clear) {
    e = cudaMemsetAsync(c->d_status, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail_cuda(e, "clear of device status");
  }
  *status_out = v;
  return TASQ_OK;
}

tasq_status tasq_set_wait_limit(tasq_ctx* c, uint64_t limit_ns) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  if (limit_ns < 1000ull) return fail(TASQ_ERR_INVALID_ARG, "wait limit below 1 us");
  c->wait_limit_ns = limit_ns;
  return TASQ_OK;
}

tasq_status tasq_layer_info(const tasq_ctx* c, int32_t layer, int32_t* N, int32_t* K, int32_t* Kp) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st = check_layer(c, layer);
  if (st != TASQ_OK) return st;
  const LayerInfo& L = c->layers[layer];
  if (N) *N = L.N;
  if (K) *K = L.K;
  if (Kp) *Kp = L.Kp;
  return TASQ_OK;
}

tasq_status tasq_debug_quantize(tasq_ctx* c, const void* x, int64_t M, int64_t ldx, int32_t layer, int8_t* xq, float* s_x,
                                void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st;
  if ((st = check_layer(c, layer)) != TASQ_OK) return st;
  if (M < 0 || M > 0x7fffffffLL) return fail(TASQ_ERR_INVALID_ARG, "M out of range");
  const LayerInfo& L = c->layers[layer];
  if ((st = check_rows(x, ldx, L.K, "x")) != TASQ_OK) return st;
  if ((st = check_rows(xq, L.Kp, L.Kp, "xq")) != TASQ_OK) return st;
  if (s_x == nullptr || !aligned16(s_x)) return fail(TASQ_ERR_INVALID_ARG, "s_x must be a 16-byte aligned pointer");
  if ((st = check_device(c)) != TASQ_OK) return st;
  if (M == 0) return TASQ_OK;
  return run_prologue(c, layer, 0, {}, x, M, ldx, xq, s_x, static_cast<cudaStream_t>(stream));
}

tasq_status tasq_debug_gemm_s32(tasq_ctx* c, const int8_t* xq, int64_t M, int32_t layer, int32_t step, int32_t* acc,
                                int64_t ld_acc, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st;
  if ((st = check_layer(c, layer)) != TASQ_OK) return st;
  if ((st = check_step(c, step)) != TASQ_OK) return st;
  if (M < 0 || M > 0x7fffffffLL) return fail(TASQ_ERR_INVALID_ARG, "M out of range");
  const LayerInfo& L = c->layers[layer];
  if ((st = check_rows(xq, L.Kp, L.Kp, "xq")) != TASQ_OK) return st;
  if ((st = check_rows(acc, ld_acc, L.N, "acc")) != TASQ_OK) return st;
  if ((st = check_device(c)) != TASQ_OK) return st;
  if (M == 0) return TASQ_OK;
  return debug_gemm(c, layer, step, xq, nullptr, M, acc, ld_acc, tasq::OutKind::S32, static_cast<cudaStream_t>(stream));
}

tasq_status tasq_debug_gemm(tasq_ctx* c, const int8_t* xq, const float* s_x, int64_t M, int32_t layer, int32_t step,
                            void* y, int64_t ldy, int32_t out_dtype, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st;
  if ((st = check_layer(c, layer)) != TASQ_OK) return st;
  if ((st = check_step(c, step)) != TASQ_OK) return st;
  if (M < 0 || M > 0x7fffffffLL) return fail(TASQ_ERR_INVALID_ARG, "M out of range");
  if (out_dtype != TASQ_OUT_F16 && out_dtype != TASQ_OUT_BF16) return fail(TASQ_ERR_INVALID_ARG, "bad out_dtype");
  const LayerInfo& L = c->layers[layer];
  if ((st = check_rows(xq, L.Kp, L.Kp, "xq")) != TASQ_OK) return st;
  if (s_x == nullptr || !aligned16(s_x)) return fail(TASQ_ERR_INVALID_ARG, "s_x must be a 16-byte aligned pointer");
  if ((st = check_rows(y, ldy, L.N, "y")) != TASQ_OK) return st;
  if ((st = check_device(c)) != TASQ_OK) return st;
  if (M == 0) return TASQ_OK;
  const tasq::OutKind out = out_dtype == TASQ_OUT_BF16 ? tasq::OutKind::BF16 : tasq::OutKind::F16;
  return debug_gemm(c, layer, step, xq, s_x, M, y, ldy, out, static_cast<cudaStream_t>(stream));
}

tasq_status tasq_nvfp4_scale_bytes(int64_t rows, int32_t Kp, int64_t* bytes) {
  g_last_error.clear();
  if (bytes == nullptr) return fail(TASQ_ERR_INVALID_ARG, "bytes is NULL");
  if (rows < 0 || Kp <= 0 || Kp % 64 != 0) return fail(TASQ_ERR_INVALID_ARG, "rows >= 0 and Kp a positive multiple of 64");
  *bytes = tasq::nvfp4_sf_bytes(rows, Kp);
  return TASQ_OK;
}

tasq_status tasq_debug_quantize_nvfp4(tasq_ctx* c, const void* x, int64_t M, int64_t ldx, int32_t layer, void* codes,
                                      void* scales, float* s_x, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st;
  if ((st = check_layer(c, layer)) != TASQ_OK) return st;
  if (M < 0 || M > 0x7fffffffLL) return fail(TASQ_ERR_INVALID_ARG, "M out of range");
  const LayerInfo& L = c->layers[layer];
  if ((st = check_rows(x, ldx, L.K, "x")) != TASQ_OK) return st;
  if (codes == nullptr || !aligned16(codes) || scales == nullptr || !aligned16(scales) || s_x == nullptr)
    return fail(TASQ_ERR_INVALID_ARG, "codes and scales must be 16-byte aligned, s_x non-NULL");
  if ((st = check_device(c)) != TASQ_OK) return st;
  if (M == 0) return TASQ_OK;
  return run_prologue_nvfp4(c, layer, -1, x, M, ldx, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales), s_x,
                            nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

tasq_status tasq_debug_nvfp4_weights(tasq_ctx* c, int32_t layer, void* codes, void* scales, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st;
  if ((st = check_layer(c, layer)) != TASQ_OK) return st;
  if (codes == nullptr || !aligned16(codes) || scales == nullptr || !aligned16(scales))
    return fail(TASQ_ERR_INVALID_ARG, "codes and scales must be 16-byte aligned");
  if ((st = check_device(c)) != TASQ_OK) return st;
  return run_prologue_nvfp4(c, layer, -1, nullptr, 0, c->layers[layer].K, nullptr, nullptr, nullptr,
                            static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                            static_cast<cudaStream_t>(stream));
}

tasq_status tasq_debug_gemm_nvfp4(tasq_ctx* c, const void* codes, const void* scales, const float* s_x, int64_t M,
                                  int32_t layer, void* y, int64_t ldy, int32_t out_kind, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st;
  if ((st = check_layer(c, layer)) != TASQ_OK) return st;
  if (M < 0 || M > 0x7fffffffLL) return fail(TASQ_ERR_INVALID_ARG, "M out of range");
  if (out_kind != TASQ_OUT_F16 && out_kind != TASQ_OUT_BF16 && out_kind != TASQ_NVFP4_RAW_ACC)
    return fail(TASQ_ERR_INVALID_ARG, "bad out_kind");
  const LayerInfo& L = c->layers[layer];
  if (codes == nullptr || !aligned16(codes) || scales == nullptr || !aligned16(scales))
    return fail(TASQ_ERR_INVALID_ARG, "codes and scales must be 16-byte aligned");
  if (s_x == nullptr || !aligned16(s_x)) return fail(TASQ_ERR_INVALID_ARG, "s_x must be a 16-byte aligned pointer");
  if (out_kind == TASQ_NVFP4_RAW_ACC) {
    if (y == nullptr || !aligned16(y) || ldy < L.N || ldy % 4 != 0)
      return fail(TASQ_ERR_INVALID_ARG, "y must be 16-byte aligned with a row stride >= N and a multiple of 4");
  } else if ((st = check_rows(y, ldy, L.N, "y")) != TASQ_OK) {
    return st;
  }
  if ((st = check_device(c)) != TASQ_OK) return st;
  if (M == 0) return TASQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the layer's weights are converted into slot 0, then the GEMM reads them from there
  if ((st = run_prologue_nvfp4(c, layer, -1, nullptr, 0, L.K, nullptr, nullptr, nullptr, nvfp4_w_codes(c, 0),
                               nvfp4_w_sf(c, layer, 0), s)) != TASQ_OK)
    return st;
  const tasq::OutKind out = out_kind == TASQ_NVFP4_RAW_ACC ? tasq::OutKind::S32
                            : out_kind == TASQ_OUT_BF16     ? tasq::OutKind::BF16
                                                            : tasq::OutKind::F16;
  return run_gemm_nvfp4(c, layer, -1, static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(scales), s_x,
                        M, y, ldy, out, 0, s);
}

tasq_status tasq_get_schedule(tasq_ctx* c, uint8_t* bits_host, void* stream) {
  g_last_error.clear();
  if (c == nullptr || bits_host == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx or bits is NULL");
  tasq_status st = check_device(c);
  if (st != TASQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t table = static_cast<size_t>(c->num_layers) * c->num_steps;
  cudaError_t e = cudaMemcpyAsync(bits_host, c->d_bits, table, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail_cuda(e, "read of schedule");
  return TASQ_OK;
}

tasq_status tasq_dmpq_update(tasq_ctx* c, const void* block_in, int64_t ld_in, const void* block_out, int64_t ld_out,
                             int64_t M, int32_t D, const int32_t* layers, int32_t num_block_layers, int32_t step,
                             double tau, int32_t bits_unstable, int32_t bits_stable, double* gamma_out, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st;
  if ((st = check_step(c, step)) != TASQ_OK) return st;
  if (layers == nullptr || num_block_layers < 1 || num_block_layers > TASQ_DMPQ_MAX_LAYERS)
    return fail(TASQ_ERR_INVALID_ARG, "need 1 to TASQ_DMPQ_MAX_LAYERS layer indices");
  for (int32_t i = 0; i < num_block_layers; ++i)
    if ((st = check_layer(c, layers[i])) != TASQ_OK) return st;
  if (bits_unstable < 0 || bits_unstable > 8 || bits_stable < 0 || bits_stable > 8)
    return fail(TASQ_ERR_INVALID_ARG, "widths must be in [0, 8] (0: NVFP4)");
  if (!(tau == tau)) return fail(TASQ_ERR_INVALID_ARG, "tau is NaN");
  if (M < 0 || M > 0x7fffffffLL) return fail(TASQ_ERR_INVALID_ARG, "M out of range");
  if (D < 8 || D % 8 != 0) return fail(TASQ_ERR_INVALID_ARG, "D must be a positive multiple of 8");
  if ((st = check_rows(block_in, ld_in, D, "block_in")) != TASQ_OK) return st;
  if ((st = check_rows(block_out, ld_out, D, "block_out")) != TASQ_OK) return st;
  if (gamma_out != nullptr && reinterpret_cast<uintptr_t>(gamma_out) % 8 != 0)
    return fail(TASQ_ERR_INVALID_ARG, "gamma_out must be 8-byte aligned");
  // every thread of the reduction adds at most 2^21 terms below 2^41 units: no 64-bit overflow
  const int ctas = tasq::dmpq_partial_ctas(M, D, c->num_sms);
  const int64_t per_thread = (M * D + static_cast<int64_t>(ctas) * 256 - 1) / (static_cast<int64_t>(ctas) * 256);
  if (per_thread > (1LL << 21)) return fail(TASQ_ERR_INVALID_ARG, "M * D too large for exact 64-bit partial sums");
  if ((st = check_device(c)) != TASQ_OK) return st;
  tasq::DmpqArgs a{};
  a.in = block_in;
  a.out = block_out;
  a.ld_in = ld_in;
  a.ld_out = ld_out;
  a.M = M;
  a.D = D;
  a.tau = tau;
  a.bits_unstable = bits_unstable;
  a.bits_stable = bits_stable;
  a.table = c->d_bits;
  a.num_entries = num_block_layers;
  for (int32_t i = 0; i < num_block_layers; ++i) a.entries[i] = layers[i] * c->num_steps + step;
  a.gamma_out = gamma_out;
  cudaError_t e = tasq::launch_dmpq(a, c->d_dmpq, c->d_dmpq_arrived, c->num_sms, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "predictor launch");
  // the host copy of the table steers where the mask is applied and which kernels a forward
  // launches. Both widths INT8: take the narrower one, so that a dropped bit is masked once ahead
  // of the GEMM whichever way the device decides. One of them NVFP4: keep the INT8 one and mark
  // the entry, so that its forwards launch both paths gated on the table. Both NVFP4: NVFP4.
  const bool f4u = bits_unstable == 0, f4s = bits_stable == 0;
  const uint8_t hint = static_cast<uint8_t>(f4u && f4s ? 0
                                            : f4u       ? bits_stable
                                            : f4s       ? bits_unstable
                                            : (bits_unstable < bits_stable ? bits_unstable : bits_stable));
  const uint8_t either = (f4u != f4s) ? 1 : 0;
  for (int32_t i = 0; i < num_block_layers; ++i) {
    const size_t entry = static_cast<size_t>(layers[i]) * c->num_steps + step;
    c->bits_host[entry] = hint;
    c->maybe_nvfp4[entry] = either;
  }
  return TASQ_OK;
}

tasq_status tasq_debug_set_gemm_mode(tasq_ctx* c, int32_t mode) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  if (mode < 0 || mode > 2) return fail(TASQ_ERR_INVALID_ARG, "mode must be 0, 1 or 2");
  c->gemm_mode = mode;
  return TASQ_OK;
}

tasq_status tasq_gemm_choice(int64_t M, int32_t N, int32_t num_sms, int32_t* pair) {
  g_last_error.clear();
  if (pair == nullptr) return fail(TASQ_ERR_INVALID_ARG, "pair is NULL");
  if (M <= 0 || N <= 0 || num_sms <= 1) return fail(TASQ_ERR_INVALID_ARG, "M and N must be positive, num_sms > 1");
  *pair = tasq::gemm_use_pair(M, N, num_sms) ? 1 : 0;
  return TASQ_OK;
}

tasq_status tasq_nvfp4_gemm_choice(int64_t M, int32_t N, int32_t num_sms, int32_t* pair) {
  g_last_error.clear();
  if (pair == nullptr) return fail(TASQ_ERR_INVALID_ARG, "pair is NULL");
  if (M <= 0 || N <= 0 || num_sms <= 1) return fail(TASQ_ERR_INVALID_ARG, "M and N must be positive, num_sms > 1");
  *pair = tasq::nvfp4_use_pair(M, N, num_sms) ? 1 : 0;
  return TASQ_OK;
}

tasq_status tasq_debug_set_prologue_mode(tasq_ctx* c, int32_t mode) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  if (mode < 0 || mode > 3) return fail(TASQ_ERR_INVALID_ARG, "mode must be 0, 1, 2 or 3");
  c->prologue_mode = mode;
  return TASQ_OK;
}

tasq_status tasq_debug_set_mask_mode(tasq_ctx* c, int32_t mode) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  if (mode < 0 || mode > 2) return fail(TASQ_ERR_INVALID_ARG, "mode must be 0, 1 or 2");
  c->mask_mode = mode;
  return TASQ_OK;
}

tasq_status tasq_debug_stuck_wait(tasq_ctx* c, void* stream) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  tasq_status st = check_device(c);
  if (st != TASQ_OK) return st;
  cudaError_t e = tasq::launch_stuck_wait(c->d_status, c->wait_limit_ns, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "stuck-wait launch");
  return TASQ_OK;
}

tasq_status tasq_trace_enable(tasq_ctx* c, int32_t capacity) {
  g_last_error.clear();
  if (c == nullptr || capacity < 0) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL or capacity < 0");
  tasq_status st = check_device(c);
  if (st != TASQ_OK) return st;
  while (static_cast<int32_t>(c->trace.size()) < capacity) {
    TraceRec r{};
    cudaError_t e = cudaEventCreate(&r.e0);
    if (e == cudaSuccess) e = cudaEventCreate(&r.e1);
    if (e == cudaSuccess) e = cudaEventCreate(&r.e2);
    if (e != cudaSuccess) return fail_cuda(e, "cudaEventCreate");
    c->trace.push_back(r);
  }
  c->trace_cap = capacity;
  c->trace_count = 0;
  return TASQ_OK;
}

tasq_status tasq_trace_read(tasq_ctx* c, int32_t* prologue_launches, double* prologue_ms, int32_t* gemm_launches,
                            double* gemm_ms, double* gemm_ops, double* prologue_bytes, double* weight_pass_bytes) {
  g_last_error.clear();
  if (c == nullptr) return fail(TASQ_ERR_INVALID_ARG, "ctx is NULL");
  double pm = 0, gm = 0, ops = 0, bytes = 0, wbytes = 0;
  for (int32_t i = 0; i < c->trace_count; ++i) {
    TraceRec& r = c->trace[i];
    cudaError_t e = cudaEventSynchronize(r.e2);
    if (e != cudaSuccess) return fail_cuda(e, "cudaEventSynchronize");
    float a = 0, b = 0;
    e = cudaEventElapsedTime(&a, r.e0, r.e1);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&b, r.e1, r.e2);
    if (e != cudaSuccess) return fail_cuda(e, "cudaEventElapsedTime");
    pm += a;
    gm += b;
    ops += r.ops;
    bytes += r.bytes;
    wbytes += r.wbytes;
  }
  if (prologue_launches) *prologue_launches = c->trace_count;
  if (gemm_launches) *gemm_launches = c->trace_count;
  if (prologue_ms) *prologue_ms = pm;
  if (gemm_ms) *gemm_ms = gm;
  if (gemm_ops) *gemm_ops = ops;
  if (prologue_bytes) *prologue_bytes = bytes;
  if (weight_pass_bytes) *weight_pass_bytes = wbytes;
  c->trace_count = 0;
  return TASQ_OK;
}

}  // extern "C"
