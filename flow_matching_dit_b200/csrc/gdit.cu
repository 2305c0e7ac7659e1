// Runtime and C ABI of the flow-matching DiT action head (see include/gdit.h).
//
// One call of gdit_get_action enqueues, on the caller's stream:
//   route (stable sort by embodiment id) -> pack valid backbone tokens ->
//   gather noise / state -> K/V projection of every cross layer (one GEMM) ->
//   state encoder -> K x { action encoder -> 32 DiT blocks -> norm_out +
//   proj_out -> action decoder with the Euler update fused } -> scatter.
// (Isaac-GR00T architecture page, "Inference (denoising)".)  The sequence is
// captured once per (batch, seq, K, feature dtype) profile as a CUDA graph;
// replays read the caller's pointers from a small device block written by a
// one-thread kernel before each replay.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <memory>
#include <stdexcept>
#include <string>
#include <tuple>
#include <unordered_map>
#include <vector>

#include "gdit.h"
#include "attention.cuh"
#include "gemm_skinny.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "small_loop.cuh"

using namespace gdit;

namespace {

// ------------------------------------------------------------------ errors

struct GditError : std::runtime_error {
  int code;
  GditError(int c, const std::string& m) : std::runtime_error(m), code(c) {}
};

std::string fmt(const char* f, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, f);
  vsnprintf(buf, sizeof(buf), f, ap);
  va_end(ap);
  return buf;
}

#define CUDA_TRY(expr)                                                                                  \
  do {                                                                                                  \
    cudaError_t e_ = (expr);                                                                            \
    if (e_ != cudaSuccess)                                                                              \
      throw GditError(e_ == cudaErrorMemoryAllocation ? GDIT_ENOMEM : GDIT_ECUDA,                       \
                      fmt("%s failed: %s (%s:%d)", #expr, cudaGetErrorString(e_), __FILE__, __LINE__)); \
  } while (0)

#define REQUIRE(cond, ...)                                  \
  do {                                                      \
    if (!(cond)) throw GditError(GDIT_EINVAL, fmt(__VA_ARGS__)); \
  } while (0)

thread_local std::string g_create_error;

// ------------------------------------------------------------------ host bf16

uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);   // quiet NaN
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

float bf16_to_f32(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// ------------------------------------------------------------------ TMA descriptors

typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                       const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                       CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled_t encode_fn() {
  static PFN_encodeTiled_t fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    CUDA_TRY(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q));
    if (p == nullptr || q != cudaDriverEntryPointSuccess)
      throw GditError(GDIT_ECUDA, "cuTensorMapEncodeTiled not available from the driver");
    fn = reinterpret_cast<PFN_encodeTiled_t>(p);
  }
  return fn;
}

// bf16 matrix [rows, cols] with row pitch `pitch` elements; boxes of box_rows x 64,
// 128-byte swizzle (the layout the UMMA descriptors expect).
CUtensorMap make_tmap(const void* ptr, long long rows, long long cols, long long pitch, int box_rows) {
  REQUIRE(((uintptr_t)ptr & 15u) == 0, "TMA base pointer not 16-byte aligned");
  REQUIRE((pitch * 2) % 16 == 0, "TMA row pitch %lld elements is not a multiple of 16 bytes", pitch);
  REQUIRE(box_rows >= 1 && box_rows <= 256, "TMA box rows %d", box_rows);
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)std::max<long long>(rows, 1)};
  cuuint64_t strides[1] = {(cuuint64_t)(pitch * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode_fn()(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) throw GditError(GDIT_ECUDA, fmt("cuTensorMapEncodeTiled failed (%d)", (int)r));
  return m;
}

// The K/V cache as a 2-D tensor of head_dim-wide bf16 rows, for TMA boxes of
// box_rows rows with the shared-memory swizzle of one row (128 bytes for
// head_dim 64, 64 bytes for 32).
CUtensorMap make_kv_tmap(const void* ptr, long long rows, int head_dim, int box_rows) {
  REQUIRE(((uintptr_t)ptr & 15u) == 0, "TMA base pointer not 16-byte aligned");
  REQUIRE(head_dim == 32 || head_dim == 64, "head_dim %d", head_dim);
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
  cuuint32_t box[2] = {(cuuint32_t)head_dim, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode_fn()(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           head_dim == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) throw GditError(GDIT_ECUDA, fmt("cuTensorMapEncodeTiled (K/V cache) failed (%d)", (int)r));
  return m;
}

// Output map of the head-major K/V cache for the TMA-store epilogue: a 3-D
// bf16 tensor [blocks][rows][64] (one (layer, K|V, head) block of head_dim 64
// per index of the outer dimension), boxes of 64 columns x 32 rows x 1 block,
// 128-byte swizzle like the 2-D output boxes.
CUtensorMap make_kv_out_tmap(const void* ptr, long long blocks, long long rows) {
  REQUIRE(((uintptr_t)ptr & 15u) == 0, "TMA base pointer not 16-byte aligned");
  CUtensorMap m;
  cuuint64_t dims[3] = {64u, (cuuint64_t)std::max<long long>(rows, 1), (cuuint64_t)std::max<long long>(blocks, 1)};
  cuuint64_t strides[2] = {64u * 2u, (cuuint64_t)rows * 64u * 2u};
  cuuint32_t box[3] = {64u, 32u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = encode_fn()(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) throw GditError(GDIT_ECUDA, fmt("cuTensorMapEncodeTiled (K/V output) failed (%d)", (int)r));
  return m;
}

// Output map for the TMA-store epilogue: [rows, cols] with row pitch `pitch`
// elements, 32-row boxes of 128 bytes (bf16: 64 columns, f32: 32), 128-byte swizzle.
CUtensorMap make_out_tmap(const void* ptr, bool f32, long long rows, long long cols, long long pitch) {
  const int esz = f32 ? 4 : 2;
  REQUIRE(((uintptr_t)ptr & 15u) == 0, "TMA base pointer not 16-byte aligned");
  REQUIRE((pitch * esz) % 16 == 0, "output row pitch not a multiple of 16 bytes");
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)std::max<long long>(rows, 1)};
  cuuint64_t strides[1] = {(cuuint64_t)(pitch * esz)};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esz), 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode_fn()(&m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                           const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) throw GditError(GDIT_ECUDA, fmt("cuTensorMapEncodeTiled (output) failed (%d)", (int)r));
  return m;
}

// ------------------------------------------------------------------ launch helper

bool g_pdl_default = true;

template <typename... KArgs, typename... Args>
void launch_k(cudaStream_t s, bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...));
}

// ------------------------------------------------------------------ GEMM ops

struct GemmOp {
  CUtensorMap ta, tb, to;
  GemmArgs args;
  int bn = 64;
  int grid = 1;
  bool pair = false;   // CTA-pair kernel (256-row tiles, cta_group::2)
  // algorithmic accounting: rows actually multiplied are known after routing
  int rows_kind = 0;   // 0 fixed M, 1 = total valid tokens, 2 = all rows (grouped)
  long long weight_bytes = 0;
  int out_bytes = 2;
  const void* a_ptr = nullptr;   // the operands (the skinny-M kernel takes plain pointers)
  const void* b_ptr = nullptr;
  int sk_mt = 0;                 // > 0: the skinny-M kernel, row blocks of 16 sk_mt rows
  int sk_nu = 0;                 // its units of 8 features per item
  int sk_stages = 0;             // its ring depth
};

// Few rows (a batch of a few samples) use the skinny-M kernel: all SMs stream
// the weights instead of a handful of 128-row tensor-core tiles.
constexpr long long kSkinnyMaxRows = 160;
// per-item cost beyond its bytes (pipeline fill, reduction, epilogue), in
// bytes of streaming
constexpr double kSkinnyItemBytes = 64.0 * 1024;

// Row block (16 mt rows) and units per item for an [M, K] x [N, K]^T GEMM:
// the least bytes streamed by the busiest CTA, with a ring of at least 2
// stages and at most one item per SM.  False if none fits: with two rounds of
// items (FF1 at 136 rows, 3-stage rings: 18.9 us against 15.6 us for the
// tensor-core GEMM) the skinny kernel loses, while one round on a 2-stage
// ring (48-row blocks of 11 units) wins (B = 8: 8.70 ms per call against 8.76).
bool plan_skinny(long long M, int N, int K, int num_sms, int& mt, int& nu, int& stages) {
  double best = 0.0;
  bool found = false;
  const long long units = N / 8;
  for (int m : {1, 2, 3, 5}) {
    const long long rows = 16LL * m, nrb = (M + rows - 1) / rows;
    for (int u = 1; u <= sk_max_units(m); ++u) {
      const long long items = nrb * ((units + u - 1) / u);
      const int st = std::min(8, (kSkSmemMax - 1024 - sk_red_bytes(m, u) - 64) / sk_stage_bytes(m, u));
      if (st < 2 || items > num_sms) continue;
      const double cost = (double)(std::min(rows, M) + 8LL * u) * K * 2.0 + kSkinnyItemBytes;
      if (!found || cost < best) {
        found = true;
        best = cost;
        mt = m;
        nu = u;
        stages = st;
      }
    }
  }
  return found;
}

// Shapes the skinny-M kernel takes: few rows, whole units of 8 features,
// K in 64-column boxes.
bool skinny_shape_ok(long long M, int N, int K) {
  return M >= 1 && M <= kSkinnyMaxRows && N >= 8 && N % 8 == 0 && K >= 64 && K % 64 == 0;
}

// Switch a planned dense GEMM with few rows to the skinny-M kernel (plain
// [M, K] x [N, K]^T layout, one output row per input row, no split).
void enable_skinny(GemmOp& op, int num_sms) {
  GemmArgs& a = op.args;
  const bool epi_ok = a.epi == EPI_BF16 || a.epi == EPI_GELU_BF16 || a.epi == EPI_RELU_BF16 || a.epi == EPI_F32 ||
                      a.epi == EPI_RESID_F32;
  const bool aligned = ((uintptr_t)op.a_ptr % 16) == 0 && ((uintptr_t)op.b_ptr % 16) == 0;
  if (!skinny_shape_ok(a.M, a.N, a.K) || a.splits != 1 || a.num_groups != 0 || a.m_dev != nullptr || a.nblk != 0 ||
      a.in_group != 0x7fffffff || a.out_off != 0 || !epi_ok || !aligned)
    return;
  int mt, nu, stages;
  if (!plan_skinny(a.M, a.N, a.K, num_sms, mt, nu, stages)) return;
  op.sk_mt = mt;
  op.sk_nu = nu;
  op.sk_stages = stages;
  op.ta = make_tmap(op.a_ptr, a.M, a.K, a.K, 16 * mt);
  op.tb = make_tmap(op.b_ptr, a.N, a.K, a.K, 8 * nu);
  const long long items = ((a.M + 16LL * mt - 1) / (16LL * mt)) * ((a.N / 8 + nu - 1) / nu);
  op.grid = (int)std::min<long long>(items, num_sms);
  op.pair = false;
  a.tma_out = 0;
}

// Switch a planned dense GEMM to the TMA-store epilogue when its output is a
// plain [M, N] matrix (no split-K, no row remap, no column blocking).
void enable_tma_out(GemmOp& op) {
  GemmArgs& a = op.args;
  const bool plain_epi = a.epi == EPI_BF16 || a.epi == EPI_GELU_BF16 || a.epi == EPI_RELU_BF16 ||
                         a.epi == EPI_F32 || a.epi == EPI_RESID_F32;
  if (a.splits != 1 || a.num_groups != 0 || a.m_dev != nullptr || a.nblk != 0 || a.in_group != 0x7fffffff ||
      a.out_off != 0 || !plain_epi || op.bn < 64)
    return;
  const bool f32 = a.epi == EPI_F32 || a.epi == EPI_RESID_F32;
  op.to = make_out_tmap(a.out, f32, a.M, a.N, a.ldo);
  a.tma_out = 1;
}

// Move a dense TMA-store GEMM to the CTA-pair kernel when its 256-row tiles
// still occupy about as many SMs as the 128-row tiles would: the pair tile
// reads a third less operand data from L2 per unit of tensor work.
void enable_pair(GemmOp& op, const void* A, const void* W, int num_sms) {
  GemmArgs& a = op.args;
  if (!a.tma_out || (op.bn != 256 && op.bn != 128) || a.m_dev != nullptr) return;
  const long long nt = (a.N + op.bn - 1) / op.bn;
  const long long pair_tiles = ((a.M + kPairBM - 1) / kPairBM) * nt;
  const long long one_tiles = ((a.M + kBM - 1) / kBM) * nt;
  const long long pair_sms = std::min<long long>(2 * pair_tiles, num_sms - num_sms % 2);
  const long long one_sms = std::min<long long>(one_tiles, num_sms);
  if (10 * pair_sms < 9 * one_sms) return;
  op.pair = true;
  op.ta = make_tmap(A, a.M, a.K, a.K, 128);
  op.tb = make_tmap(W, a.N, a.K, a.K, op.bn / 2);
  op.grid = (int)(2 * std::min<long long>(pair_tiles, num_sms / 2));
}

template <int BN>
void set_gemm_attr() {
  CUDA_TRY(cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<BN>::SMEM));
}

template <int BN>
void set_gemm_pair_attr() {
  CUDA_TRY(cudaFuncSetAttribute(gemm_tc_pair_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GemmPairCfg<BN>::SMEM));
}

// CTA-pair GEMM: clusters of two CTAs (grid even), optionally after the
// previous kernel by programmatic dependent launch.
template <int BN>
void launch_gemm_pair(const GemmOp& op, const GemmArgs& a, cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(op.grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = GemmPairCfg<BN>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_tc_pair_kernel<BN>, op.ta, op.tb, op.to, a));
}

void launch_gemm_skinny(const GemmOp& op, const GemmArgs& a, cudaStream_t s, bool pdl) {
  SkinnyArgs k;
  k.W = static_cast<const __nv_bfloat16*>(op.b_ptr);
  k.bias = a.bias;
  k.out = a.out;
  k.ldo = a.ldo;
  k.M = a.M;
  k.N = a.N;
  k.K = a.K;
  k.epi = a.epi;
  k.nu = op.sk_nu;
  k.stages = op.sk_stages;
  k.err = a.err;
  const int smem = sk_smem_bytes(op.sk_mt, op.sk_nu, op.sk_stages);
  const dim3 grid(op.grid), block(kSkThreads);
  switch (op.sk_mt) {
    case 1: launch_k(s, pdl, gemm_skinny_kernel<1>, grid, block, smem, op.ta, op.tb, k); break;
    case 2: launch_k(s, pdl, gemm_skinny_kernel<2>, grid, block, smem, op.ta, op.tb, k); break;
    case 3: launch_k(s, pdl, gemm_skinny_kernel<3>, grid, block, smem, op.ta, op.tb, k); break;
    case 5: launch_k(s, pdl, gemm_skinny_kernel<5>, grid, block, smem, op.ta, op.tb, k); break;
    default: throw GditError(GDIT_EINVAL, fmt("bad skinny row block %d", op.sk_mt));
  }
}

void launch_gemm(const GemmOp& op, const GemmArgs& a, cudaStream_t s, bool pdl) {
  if (op.sk_mt > 0) {
    launch_gemm_skinny(op, a, s, pdl);
    return;
  }
  if (op.pair) {
    if (op.bn == 256)
      launch_gemm_pair<256>(op, a, s, pdl);
    else if (op.bn == 128)
      launch_gemm_pair<128>(op, a, s, pdl);
    else
      throw GditError(GDIT_EINVAL, fmt("bad CTA-pair tile width %d", op.bn));
    return;
  }
  switch (op.bn) {
    case 32:
      launch_k(s, pdl, gemm_tc_kernel<32>, dim3(op.grid), dim3(kGemmThreads), GemmCfg<32>::SMEM, op.ta, op.tb, op.to, a);
      break;
    case 64:
      launch_k(s, pdl, gemm_tc_kernel<64>, dim3(op.grid), dim3(kGemmThreads), GemmCfg<64>::SMEM, op.ta, op.tb, op.to, a);
      break;
    case 128:
      launch_k(s, pdl, gemm_tc_kernel<128>, dim3(op.grid), dim3(kGemmThreads), GemmCfg<128>::SMEM, op.ta, op.tb, op.to, a);
      break;
    case 256:
      launch_k(s, pdl, gemm_tc_kernel<256>, dim3(op.grid), dim3(kGemmThreads), GemmCfg<256>::SMEM, op.ta, op.tb, op.to, a);
      break;
    default:
      throw GditError(GDIT_EINVAL, fmt("bad GEMM tile width %d", op.bn));
  }
}

GemmArgs default_args() {
  GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.splits = 1;
  a.in_group = 0x7fffffff;
  a.in_skip = 0;
  a.out_group = 0;
  a.out_off = 0;
  return a;
}

constexpr long long kWsFloats = 16ll << 20;   // split-K partials (64 MB)
// guard bands of the range-checked build (a multiple of 256 bytes: the
// buffers keep cudaMalloc's alignment)
constexpr size_t kGuardBytes = GDIT_CHECKED ? 4096 : 0;
constexpr uint8_t kGuardByte = 0xA5;
constexpr int kHostChunks = 4;                // sample chunks of the host-buffer entry point
constexpr int kSmallMaxPhases = 64 * (5 * kSmallMaxLayers + 6);
constexpr int kCounters = 1 << 16;

// Picks the tile width and split-K factor.  Large row counts use wide tiles,
// small ones narrow tiles.  The planned GEMMs never split K: measured on the
// workloads from B = 1 to 256, a split (partials written, a tile counter, the
// last CTA of a tile reducing them) cost more than the SMs it filled, and it
// rules out the TMA-store and CTA-pair epilogues (no split: sweep8 11.4 ->
// 9.3 ms, sweep32 17.3 -> 11.9, sweep128 27.2 -> 17.4, batched 18.3 -> 12.9,
// B = 256 unchanged).  The split-K kernel path serves the GEMM entry points
// that take an explicit split count.
void choose_tiling(long long rows_est, int groups_est, int N, int K, int num_sms, long long ws_rows, int& bn,
                   int& splits) {
  (void)groups_est;
  (void)K;
  (void)num_sms;
  (void)ws_rows;
  // (measured: 256 from 512 rows; 128 from 256 rows, e.g. long_chunk's 408,
  // 7 % faster there than 64; 64 below, e.g. 136 rows at B = 8)
  if (N <= 32)
    bn = 32;
  else if (rows_est >= 512 && N % 256 == 0)
    bn = 256;
  else if (N >= 16384 && N % 256 == 0)
    bn = 256;   // few rows, very wide N (the K/V projection of a few hundred tokens): each column tile
                // re-reads all the rows of A, so wide tiles read A 4x less often than 64-wide ones
  else if (rows_est >= 256 && N % 128 == 0)
    bn = 128;
  else
    bn = 64;
  splits = 1;
}

// ------------------------------------------------------------------ weights

struct WeightSpec {
  std::string name;
  std::vector<int64_t> shape;
};

struct DevModel {
  // bf16 matrices
  __nv_bfloat16 *t1w, *t2w, *ada_w, *wkv, *proj_w;
  float* vlln_g = nullptr;   // optional vision-language layer norm (f32 [Dvl])
  float* vlln_b = nullptr;
  std::vector<__nv_bfloat16*> wq;     // per layer: [3D, D] (self) or [D, D] (cross)
  std::vector<__nv_bfloat16*> wo, wff1, wff2;
  __nv_bfloat16 *ws1t, *ws2t, *wa1t, *wa2at, *wa2taut, *wa3t, *wd1t, *wd2t;
  // f32 vectors
  float *t1b, *t2b, *ada_b, *bkv, *proj_b;
  std::vector<float*> bq, bo, ln3g, ln3b, bff1, bff2;
  float *bs1, *bs2, *ba1, *ba2, *ba3, *bd1, *bd2;
};

struct Tables {
  int K = 0;
  float* ada = nullptr;   // [K][L+1][2D]
  float* tw2 = nullptr;   // [K][C][D]
  std::vector<float> td;  // host copy
};

struct Profile {
  int B, S, K, bf16;
  GemmOp kv, st1, st2, a1, a2, a3, proj, d1, d2;
  std::vector<GemmOp> q, o, ff1, ff2;
  cudaGraphExec_t exec = nullptr;        // the whole call
  cudaGraphExec_t exec_main = nullptr;   // the call after the K/V projection (host-buffer entry point)
  // single-sample profiles run the K-step loop as one persistent kernel
  bool small = false;
  SmallPlan* small_plan = nullptr;   // device copies, one per sample
  int small_phases = 0;              // per sample
  int small_groups = 0;              // samples (CTA groups) of the loop
  int small_gsize = 0;               // CTAs per group
  bool small_grouped = false;        // several groups, or more than kSmallMaxUnits units of a CTA in some linear
};

struct KStat {
  std::string name;
  int launches = 0;
  double ms = 0, flops = 0, bytes = 0;
};

struct Recorder {
  struct Ev {
    int cls;
    cudaEvent_t a, b;
    double flops, bytes;
    const GemmOp* op;
  };
  std::vector<Ev> evs;
  std::vector<std::string> names;
  int cls(const std::string& n) {
    for (size_t i = 0; i < names.size(); ++i)
      if (names[i] == n) return (int)i;
    names.push_back(n);
    return (int)names.size() - 1;
  }
};

}  // namespace

struct gdit_handle {
  gdit_config cfg;
  int L, D, F, Dvl, A, Sd, H, C, Tf, N, Lc;
  int num_sms = 148;
  bool pdl = true;
  bool use_graph = true;
  bool strict = false;
  std::string last_error;

  // device memory
  std::vector<void*> allocs;
  DevModel w;
  __nv_bfloat16 *xp, *kv, *u, *qkv, *o, *f, *xb, *abf, *zbf, *ybf, *rbf, *sb, *s1;
  uint8_t* kflag;           // image flag of each packed backbone token
  float *h, *x, *sfeat, *ws;
  int *perm, *seg, *vofs, *kspan, *counters;
  int* phase_counters;      // per-phase arrival counters of the single-sample loop
  SmallPhase* phase_table;  // per-phase descriptors of the single-sample loop
  float2* ln_part;          // LayerNorm statistics pieces of the single-sample loop
  uint8_t* bad;
  unsigned* status;
  IoPtrs* io;
  long long max_tok;

  // per-K tables and per-profile plans
  std::map<int, Tables> tables;
  std::map<std::tuple<int, int, int, int>, std::unique_ptr<Profile>> profiles;
  cudaStream_t cap_stream = nullptr;
  cudaStream_t last_stream = nullptr;

  // host-buffer staging (gdit_get_action_host): the features are copied in
  // sample chunks on copy_stream, each chunk packed and projected to K/V as
  // soon as it has landed
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t small_ev = nullptr;           // the small inputs have landed
  cudaEvent_t chunk_ev[kHostChunks] = {};
  void* st_feats = nullptr;
  size_t st_feats_bytes = 0;
  uint8_t* st_mask = nullptr;
  float *st_state = nullptr, *st_noise = nullptr, *st_out = nullptr;
  int32_t* st_ids = nullptr;

  Recorder* rec = nullptr;   // non-null during gdit_profile_get_action
  int last_B = 0;

  // Host-side fault injection, read from GDIT_FAULT at create
  // ("alloc:N,graph:N,upload:N"): the N-th device allocation, CUDA-graph
  // instantiation or weight upload of this handle (counted from 1) fails the
  // way the real call would.  Nothing on the device is made to fail.
  struct Faults {
    long long alloc = 0, graph = 0, upload = 0;      // 0: never
    long long n_alloc = 0, n_graph = 0, n_upload = 0;
  } fault;

  // Range-checked builds put a guard band of kGuardBytes before and after
  // every allocation, filled with kGuardByte; gdit_check_canaries counts the
  // guard bytes that changed (a write past either end of a buffer).
  struct Guarded {
    uint8_t* base;      // start of the front band
    size_t bytes;       // the buffer between the bands
  };
  std::vector<Guarded> guarded_allocs;

  template <typename T>
  T* dalloc(size_t count) {
    if (++fault.n_alloc == fault.alloc)
      throw GditError(GDIT_ENOMEM, fmt("injected fault: device allocation %lld failed", fault.n_alloc));
    void* p = nullptr;
    const size_t bytes = std::max<size_t>(count * sizeof(T), 256);
    CUDA_TRY(cudaMalloc(&p, bytes + 2 * kGuardBytes));
    allocs.push_back(p);
    if (kGuardBytes > 0) {
      uint8_t* b = static_cast<uint8_t*>(p);
      CUDA_TRY(cudaMemset(b, kGuardByte, kGuardBytes));
      CUDA_TRY(cudaMemset(b + kGuardBytes + bytes, kGuardByte, kGuardBytes));
      guarded_allocs.push_back({b, bytes});
    }
    return reinterpret_cast<T*>(static_cast<uint8_t*>(p) + kGuardBytes);
  }

  // host -> device copy of weight data (synchronous)
  void upload(void* dst, const void* src, size_t bytes) {
    if (++fault.n_upload == fault.upload)
      throw GditError(GDIT_ECUDA, fmt("injected fault: weight upload %lld failed", fault.n_upload));
    CUDA_TRY(cudaMemcpy(dst, src, bytes, cudaMemcpyHostToDevice));
  }
};

namespace {

// ------------------------------------------------------------------ validation

// GDIT_FAULT = comma-separated "kind:N" with kind alloc, graph or upload and
// N >= 1 (see gdit_handle::Faults).
void parse_faults(const char* spec, gdit_handle::Faults& f) {
  if (spec == nullptr || spec[0] == '\0') return;
  std::string s(spec);
  size_t pos = 0;
  while (pos <= s.size()) {
    size_t end = s.find(',', pos);
    if (end == std::string::npos) end = s.size();
    const std::string item = s.substr(pos, end - pos);
    const size_t colon = item.find(':');
    REQUIRE(colon != std::string::npos, "GDIT_FAULT item '%s' is not kind:N", item.c_str());
    const std::string kind = item.substr(0, colon);
    char* stop = nullptr;
    const long long n = std::strtoll(item.c_str() + colon + 1, &stop, 10);
    REQUIRE(stop != nullptr && *stop == '\0' && n >= 1, "GDIT_FAULT item '%s': N must be an integer >= 1",
            item.c_str());
    if (kind == "alloc")
      f.alloc = n;
    else if (kind == "graph")
      f.graph = n;
    else if (kind == "upload")
      f.upload = n;
    else
      throw GditError(GDIT_EINVAL, fmt("GDIT_FAULT kind '%s' is not alloc, graph or upload", kind.c_str()));
    pos = end + 1;
  }
}

void validate_config(const gdit_config& c) {
  REQUIRE(c.num_layers >= 2 && c.num_layers % 2 == 0, "num_layers must be even and >= 2 (got %d)", c.num_layers);
  REQUIRE(c.head_dim == 32 || c.head_dim == 64, "head_dim must be 32 or 64 (got %d)", c.head_dim);
  REQUIRE(c.num_heads >= 1 && c.hidden == c.num_heads * c.head_dim, "hidden (%d) must equal num_heads * head_dim",
          c.hidden);
  REQUIRE(c.hidden == 128 || c.hidden == 256 || c.hidden == 512 || c.hidden == 1024 || c.hidden == 2048,
          "hidden must be one of 128, 256, 512, 1024, 2048 (got %d)", c.hidden);
  REQUIRE(c.mlp_hidden >= 64 && c.mlp_hidden % 64 == 0, "mlp_hidden must be a positive multiple of 64");
  REQUIRE(c.backbone_dim >= 64 && c.backbone_dim % 64 == 0, "backbone_dim must be a positive multiple of 64");
  REQUIRE(c.action_dim >= 32 && c.action_dim <= 256 && c.action_dim % 32 == 0,
          "action_dim must be a multiple of 32 in [32, 256] (got %d)", c.action_dim);
  REQUIRE(c.state_dim >= 32 && c.state_dim <= 256 && c.state_dim % 32 == 0,
          "state_dim must be a multiple of 32 in [32, 256] (got %d)", c.state_dim);
  REQUIRE(c.action_horizon >= 1 && c.action_horizon + 1 <= 64, "action_horizon must be in [1, 63] (got %d)",
          c.action_horizon);
  REQUIRE(c.num_embodiments >= 1 && c.num_embodiments <= kMaxGroups, "num_embodiments must be in [1, %d]",
          kMaxGroups);
  REQUIRE(c.max_batch >= 1 && c.max_batch <= kMaxBatch, "max_batch must be in [1, %d]", kMaxBatch);
  REQUIRE(c.max_backbone_seq >= 1 && c.max_backbone_seq <= 65536, "max_backbone_seq must be in [1, 65536]");
  REQUIRE(c.time_freq_dim >= 2 && c.time_freq_dim % 2 == 0, "time_freq_dim must be even and >= 2");
  REQUIRE(c.num_timestep_buckets >= 1, "num_timestep_buckets must be >= 1");
  REQUIRE(c.ln_eps > 0.0f, "ln_eps must be > 0");
  REQUIRE(c.attend_text_every_n_blocks >= 0, "attend_text_every_n_blocks must be >= 0");
}

// Which keys cross layer `layer` attends to (AlternateVLDiT image/text split):
// -1 every valid key (no split), 0 the text keys, 1 the image keys.
int cross_key_sel(const gdit_config& c, int layer) {
  const int n = c.attend_text_every_n_blocks;
  if (n <= 0) return -1;
  return layer % (2 * n) == 0 ? 0 : 1;
}

std::vector<WeightSpec> weight_specs(const gdit_config& c) {
  const int64_t D = c.hidden, F = c.mlp_hidden, C = c.num_embodiments;
  std::vector<WeightSpec> v;
  auto add = [&](const std::string& n, std::vector<int64_t> s) { v.push_back({n, s}); };
  add("t_enc.l1.w", {D, c.time_freq_dim});
  add("t_enc.l1.b", {D});
  add("t_enc.l2.w", {D, D});
  add("t_enc.l2.b", {D});
  for (int l = 0; l < c.num_layers; ++l) {
    const int64_t din = (l % 2 == 0) ? c.backbone_dim : D;
    const std::string p = "blk" + std::to_string(l) + ".";
    add(p + "ada.w", {2 * D, D});
    add(p + "ada.b", {2 * D});
    add(p + "q.w", {D, D});
    add(p + "q.b", {D});
    add(p + "k.w", {D, din});
    add(p + "k.b", {D});
    add(p + "v.w", {D, din});
    add(p + "v.b", {D});
    add(p + "o.w", {D, D});
    add(p + "o.b", {D});
    add(p + "ln3.g", {D});
    add(p + "ln3.b", {D});
    add(p + "ff1.w", {F, D});
    add(p + "ff1.b", {F});
    add(p + "ff2.w", {D, F});
    add(p + "ff2.b", {D});
  }
  add("out.ada.w", {2 * D, D});
  add("out.ada.b", {2 * D});
  add("out.proj.w", {D, D});
  add("out.proj.b", {D});
  add("state_enc.l1.W", {C, c.state_dim, D});
  add("state_enc.l1.b", {C, D});
  add("state_enc.l2.W", {C, D, D});
  add("state_enc.l2.b", {C, D});
  add("act_enc.W1.W", {C, c.action_dim, D});
  add("act_enc.W1.b", {C, D});
  add("act_enc.W2.W", {C, 2 * D, D});
  add("act_enc.W2.b", {C, D});
  add("act_enc.W3.W", {C, D, D});
  add("act_enc.W3.b", {C, D});
  add("act_dec.l1.W", {C, D, D});
  add("act_dec.l1.b", {C, D});
  add("act_dec.l2.W", {C, D, c.action_dim});
  add("act_dec.l2.b", {C, c.action_dim});
  return v;
}

// Host view of one weight as f32 values (converted from bf16 if needed).
struct HostW {
  const gdit_tensor* t;
  int64_t numel;
  float at(int64_t i) const {
    if (t->dtype == GDIT_F32) return static_cast<const float*>(t->host_ptr)[i];
    return bf16_to_f32(static_cast<const uint16_t*>(t->host_ptr)[i]);
  }
};

std::unordered_map<std::string, HostW> check_weights(const gdit_config& c, const gdit_tensor* ws, int n) {
  REQUIRE(ws != nullptr || n == 0, "weights is NULL");
  std::unordered_map<std::string, HostW> got;
  for (int i = 0; i < n; ++i) {
    const gdit_tensor& t = ws[i];
    REQUIRE(t.name != nullptr, "weight %d has no name", i);
    REQUIRE(got.find(t.name) == got.end(), "weight '%s' given twice", t.name);
    REQUIRE(t.dtype == GDIT_F32 || t.dtype == GDIT_BF16, "weight '%s': dtype must be GDIT_F32 or GDIT_BF16",
            t.name);
    REQUIRE(t.ndim >= 1 && t.ndim <= 4 && t.shape != nullptr, "weight '%s': bad ndim/shape", t.name);
    REQUIRE(t.host_ptr != nullptr, "weight '%s': host_ptr is NULL", t.name);
    int64_t numel = 1;
    for (int d = 0; d < t.ndim; ++d) numel *= t.shape[d];
    got[t.name] = HostW{&t, numel};
  }
  const auto specs = weight_specs(c);
  for (const auto& s : specs) {
    auto it = got.find(s.name);
    REQUIRE(it != got.end(), "missing weight '%s'", s.name.c_str());
    const gdit_tensor* t = it->second.t;
    bool ok = t->ndim == (int)s.shape.size();
    for (int d = 0; ok && d < t->ndim; ++d) ok = t->shape[d] == s.shape[d];
    if (!ok) {
      std::string want, have;
      for (auto x : s.shape) want += std::to_string(x) + ",";
      for (int d = 0; d < t->ndim; ++d) have += std::to_string(t->shape[d]) + ",";
      throw GditError(GDIT_EINVAL, fmt("weight '%s' has shape [%s] but [%s] is required", s.name.c_str(),
                                       have.c_str(), want.c_str()));
    }
  }
  // optional: the vision-language layer norm of the backbone features
  size_t optional = 0;
  if (got.count("vlln.g") || got.count("vlln.b")) {
    REQUIRE(got.count("vlln.g") && got.count("vlln.b"), "vlln.g and vlln.b must be given together");
    for (const char* n : {"vlln.g", "vlln.b"}) {
      const gdit_tensor* t = got.at(n).t;
      REQUIRE(t->ndim == 1 && t->shape[0] == c.backbone_dim, "weight '%s' must have shape [%d]", n, c.backbone_dim);
    }
    REQUIRE(c.backbone_dim % 256 == 0 && c.backbone_dim <= 4096,
            "vlln needs backbone_dim a multiple of 256 and <= 4096 (got %d)", c.backbone_dim);
    optional = 2;
  }
  REQUIRE(got.size() == specs.size() + optional, "%zu unknown weight name(s) given (expected exactly %zu tensors)",
          got.size() - specs.size() - optional, specs.size() + optional);
  return got;
}

// ------------------------------------------------------------------ upload

struct Uploader {
  gdit_handle* h;
  std::vector<uint16_t> hb;
  std::vector<float> hf;

  __nv_bfloat16* mat(size_t n) { return h->dalloc<__nv_bfloat16>(n); }

  // rows of `src` (a [rows, cols] row-major weight) -> bf16 at dst + row_off * cols
  void put_rows(__nv_bfloat16* dst, const HostW& w, size_t count) {
    hb.resize(count);
    for (size_t i = 0; i < count; ++i) hb[i] = f32_to_bf16_rne(w.at((int64_t)i));
    h->upload(dst, hb.data(), count * 2);
  }
  __nv_bfloat16* matrix(const HostW& w) {
    __nv_bfloat16* d = mat((size_t)w.numel);
    put_rows(d, w, (size_t)w.numel);
    return d;
  }
  // [C, in, out] -> [C, out, in] restricted to input rows [in0, in0 + nin)
  __nv_bfloat16* cat_transposed(const HostW& w, int C, int in, int out, int in0, int nin) {
    __nv_bfloat16* d = mat((size_t)C * out * nin);
    hb.resize((size_t)C * out * nin);
    for (int c = 0; c < C; ++c)
      for (int o = 0; o < out; ++o)
        for (int i = 0; i < nin; ++i)
          hb[((size_t)c * out + o) * nin + i] = f32_to_bf16_rne(w.at(((int64_t)c * in + in0 + i) * out + o));
    h->upload(d, hb.data(), hb.size() * 2);
    return d;
  }
  float* vec(const HostW& w) {
    float* d = h->dalloc<float>((size_t)w.numel);
    hf.resize((size_t)w.numel);
    for (int64_t i = 0; i < w.numel; ++i) hf[i] = w.at(i);
    h->upload(d, hf.data(), hf.size() * 4);
    return d;
  }
  void vec_into(float* d, const HostW& w) {
    hf.resize((size_t)w.numel);
    for (int64_t i = 0; i < w.numel; ++i) hf[i] = w.at(i);
    h->upload(d, hf.data(), hf.size() * 4);
  }
};

void upload_model(gdit_handle* h, const std::unordered_map<std::string, HostW>& W) {
  Uploader up{h, {}, {}};
  const int D = h->D, F = h->F, L = h->L, C = h->C, Dvl = h->Dvl, A = h->A, Sd = h->Sd;
  DevModel& m = h->w;
  auto get = [&](const std::string& n) -> const HostW& { return W.at(n); };
  if (W.count("vlln.g")) {
    m.vlln_g = up.vec(get("vlln.g"));
    m.vlln_b = up.vec(get("vlln.b"));
  }
  m.t1w = up.matrix(get("t_enc.l1.w"));
  m.t1b = up.vec(get("t_enc.l1.b"));
  m.t2w = up.matrix(get("t_enc.l2.w"));
  m.t2b = up.vec(get("t_enc.l2.b"));
  // AdaLN weights of the L blocks and of norm_out, contiguous: [(L+1)][2D][D]
  m.ada_w = up.mat((size_t)(L + 1) * 2 * D * D);
  m.ada_b = h->dalloc<float>((size_t)(L + 1) * 2 * D);
  for (int l = 0; l <= L; ++l) {
    const std::string p = l < L ? "blk" + std::to_string(l) + ".ada" : std::string("out.ada");
    up.put_rows(m.ada_w + (size_t)l * 2 * D * D, get(p + ".w"), (size_t)2 * D * D);
    up.vec_into(m.ada_b + (size_t)l * 2 * D, get(p + ".b"));
  }
  // K/V weights of all cross layers: [Lc][2][D][Dvl] rows, biases [Lc][2D]
  m.wkv = up.mat((size_t)h->Lc * 2 * D * Dvl);
  m.bkv = h->dalloc<float>((size_t)h->Lc * 2 * D);
  m.wq.resize(L);
  m.bq.resize(L);
  m.wo.resize(L);
  m.bo.resize(L);
  m.ln3g.resize(L);
  m.ln3b.resize(L);
  m.wff1.resize(L);
  m.bff1.resize(L);
  m.wff2.resize(L);
  m.bff2.resize(L);
  for (int l = 0; l < L; ++l) {
    const std::string p = "blk" + std::to_string(l) + ".";
    if (l % 2 == 0) {
      const int li = l / 2;
      up.put_rows(m.wkv + (size_t)li * 2 * D * Dvl, get(p + "k.w"), (size_t)D * Dvl);
      up.put_rows(m.wkv + (size_t)li * 2 * D * Dvl + (size_t)D * Dvl, get(p + "v.w"), (size_t)D * Dvl);
      up.vec_into(m.bkv + (size_t)li * 2 * D, get(p + "k.b"));
      up.vec_into(m.bkv + (size_t)li * 2 * D + D, get(p + "v.b"));
      m.wq[l] = up.matrix(get(p + "q.w"));
      m.bq[l] = up.vec(get(p + "q.b"));
    } else {
      m.wq[l] = up.mat((size_t)3 * D * D);
      up.put_rows(m.wq[l], get(p + "q.w"), (size_t)D * D);
      up.put_rows(m.wq[l] + (size_t)D * D, get(p + "k.w"), (size_t)D * D);
      up.put_rows(m.wq[l] + (size_t)2 * D * D, get(p + "v.w"), (size_t)D * D);
      m.bq[l] = h->dalloc<float>((size_t)3 * D);
      up.vec_into(m.bq[l], get(p + "q.b"));
      up.vec_into(m.bq[l] + D, get(p + "k.b"));
      up.vec_into(m.bq[l] + 2 * D, get(p + "v.b"));
    }
    m.wo[l] = up.matrix(get(p + "o.w"));
    m.bo[l] = up.vec(get(p + "o.b"));
    m.ln3g[l] = up.vec(get(p + "ln3.g"));
    m.ln3b[l] = up.vec(get(p + "ln3.b"));
    m.wff1[l] = up.matrix(get(p + "ff1.w"));
    m.bff1[l] = up.vec(get(p + "ff1.b"));
    m.wff2[l] = up.matrix(get(p + "ff2.w"));
    m.bff2[l] = up.vec(get(p + "ff2.b"));
  }
  m.proj_w = up.matrix(get("out.proj.w"));
  m.proj_b = up.vec(get("out.proj.b"));
  // category-specific weights, transposed to [C][out][in] (K-major for the GEMM)
  m.ws1t = up.cat_transposed(get("state_enc.l1.W"), C, Sd, D, 0, Sd);
  m.bs1 = up.vec(get("state_enc.l1.b"));
  m.ws2t = up.cat_transposed(get("state_enc.l2.W"), C, D, D, 0, D);
  m.bs2 = up.vec(get("state_enc.l2.b"));
  m.wa1t = up.cat_transposed(get("act_enc.W1.W"), C, A, D, 0, A);
  m.ba1 = up.vec(get("act_enc.W1.b"));
  m.wa2at = up.cat_transposed(get("act_enc.W2.W"), C, 2 * D, D, 0, D);       // action half
  m.wa2taut = up.cat_transposed(get("act_enc.W2.W"), C, 2 * D, D, D, D);     // timestep half
  m.ba2 = up.vec(get("act_enc.W2.b"));
  m.wa3t = up.cat_transposed(get("act_enc.W3.W"), C, D, D, 0, D);
  m.ba3 = up.vec(get("act_enc.W3.b"));
  m.wd1t = up.cat_transposed(get("act_dec.l1.W"), C, D, D, 0, D);
  m.bd1 = up.vec(get("act_dec.l1.b"));
  m.wd2t = up.cat_transposed(get("act_dec.l2.W"), C, D, A, 0, D);
  m.bd2 = up.vec(get("act_dec.l2.b"));
}

void alloc_workspace(gdit_handle* h) {
  const long long Bm = h->cfg.max_batch, Sm = h->cfg.max_backbone_seq;
  const int D = h->D, F = h->F, N = h->N, H = h->H, A = h->A;
  h->max_tok = Bm * Sm;
  h->xp = h->dalloc<__nv_bfloat16>((size_t)h->max_tok * h->Dvl);
  h->kflag = h->dalloc<uint8_t>((size_t)h->max_tok);
  h->kv = h->dalloc<__nv_bfloat16>((size_t)h->Lc * h->max_tok * 2 * D);
  h->h = h->dalloc<float>((size_t)Bm * N * D);
  h->u = h->dalloc<__nv_bfloat16>((size_t)Bm * N * D);
  h->qkv = h->dalloc<__nv_bfloat16>((size_t)Bm * N * 3 * D);
  h->o = h->dalloc<__nv_bfloat16>((size_t)Bm * N * D);
  h->f = h->dalloc<__nv_bfloat16>((size_t)Bm * N * F);
  h->x = h->dalloc<float>((size_t)Bm * H * A);
  h->xb = h->dalloc<__nv_bfloat16>((size_t)Bm * H * A);
  h->abf = h->dalloc<__nv_bfloat16>((size_t)Bm * H * D);
  h->zbf = h->dalloc<__nv_bfloat16>((size_t)Bm * H * D);
  h->ybf = h->dalloc<__nv_bfloat16>((size_t)Bm * H * D);
  h->rbf = h->dalloc<__nv_bfloat16>((size_t)Bm * H * D);
  h->sb = h->dalloc<__nv_bfloat16>((size_t)Bm * h->Sd);
  h->s1 = h->dalloc<__nv_bfloat16>((size_t)Bm * D);
  h->sfeat = h->dalloc<float>((size_t)Bm * D);
  h->perm = h->dalloc<int>((size_t)Bm);
  h->seg = h->dalloc<int>((size_t)h->C + 1);
  h->vofs = h->dalloc<int>((size_t)Bm + 1);
  h->kspan = h->dalloc<int>((size_t)2 * Bm);
  h->bad = h->dalloc<uint8_t>((size_t)Bm);
  h->status = h->dalloc<unsigned>(1);
  h->io = h->dalloc<IoPtrs>(1);
  h->ws = h->dalloc<float>((size_t)kWsFloats);
  h->counters = h->dalloc<int>((size_t)kCounters);
  h->phase_counters = h->dalloc<int>((size_t)kSmallMaxPhases);
  h->phase_table = h->dalloc<SmallPhase>((size_t)kSmallMaxPhases);
  h->ln_part = h->dalloc<float2>((size_t)kSmallMaxGroups * kSmallMaxTok * kLnPieces);
  CUDA_TRY(cudaMemset(h->counters, 0, sizeof(int) * kCounters));
  CUDA_TRY(cudaMemset(h->status, 0, sizeof(unsigned)));
  CUDA_TRY(cudaMemset(h->h, 0, sizeof(float) * (size_t)Bm * N * D));
}

template <typename K>
void max_shared_carveout(K* kern) {
  CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                (int)cudaSharedmemCarveoutMaxShared));
}

// CTAs of the warp-schedule attention kernel resident per SM, by (MT == 4, DH == 64)
int g_attn_warp_ctas[2][2];

template <int MT, int DH>
void set_attn_attrs() {
  CUDA_TRY(cudaFuncSetAttribute(attention_split_kernel<MT, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                AttnSmem<MT, DH>::SPLIT_TOTAL));
  CUDA_TRY(cudaFuncSetAttribute(attention_warp_kernel<MT, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                AttnSmem<MT, DH, kWarpRing>::WARP_TOTAL));
  max_shared_carveout(attention_split_kernel<MT, DH>);
  max_shared_carveout(attention_warp_kernel<MT, DH>);
  int n = 0;
  CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, attention_warp_kernel<MT, DH>, kAttnThreads,
                                                         AttnSmem<MT, DH, kWarpRing>::WARP_TOTAL));
  g_attn_warp_ctas[MT == 4][DH == 64] = n > 0 ? n : 1;
}

void set_kernel_attrs() {
  static bool done = false;
  if (done) return;
  // One shared-memory carveout for every kernel, so consecutive launches never
  // wait for an SM to repartition L1 / shared memory.
  max_shared_carveout(route_kernel);
  max_shared_carveout(pack_features_kernel);
  max_shared_carveout(gather_inputs_kernel);
  max_shared_carveout(scatter_out_kernel);
  max_shared_carveout(set_io_kernel);
  max_shared_carveout(layernorm_kernel<1>);
  max_shared_carveout(layernorm_kernel<2>);
  max_shared_carveout(layernorm_kernel<4>);
  max_shared_carveout(layernorm_kernel<8>);
  max_shared_carveout(layernorm_kernel<16>);
  max_shared_carveout(gemm_tc_kernel<32>);
  max_shared_carveout(gemm_tc_kernel<64>);
  max_shared_carveout(gemm_tc_kernel<128>);
  max_shared_carveout(gemm_tc_kernel<256>);
  set_gemm_attr<32>();
  set_gemm_attr<64>();
  set_gemm_attr<128>();
  set_gemm_attr<256>();
  set_gemm_pair_attr<128>();
  set_gemm_pair_attr<256>();
  max_shared_carveout(gemm_tc_pair_kernel<128>);
  max_shared_carveout(gemm_tc_pair_kernel<256>);
  CUDA_TRY(cudaFuncSetAttribute(small_loop_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SmallSmem<64>::TOTAL));
  CUDA_TRY(cudaFuncSetAttribute(small_loop_kernel<32, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SmallSmem<32>::TOTAL));
  CUDA_TRY(cudaFuncSetAttribute(small_loop_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SmallSmem<64>::TOTAL));
  CUDA_TRY(cudaFuncSetAttribute(small_loop_kernel<32, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SmallSmem<32>::TOTAL));
  max_shared_carveout(small_loop_kernel<64, false>);
  max_shared_carveout(small_loop_kernel<32, false>);
  max_shared_carveout(small_loop_kernel<64, true>);
  max_shared_carveout(small_loop_kernel<32, true>);
  max_shared_carveout(small_describe_kernel);
  for (const void* f : {(const void*)gemm_skinny_kernel<1>, (const void*)gemm_skinny_kernel<2>,
                        (const void*)gemm_skinny_kernel<3>, (const void*)gemm_skinny_kernel<5>}) {
    CUDA_TRY(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSkSmemMax));
    CUDA_TRY(cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
  }
  set_attn_attrs<2, 64>();
  set_attn_attrs<4, 64>();
  set_attn_attrs<2, 32>();
  set_attn_attrs<4, 32>();
  done = true;
}

// ------------------------------------------------------------------ tables

void compute_tables(gdit_handle* h, int K, cudaStream_t s) {
  if (h->tables.count(K)) return;
  Tables t;
  t.K = K;
  const int D = h->D, L = h->L, C = h->C, Tf = h->Tf;
  // t_k = k / K; t_discretized = floor(t_k * buckets), in double (Isaac-GR00T
  // architecture page, "Inference (denoising)"; GR00T model class page,
  // num_timestep_buckets).
  for (int k = 0; k < K; ++k) {
    const double tk = (double)k / (double)K;
    t.td.push_back((float)std::floor(tk * (double)h->cfg.num_timestep_buckets));
  }
  t.ada = h->dalloc<float>((size_t)K * (L + 1) * 2 * D);
  t.tw2 = h->dalloc<float>((size_t)K * C * D);
  float* td = h->dalloc<float>((size_t)K);
  float* phiT = h->dalloc<float>((size_t)K * Tf);
  float* phiD = h->dalloc<float>((size_t)K * D);
  float* t1 = h->dalloc<float>((size_t)K * D);
  float* temb = h->dalloc<float>((size_t)K * D);
  CUDA_TRY(cudaMemcpyAsync(td, t.td.data(), sizeof(float) * K, cudaMemcpyHostToDevice, s));
  const int thr = 256;
  sinusoid_kernel<<<(K * Tf + thr - 1) / thr, thr, 0, s>>>(td, K, Tf, phiT);
  sinusoid_kernel<<<(K * D + thr - 1) / thr, thr, 0, s>>>(td, K, D, phiD);
  // TimestepEncoder: temb = L2(SiLU(L1(phi_Tf(td))))
  gemv_rows_kernel<<<(D + 7) / 8, 256, 0, s>>>(h->w.t1w, D, Tf, phiT, K, h->w.t1b, 0, 1, t1, D);
  gemv_rows_kernel<<<(D + 7) / 8, 256, 0, s>>>(h->w.t2w, D, D, t1, K, h->w.t2b, 0, 0, temb, D);
  // AdaLN modulation of every block and of norm_out: Lin_l(SiLU(temb)) -> [K][L+1][2D]
  const int R = (L + 1) * 2 * D;
  gemv_rows_kernel<<<(R + 7) / 8, 256, 0, s>>>(h->w.ada_w, R, D, temb, K, h->w.ada_b, 1, 0, t.ada, R);
  // timestep half of the action encoder's W2 (+ its bias): phi_D(td) W2[c][D:2D] + b2[c] -> [K][C][D]
  gemv_rows_kernel<<<(C * D + 7) / 8, 256, 0, s>>>(h->w.wa2taut, C * D, D, phiD, K, h->w.ba2, 0, 0, t.tw2,
                                                  (long long)C * D);
  CUDA_TRY(cudaGetLastError());
  h->tables[K] = std::move(t);
}

// ------------------------------------------------------------------ planning

// The cross-attention K/V projection on the CTA-pair kernel.  Its output, the
// head-major cache [layer][K | V][head][token][head_dim], is the 3-D tensor
// [Lc * 2 * heads][max_tok][head_dim]: with head_dim 64 every 64-column
// epilogue box is one head block, written by a 3-D TMA store.  Its rows are
// the packed token range the router wrote, read by the kernel after its
// dependency wait.  The last row tile also writes rows past that range
// (projections of stale packed rows): no reader looks past a sample's keys
// (the attention kernels zero-fill those rows), and a later chunk of the same
// call rewrites its own rows.
void enable_pair_kv(GemmOp& op, const gdit_handle* h, const void* A, const void* W) {
  GemmArgs& a = op.args;
  if (h->cfg.head_dim != 64 || a.splits != 1 || (op.bn != 256 && op.bn != 128) || a.N % op.bn != 0 ||
      a.N % 64 != 0 || a.num_groups != 0)
    return;
  const long long nt = a.N / op.bn;
  const long long pair_tiles = ((a.M + kPairBM - 1) / kPairBM) * nt;
  const long long one_tiles = ((a.M + kBM - 1) / kBM) * nt;
  const long long pair_sms = std::min<long long>(2 * pair_tiles, h->num_sms - h->num_sms % 2);
  const long long one_sms = std::min<long long>(one_tiles, h->num_sms);
  if (10 * pair_sms < 9 * one_sms) return;
  op.to = make_kv_out_tmap(a.out, a.N / 64, h->max_tok);
  a.tma_out = 1;
  a.out3d = 1;
  op.pair = true;
  op.ta = make_tmap(A, a.M, a.K, a.K, 128);
  op.tb = make_tmap(W, a.N, a.K, a.K, op.bn / 2);
  op.grid = (int)(2 * std::min<long long>(pair_tiles, h->num_sms / 2));
}

GemmOp plan_gemm(gdit_handle* h, const void* A, long long a_rows, int K, const void* Bw, long long b_rows, int N,
                 int epi, long long rows_est, int groups, int rows_per_sample, int groups_est) {
  GemmOp op;
  op.args = default_args();
  GemmArgs& a = op.args;
  a.M = (int)a_rows;
  a.N = N;
  a.K = K;
  a.num_groups = groups;
  a.seg = groups ? h->seg : nullptr;
  a.rows_per_sample = rows_per_sample;
  a.b_group_rows = N;
  a.epi = epi;
  a.ws = h->ws;
  a.counters = h->counters;
  a.err = h->status;
  int bn, splits;
  choose_tiling(rows_est, groups_est, N, K, h->num_sms, a_rows, bn, splits);
  op.bn = bn;
  a.splits = splits;
  op.ta = make_tmap(A, a_rows, K, K, kBM);
  op.tb = make_tmap(Bw, b_rows, K, K, bn);
  op.a_ptr = A;
  op.b_ptr = Bw;
  op.to = op.ta;   // placeholder unless the TMA-store epilogue is enabled
  const long long nt = (N + bn - 1) / bn;
  long long max_units = ((a_rows + kBM - 1) / kBM + (groups ? std::min<long long>(groups, a_rows) : 0)) * nt;
  if (splits > 1 && max_units > kCounters) throw GditError(GDIT_EINVAL, "too many split-K tiles");
  op.grid = (int)std::max<long long>(1, std::min<long long>(max_units * splits, h->num_sms));
  op.out_bytes = (epi <= EPI_SWISH_VEC_BF16) ? 2 : 4;
  return op;
}

// Whether one sample of N tokens fits the single-sample loop run by `ctas`
// CTAs: its shared buffers, its weight chunking (K <= 1024 or a multiple of
// 1024), one CTA per head, and, where a CTA has more than kSmallMaxUnits units
// of 8 features in a linear (it takes them in passes), room for the
// reduction area after the normalised / attention rows, which are read again.
bool small_loop_fits(const gdit_config& c, int N, int ctas) {
  const long long D = c.hidden, F = c.mlp_hidden, A = c.action_dim;
  if (N > kSmallMaxTok || D > kSmallMaxD || c.num_layers > kSmallMaxLayers || c.num_heads > ctas) return false;
  // the K/V cache rows (with one box of slack) are addressed by 32-bit TMA coordinates
  if ((long long)(c.num_layers / 2) * 2 * c.num_heads * ((long long)c.max_batch * c.max_backbone_seq + kSmallAttnKB) >=
      (1LL << 31))
    return false;
  if ((long long)N * (D + 8) * 2 > kSmLnScratch) return false;   // LN output rows below the LN scratch
  // LN: the staged f32 rows and their statistics pieces, after the output rows
  if ((long long)small_ln_piece_offset(N, (int)D) + (long long)N * kLnPieces * 8 > kSmLnScratch) return false;
  for (long long K : {A, D, F}) {
    if (K % 16 != 0 || (K > kSmallKC && K % kSmallKC != 0)) return false;
    if ((long long)N * (K + 8) * 2 > kSmXBytes) return false;
  }
  // self layers: the attention output rows and the QKV rows share the X area
  if ((((long long)N * (D + 8) * 2 + 127) & ~127LL) + (long long)N * (3 * D + 8) * 2 > kSmXBytes) return false;
  bool passes = false;
  for (long long n_out : {A, D, 3 * D, F}) {
    if (n_out % kSmallUF != 0) return false;
    if ((n_out / kSmallUF + ctas - 1) / ctas > kSmallMaxUnits) passes = true;
  }
  if (passes && (long long)small_ln_stage_offset(N, (int)D) + kSmRedBytes > kSmLnScratch) return false;
  return true;
}

// Whether a batch of B samples runs the K-step loop as the persistent kernel
// (one sample, or up to kSmallMaxGroups with one CTA group of num_sms / B
// CTAs per sample), its CTAs per group, and whether the grouped instantiation
// (several groups, or a CTA with more than kSmallMaxUnits units of a linear)
// runs.  False: the per-layer kernels.
bool plan_small(const gdit_config& c, int B, int K, int num_sms, int& gsize, bool& grouped) {
  const int N = c.action_horizon + 1, L = c.num_layers;
  const long long D = c.hidden, F = c.mlp_hidden, A = c.action_dim;
  gsize = B >= 1 ? num_sms / B : 0;
  grouped = false;
  if (B < 1 || B > kSmallMaxGroups || (c.flags & GDIT_FLAG_NO_SMALL) != 0 ||
      (long long)B * small_phases_per_step(L) * K > kSmallMaxPhases || !small_loop_fits(c, N, gsize))
    return false;
  grouped = B > 1;
  for (long long n_out : {A, D, 3 * D, F})
    if ((n_out / kSmallUF + gsize - 1) / gsize > kSmallMaxUnits) grouped = true;
  return true;
}

std::unique_ptr<Profile> build_profile(gdit_handle* h, int B, int S, int K, int bf16) {
  auto p = std::make_unique<Profile>();
  p->B = B;
  p->S = S;
  p->K = K;
  p->bf16 = bf16;
  const int D = h->D, F = h->F, N = h->N, H = h->H, A = h->A, C = h->C, Dvl = h->Dvl, Sd = h->Sd, L = h->L;
  const long long rows = (long long)B * N;
  const long long arows = (long long)B * H;
  const int gest = std::min(B, C);
  DevModel& m = h->w;

  // cross-attention K/V of every cross layer, over the packed valid tokens:
  // [tok, Dvl] x [Lc*2D, Dvl]^T -> KV [Lc][tok][2D] (column blocks of 2D)
  p->kv = plan_gemm(h, h->xp, (long long)B * S, Dvl, m.wkv, (long long)h->Lc * 2 * D, h->Lc * 2 * D, EPI_BF16,
                    (long long)B * S, 0, 0, 1);
  p->kv.args.m_dev = h->vofs + B;
  p->kv.args.bias = m.bkv;
  p->kv.args.out = h->kv;
  p->kv.args.ldo = 2 * D;
  // head-major cache: layer block [K | V][head][token][head_dim], so the
  // attention of one (sample, head) streams contiguous rows
  p->kv.args.nblk = 2 * D;
  p->kv.args.blk_stride = h->max_tok * 2 * D;
  p->kv.args.head_cols = h->cfg.head_dim;
  p->kv.args.head_stride = h->max_tok * h->cfg.head_dim;
  p->kv.rows_kind = 1;
  p->kv.weight_bytes = (long long)h->Lc * 2 * D * Dvl * 2;
  if ((h->cfg.flags & GDIT_FLAG_NO_PAIR) == 0) enable_pair_kv(p->kv, h, h->xp, m.wkv);

  // state encoder (CategorySpecificMLP, ReLU)
  p->st1 = plan_gemm(h, h->sb, B, Sd, m.ws1t, (long long)C * D, D, EPI_RELU_BF16, B, C, 1, gest);
  p->st1.args.bias = m.bs1;
  p->st1.args.bias_gstride = D;
  p->st1.args.out = h->s1;
  p->st1.args.ldo = D;
  p->st1.rows_kind = 2;
  p->st2 = plan_gemm(h, h->s1, B, D, m.ws2t, (long long)C * D, D, EPI_F32, B, C, 1, gest);
  p->st2.args.bias = m.bs2;
  p->st2.args.bias_gstride = D;
  p->st2.args.out = h->sfeat;
  p->st2.args.ldo = D;
  p->st2.rows_kind = 2;

  // action encoder: a = x W1[c] + b1; z = swish(a W2a[c] + (phi(td) W2tau[c] + b2)); e = z W3[c] + b3 -> h rows 1..H
  p->a1 = plan_gemm(h, h->xb, arows, A, m.wa1t, (long long)C * D, D, EPI_BF16, arows, C, H, gest);
  p->a1.args.bias = m.ba1;
  p->a1.args.bias_gstride = D;
  p->a1.args.out = h->abf;
  p->a1.args.ldo = D;
  p->a1.rows_kind = 2;
  p->a2 = plan_gemm(h, h->abf, arows, D, m.wa2at, (long long)C * D, D, EPI_SWISH_VEC_BF16, arows, C, H, gest);
  p->a2.args.vec_gstride = D;   // vec set per step
  p->a2.args.out = h->zbf;
  p->a2.args.ldo = D;
  p->a2.rows_kind = 2;
  p->a3 = plan_gemm(h, h->zbf, arows, D, m.wa3t, (long long)C * D, D, EPI_F32, arows, C, H, gest);
  p->a3.args.bias = m.ba3;
  p->a3.args.bias_gstride = D;
  p->a3.args.out = h->h;
  p->a3.args.ldo = D;
  p->a3.args.in_group = H;
  p->a3.args.out_group = N;
  p->a3.args.out_off = 1;
  p->a3.rows_kind = 2;

  // DiT blocks
  p->q.resize(L);
  p->o.resize(L);
  p->ff1.resize(L);
  p->ff2.resize(L);
  for (int l = 0; l < L; ++l) {
    const int nq = (l % 2 == 1) ? 3 * D : D;
    p->q[l] = plan_gemm(h, h->u, rows, D, m.wq[l], nq, nq, EPI_BF16, rows, 0, 0, 1);
    p->q[l].args.bias = m.bq[l];
    p->q[l].args.out = h->qkv;
    p->q[l].args.ldo = nq;
    p->q[l].weight_bytes = (long long)nq * D * 2;
    p->o[l] = plan_gemm(h, h->o, rows, D, m.wo[l], D, D, EPI_RESID_F32, rows, 0, 0, 1);
    p->o[l].args.bias = m.bo[l];
    p->o[l].args.out = h->h;
    p->o[l].args.ldo = D;
    p->o[l].weight_bytes = (long long)D * D * 2;
    p->ff1[l] = plan_gemm(h, h->u, rows, D, m.wff1[l], F, F, EPI_GELU_BF16, rows, 0, 0, 1);
    p->ff1[l].args.bias = m.bff1[l];
    p->ff1[l].args.out = h->f;
    p->ff1[l].args.ldo = F;
    p->ff1[l].weight_bytes = (long long)F * D * 2;
    p->ff2[l] = plan_gemm(h, h->f, rows, F, m.wff2[l], D, D, EPI_RESID_F32, rows, 0, 0, 1);
    p->ff2[l].args.bias = m.bff2[l];
    p->ff2[l].args.out = h->h;
    p->ff2[l].args.ldo = D;
    p->ff2[l].weight_bytes = (long long)D * F * 2;
    if ((h->cfg.flags & GDIT_FLAG_NO_TMA_STORE) == 0)
      for (GemmOp* g : {&p->q[l], &p->o[l], &p->ff1[l], &p->ff2[l]}) enable_tma_out(*g);
    if ((h->cfg.flags & GDIT_FLAG_NO_PAIR) == 0) {
      enable_pair(p->q[l], h->u, m.wq[l], h->num_sms);
      enable_pair(p->o[l], h->o, m.wo[l], h->num_sms);
      enable_pair(p->ff1[l], h->u, m.wff1[l], h->num_sms);
      enable_pair(p->ff2[l], h->f, m.wff2[l], h->num_sms);
    }
    if ((h->cfg.flags & GDIT_FLAG_NO_SKINNY) == 0)
      for (GemmOp* g : {&p->q[l], &p->o[l], &p->ff1[l], &p->ff2[l]}) enable_skinny(*g, h->num_sms);
  }
  // norm_out + proj_out on every token; only the H action rows are kept (compact)
  p->proj = plan_gemm(h, h->u, rows, D, m.proj_w, D, D, EPI_BF16, rows, 0, 0, 1);
  p->proj.args.bias = m.proj_b;
  p->proj.args.out = h->ybf;
  p->proj.args.ldo = D;
  p->proj.args.in_group = N;
  p->proj.args.in_skip = 1;
  p->proj.args.out_group = H;
  p->proj.weight_bytes = (long long)D * D * 2;
  // action decoder (CategorySpecificMLP, ReLU), Euler update fused into layer 2
  p->d1 = plan_gemm(h, h->ybf, arows, D, m.wd1t, (long long)C * D, D, EPI_RELU_BF16, arows, C, H, gest);
  p->d1.args.bias = m.bd1;
  p->d1.args.bias_gstride = D;
  p->d1.args.out = h->rbf;
  p->d1.args.ldo = D;
  p->d1.rows_kind = 2;
  p->d2 = plan_gemm(h, h->rbf, arows, D, m.wd2t, (long long)C * A, A, EPI_EULER, arows, C, H, gest);
  p->d2.args.bias = m.bd2;
  p->d2.args.bias_gstride = A;
  p->d2.args.out = h->x;
  p->d2.args.ldo = A;
  p->d2.args.out2 = h->xb;
  p->d2.args.ldo2 = A;
  p->d2.args.alpha = 1.0f / (float)K;
  p->d2.rows_kind = 2;
  for (GemmOp* g : {&p->st1, &p->st2, &p->a1, &p->a2, &p->a3, &p->d1, &p->d2})
    g->weight_bytes = (long long)g->args.N * g->args.K * 2;   // per category used

  // one sample, or up to kSmallMaxGroups: the K-step loop as one persistent
  // kernel whose CTAs form one group per sample
  int gsize = 0;
  bool grouped = false;
  p->small = plan_small(h->cfg, B, K, h->num_sms, gsize, grouped);
  if (p->small) {
    const Tables& t = h->tables.at(K);
    SmallPlan sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.D = D; sp.F = F; sp.A = A; sp.H = H; sp.N = N; sp.nh = h->cfg.num_heads; sp.dh = h->cfg.head_dim;
    sp.L = L; sp.K = K; sp.C = C;
    sp.eps = h->cfg.ln_eps;
    sp.scale_log2 = 1.4426950408889634f / std::sqrt((float)h->cfg.head_dim);
    sp.max_tok = h->max_tok;
    sp.h = h->h; sp.x = h->x; sp.xb = h->xb;
    sp.abf = h->abf; sp.zbf = h->zbf; sp.qkv = h->qkv; sp.o = h->o; sp.f = h->f; sp.ybf = h->ybf; sp.rbf = h->rbf;
    sp.sfeat = h->sfeat; sp.seg = h->seg; sp.vofs = h->vofs; sp.kspan = h->kspan; sp.kflag = h->kflag;
    sp.text_every = h->cfg.attend_text_every_n_blocks;
    sp.ada = t.ada; sp.tw2 = t.tw2;
    sp.wa1t = m.wa1t; sp.wa2at = m.wa2at; sp.wa3t = m.wa3t; sp.wd1t = m.wd1t; sp.wd2t = m.wd2t; sp.proj_w = m.proj_w;
    sp.ba1 = m.ba1; sp.ba3 = m.ba3; sp.bd1 = m.bd1; sp.bd2 = m.bd2; sp.proj_b = m.proj_b;
    for (int l = 0; l < L; ++l) {
      SmallLayer& y = sp.layers[l];
      y.wq = m.wq[l]; y.bq = m.bq[l]; y.wo = m.wo[l]; y.bo = m.bo[l]; y.ln3g = m.ln3g[l]; y.ln3b = m.ln3b[l];
      y.wff1 = m.wff1[l]; y.bff1 = m.bff1[l]; y.wff2 = m.wff2[l]; y.bff2 = m.bff2[l];
      y.kv = (l % 2 == 0) ? h->kv + (size_t)(l / 2) * h->max_tok * 2 * D : nullptr;
    }
    sp.kv_map = make_kv_tmap(h->kv, (long long)h->Lc * 2 * h->cfg.num_heads * h->max_tok, h->cfg.head_dim,
                             kSmallAttnKB);
    sp.err = h->status;
    sp.groups = B;
    p->small_phases = small_phases_per_step(L) * K;
    p->small_groups = B;
    p->small_gsize = gsize;
    p->small_grouped = grouped;
    // sample b (embodiment-sorted position) works on its own rows of the
    // batch buffers and on its own counters, descriptors and statistics
    std::vector<SmallPlan> plans((size_t)B, sp);
    for (int b = 0; b < B; ++b) {
      SmallPlan& q = plans[(size_t)b];
      q.sample = b;
      q.h = h->h + (size_t)b * N * D;
      q.x = h->x + (size_t)b * H * A;
      q.xb = h->xb + (size_t)b * H * A;
      q.abf = h->abf + (size_t)b * H * D;
      q.zbf = h->zbf + (size_t)b * H * D;
      q.ybf = h->ybf + (size_t)b * H * D;
      q.rbf = h->rbf + (size_t)b * H * D;
      q.qkv = h->qkv + (size_t)b * N * 3 * D;
      q.o = h->o + (size_t)b * N * D;
      q.f = h->f + (size_t)b * N * F;
      q.sfeat = h->sfeat + (size_t)b * D;
      q.kspan = h->kspan + 2 * b;
      q.counters = h->phase_counters + (size_t)b * p->small_phases;
      q.phases = h->phase_table + (size_t)b * p->small_phases;
      q.ln_part = h->ln_part + (size_t)b * kSmallMaxTok * kLnPieces;
    }
    p->small_plan = h->dalloc<SmallPlan>((size_t)B);
    CUDA_TRY(cudaMemcpy(p->small_plan, plans.data(), sizeof(SmallPlan) * (size_t)B, cudaMemcpyHostToDevice));
  }
  return p;
}

// ------------------------------------------------------------------ enqueue

struct Launcher {
  gdit_handle* h;
  cudaStream_t s;
  Recorder* rec;

  template <typename F>
  void timed(const char* name, double flops, double bytes, const GemmOp* op, F&& fn) {
    if (rec == nullptr) {
      fn();
      return;
    }
    Recorder::Ev e;
    e.cls = rec->cls(name);
    e.flops = flops;
    e.bytes = bytes;
    e.op = op;
    CUDA_TRY(cudaEventCreate(&e.a));
    CUDA_TRY(cudaEventCreate(&e.b));
    CUDA_TRY(cudaEventRecord(e.a, s));
    fn();
    CUDA_TRY(cudaEventRecord(e.b, s));
    rec->evs.push_back(e);
  }
  void gemm(const char* name, const GemmOp& op, const GemmArgs* over = nullptr) {
    timed(name, 0, 0, &op, [&] { launch_gemm(op, over ? *over : op.args, s, h->pdl); });
  }
};

// Valid backbone tokens of samples [b0, b0 + nb) -> packed rows (caller order).
void launch_pack(gdit_handle* h, cudaStream_t s, int bf16, int S, int b0, int nb) {
  launch_k(s, h->pdl, pack_features_kernel, dim3(nb, (S + 31) / 32), dim3(kPackThreads), 0, (const IoPtrs*)h->io,
           bf16, S, h->Dvl, b0, (const int*)h->vofs, h->xp, h->kflag, (long long)h->max_tok, h->status);
}

// The vision-language LayerNorm of every packed token (only with its weights).
void launch_vlln(gdit_handle* h, cudaStream_t s, int B, int S) {
  const dim3 grid((unsigned)(((long long)B * S + 7) / 8));
  const int* tot = (const int*)h->vofs + B;
  const float e = h->cfg.ln_eps;
  const bool pdl = h->pdl;
  switch (h->Dvl / 256) {
    case 1: launch_k(s, pdl, vlln_kernel<1>, grid, dim3(256), 0, h->xp, tot, h->w.vlln_g, h->w.vlln_b, e); break;
    case 2: launch_k(s, pdl, vlln_kernel<2>, grid, dim3(256), 0, h->xp, tot, h->w.vlln_g, h->w.vlln_b, e); break;
    case 4: launch_k(s, pdl, vlln_kernel<4>, grid, dim3(256), 0, h->xp, tot, h->w.vlln_g, h->w.vlln_b, e); break;
    case 8: launch_k(s, pdl, vlln_kernel<8>, grid, dim3(256), 0, h->xp, tot, h->w.vlln_g, h->w.vlln_b, e); break;
    default: launch_k(s, pdl, vlln_kernel<16>, grid, dim3(256), 0, h->xp, tot, h->w.vlln_g, h->w.vlln_b, e); break;
  }
}

void enqueue_forward(gdit_handle* h, Profile& p, cudaStream_t s, Recorder* rec, bool prologue = true) {
  Launcher lx{h, s, rec};
  const int B = p.B, S = p.S, K = p.K;
  const int D = h->D, N = h->N, H = h->H, A = h->A, L = h->L, C = h->C, Dvl = h->Dvl;
  const int rows = B * N;
  const Tables& t = h->tables.at(K);
  const bool pdl = h->pdl;
  const int vec = D / 128;
  const float eps = h->cfg.ln_eps;
  auto ln = [&](const float* p0, const float* p1, int mode, const float* restore) {
    const dim3 grid((rows + 7) / 8);
    lx.timed("layernorm", 0, (double)rows * D * 6, nullptr, [&] {
      switch (vec) {
        case 1: launch_k(s, pdl, layernorm_kernel<1>, grid, dim3(256), 0, h->h, rows, p0, p1, mode, eps, h->u, restore, N); break;
        case 2: launch_k(s, pdl, layernorm_kernel<2>, grid, dim3(256), 0, h->h, rows, p0, p1, mode, eps, h->u, restore, N); break;
        case 4: launch_k(s, pdl, layernorm_kernel<4>, grid, dim3(256), 0, h->h, rows, p0, p1, mode, eps, h->u, restore, N); break;
        case 8: launch_k(s, pdl, layernorm_kernel<8>, grid, dim3(256), 0, h->h, rows, p0, p1, mode, eps, h->u, restore, N); break;
        default: launch_k(s, pdl, layernorm_kernel<16>, grid, dim3(256), 0, h->h, rows, p0, p1, mode, eps, h->u, restore, N); break;
      }
    });
  };
  // Attention schedule: one warp per (sample, head) when there are enough of
  // them to fill the GPU (and always for self-attention: N keys); otherwise
  // one CTA per (sample, head) with the keys split across its warps.
  auto attn = [&](const char* name, const AttnArgs& aa, bool warp_sched) {
    const dim3 block(kAttnThreads);
    const int MT = N <= 32 ? 2 : 4;
    const int DH = h->cfg.head_dim;
    lx.timed(name, 0, 0, nullptr, [&] {
      if (warp_sched) {
        // persistent warps, every one with the same number of items: as many
        // rounds as a full GPU of resident warps needs, then as few CTAs as
        // still finish in that many rounds
        const long long resident = 4LL * g_attn_warp_ctas[MT == 4][DH == 64] * h->num_sms;
        const long long rounds = (aa.num_items + resident - 1) / resident;
        const long long warps = (aa.num_items + rounds - 1) / rounds;
        const dim3 grid((unsigned)((warps + 3) / 4));
        constexpr int R = kWarpRing;
        if (DH == 64 && MT == 2) launch_k(s, pdl, attention_warp_kernel<2, 64>, grid, block, AttnSmem<2, 64, R>::WARP_TOTAL, aa);
        else if (DH == 64) launch_k(s, pdl, attention_warp_kernel<4, 64>, grid, block, AttnSmem<4, 64, R>::WARP_TOTAL, aa);
        else if (MT == 2) launch_k(s, pdl, attention_warp_kernel<2, 32>, grid, block, AttnSmem<2, 32, R>::WARP_TOTAL, aa);
        else launch_k(s, pdl, attention_warp_kernel<4, 32>, grid, block, AttnSmem<4, 32, R>::WARP_TOTAL, aa);
      } else {
        const dim3 grid(aa.num_items);
        if (DH == 64 && MT == 2) launch_k(s, pdl, attention_split_kernel<2, 64>, grid, block, AttnSmem<2, 64>::SPLIT_TOTAL, aa);
        else if (DH == 64) launch_k(s, pdl, attention_split_kernel<4, 64>, grid, block, AttnSmem<4, 64>::SPLIT_TOTAL, aa);
        else if (MT == 2) launch_k(s, pdl, attention_split_kernel<2, 32>, grid, block, AttnSmem<2, 32>::SPLIT_TOTAL, aa);
        else launch_k(s, pdl, attention_split_kernel<4, 32>, grid, block, AttnSmem<4, 32>::SPLIT_TOTAL, aa);
      }
    });
  };
  const bool cross_warp_sched = B * h->cfg.num_heads >= 4 * h->num_sms;

  // routing, packing and the K/V projection of the backbone tokens (the
  // host-buffer entry point runs these itself, overlapped with the copies)
  if (prologue) {
    lx.timed("route_pack", 0, 0, nullptr, [&] {
      launch_k(s, pdl, route_kernel, dim3(1), dim3(kRouteThreads), 0, (const IoPtrs*)h->io, B, S, C, h->perm, h->seg,
               h->vofs, h->kspan, h->bad, h->status);
    });
    lx.timed("route_pack", 0, (double)B * S * Dvl * (p.bf16 ? 4 : 6), nullptr,
             [&] { launch_pack(h, s, p.bf16, S, 0, B); });
    if (h->w.vlln_g != nullptr)
      lx.timed("vlln", 0, (double)B * S * Dvl * 4, nullptr, [&] { launch_vlln(h, s, B, S); });
    lx.gemm("gemm_kv_proj", p.kv);
  }
  lx.timed("route_pack", 0, 0, nullptr, [&] {
    launch_k(s, pdl, gather_inputs_kernel, dim3(B), dim3(128), 0, (const IoPtrs*)h->io, B, H * A, h->Sd,
             (const int*)h->perm, h->x, h->xb, h->sb, h->status);
  });
  lx.gemm("gemm_embodiment", p.st1);
  lx.gemm("gemm_embodiment", p.st2);

  if (p.small) {
    lx.timed("small_loop", 0, 0, nullptr, [&] {
      const int n_desc = p.small_groups * p.small_phases;
      launch_k(s, pdl, small_describe_kernel, dim3((n_desc + 127) / 128), dim3(128), 0,
               (const SmallPlan*)p.small_plan);
      CUDA_TRY(cudaMemsetAsync(h->phase_counters, 0, sizeof(int) * (size_t)n_desc, s));
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(p.small_groups * p.small_gsize));
      cfg.blockDim = dim3(kSmallThreads);
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs co-resident: they wait on one another
      attr[0].val.cooperative = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      const SmallPlan* sp = p.small_plan;
      cfg.dynamicSmemBytes = h->cfg.head_dim == 64 ? SmallSmem<64>::TOTAL : SmallSmem<32>::TOTAL;
      if (h->cfg.head_dim == 64 && p.small_grouped)
        CUDA_TRY(cudaLaunchKernelEx(&cfg, small_loop_kernel<64, true>, sp));
      else if (h->cfg.head_dim == 64)
        CUDA_TRY(cudaLaunchKernelEx(&cfg, small_loop_kernel<64, false>, sp));
      else if (p.small_grouped)
        CUDA_TRY(cudaLaunchKernelEx(&cfg, small_loop_kernel<32, true>, sp));
      else
        CUDA_TRY(cudaLaunchKernelEx(&cfg, small_loop_kernel<32, false>, sp));
    });
    lx.timed("route_pack", 0, 0, nullptr, [&] {
      launch_k(s, pdl, scatter_out_kernel, dim3(B), dim3(128), 0, (const IoPtrs*)h->io, H * A, (const int*)h->perm,
               (const uint8_t*)h->bad, (const float*)h->x, h->status);
    });
    return;
  }

  const float scale_log2 = 1.4426950408889634f / std::sqrt((float)h->cfg.head_dim);
  for (int k = 0; k < K; ++k) {
    GemmArgs a2 = p.a2.args;
    a2.vec = t.tw2 + (size_t)k * C * D;
    lx.gemm("gemm_embodiment", p.a1);
    lx.gemm("gemm_embodiment", p.a2, &a2);
    lx.gemm("gemm_embodiment", p.a3);
    const float* ada_k = t.ada + (size_t)k * (L + 1) * 2 * D;
    for (int l = 0; l < L; ++l) {
      const float* ada = ada_k + (size_t)l * 2 * D;
      ln(ada, ada + D, 0, l == 0 ? h->sfeat : nullptr);
      lx.gemm("gemm_dit", p.q[l]);
      AttnArgs aa;
      aa.kv_rows = h->max_tok;
      aa.status = h->status;
      aa.q = h->qkv;
      aa.n_tok = N;
      aa.num_heads = h->cfg.num_heads;
      aa.num_items = B * h->cfg.num_heads;
      aa.out = h->o;
      aa.out_ld = D;
      aa.scale_log2 = scale_log2;
      aa.kflag = h->kflag;
      aa.ksel = l % 2 == 1 ? -1 : cross_key_sel(h->cfg, l);
      if (l % 2 == 1) {
        aa.q_ld = 3 * D;
        aa.k = h->qkv + D;
        aa.v = h->qkv + 2 * D;
        aa.kv_ld = 3 * D;
        aa.kv_head_stride = h->cfg.head_dim;
        aa.kspan = nullptr;
        attn("attn_self", aa, true);
      } else {
        const __nv_bfloat16* kvl = h->kv + (size_t)(l / 2) * h->max_tok * 2 * D;
        aa.q_ld = D;
        aa.k = kvl;
        aa.v = kvl + (size_t)h->cfg.num_heads * h->max_tok * h->cfg.head_dim;
        aa.kv_ld = h->cfg.head_dim;
        aa.kv_head_stride = h->max_tok * h->cfg.head_dim;
        aa.kspan = h->kspan;
        attn("attn_cross", aa, cross_warp_sched);
      }
      lx.gemm("gemm_dit", p.o[l]);
      ln(h->w.ln3g[l], h->w.ln3b[l], 1, nullptr);
      lx.gemm("gemm_dit", p.ff1[l]);
      lx.gemm("gemm_dit", p.ff2[l]);
    }
    const float* ada = ada_k + (size_t)L * 2 * D;
    ln(ada, ada + D, 0, nullptr);
    lx.gemm("gemm_dit", p.proj);
    lx.gemm("gemm_embodiment", p.d1);
    lx.gemm("gemm_embodiment", p.d2);
  }
  lx.timed("route_pack", 0, 0, nullptr, [&] {
    launch_k(s, pdl, scatter_out_kernel, dim3(B), dim3(128), 0, (const IoPtrs*)h->io, H * A, (const int*)h->perm,
             (const uint8_t*)h->bad, (const float*)h->x, h->status);
  });
}

Profile& get_profile(gdit_handle* h, int B, int S, int K, int bf16, bool allow_build) {
  const auto key = std::make_tuple(B, S, K, bf16);
  auto it = h->profiles.find(key);
  if (it != h->profiles.end()) return *it->second;
  if (!allow_build)
    throw GditError(GDIT_EPROFILE, fmt("profile (batch=%d, seq=%d, steps=%d, bf16=%d) was not prepared", B, S, K, bf16));
  auto p = build_profile(h, B, S, K, bf16);
  if (h->use_graph) {
    if (h->cap_stream == nullptr) CUDA_TRY(cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking));
    // the whole call, and the call after the K/V projection
    for (int part = 0; part < 2; ++part) {
      cudaGraph_t graph = nullptr;
      CUDA_TRY(cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal));
      try {
        enqueue_forward(h, *p, h->cap_stream, nullptr, part == 0);
      } catch (...) {
        cudaStreamEndCapture(h->cap_stream, &graph);
        if (graph) cudaGraphDestroy(graph);
        if (p->exec) cudaGraphExecDestroy(p->exec);
        throw;
      }
      CUDA_TRY(cudaStreamEndCapture(h->cap_stream, &graph));
      if (++h->fault.n_graph == h->fault.graph) {
        cudaGraphDestroy(graph);
        if (p->exec) cudaGraphExecDestroy(p->exec);
        throw GditError(GDIT_ECUDA, fmt("injected fault: graph instantiation %lld failed", h->fault.n_graph));
      }
      cudaGraphExec_t& ex = part == 0 ? p->exec : p->exec_main;
      cudaError_t e = cudaGraphInstantiate(&ex, graph, 0);
      cudaGraphDestroy(graph);
      if (e != cudaSuccess && p->exec && part == 1) {
        cudaGraphExecDestroy(p->exec);
        p->exec = nullptr;
      }
      CUDA_TRY(e);
    }
  }
  Profile& ref = *p;
  h->profiles[key] = std::move(p);
  return ref;
}

void check_call(gdit_handle* h, const void* feats, int bb_dtype, const void* mask, const void* state, const void* ids,
                const void* noise, int K, const void* out, int B, int S) {
  REQUIRE(h != nullptr, "handle is NULL");
  REQUIRE(feats && mask && state && ids && noise && out, "a required pointer argument is NULL");
  REQUIRE(bb_dtype == GDIT_F32 || bb_dtype == GDIT_BF16, "bb_dtype must be GDIT_F32 or GDIT_BF16");
  REQUIRE(K >= 1 && K <= 64, "num_steps must be in [1, 64] (got %d)", K);
  REQUIRE(B >= 1 && B <= h->cfg.max_batch, "batch %d outside [1, max_batch=%d]", B, h->cfg.max_batch);
  REQUIRE(S >= 1 && S <= h->cfg.max_backbone_seq, "seq %d outside [1, max_backbone_seq=%d]", S,
          h->cfg.max_backbone_seq);
  REQUIRE(((uintptr_t)feats & 15u) == 0, "backbone_features must be 16-byte aligned");
}

void run_call(gdit_handle* h, const void* feats, int bb_dtype, const uint8_t* mask, const float* state,
              const int32_t* ids, const float* noise, int K, float* out, int B, int S, cudaStream_t s,
              const uint8_t* image_mask = nullptr) {
  CUDA_TRY(cudaSetDevice(h->cfg.device));
  compute_tables(h, K, s);
  Profile& p = get_profile(h, B, S, K, bb_dtype == GDIT_BF16, !h->strict);
  IoPtrs io{feats, mask, state, ids, noise, out, image_mask};
  set_io_kernel<<<1, 1, 0, s>>>(h->io, io);
  CUDA_TRY(cudaGetLastError());
  if (p.exec != nullptr)
    CUDA_TRY(cudaGraphLaunch(p.exec, s));
  else
    enqueue_forward(h, p, s, h->rec);
  h->last_stream = s;
  h->last_B = B;
}

template <typename F>
int guarded(gdit_handle* h, F&& fn) {
  try {
    fn();
    return GDIT_OK;
  } catch (const GditError& e) {
    if (h) h->last_error = e.what();
    else g_create_error = e.what();
    return e.code;
  } catch (const std::bad_alloc&) {
    if (h) h->last_error = "host allocation failed";
    else g_create_error = "host allocation failed";
    return GDIT_ENOMEM;
  } catch (const std::exception& e) {
    if (h) h->last_error = e.what();
    else g_create_error = e.what();
    return GDIT_ECUDA;
  }
}

void free_handle(gdit_handle* h) {
  if (!h) return;
  cudaSetDevice(h->cfg.device);
  cudaDeviceSynchronize();
  for (auto& kv : h->profiles) {
    if (kv.second->exec) cudaGraphExecDestroy(kv.second->exec);
    if (kv.second->exec_main) cudaGraphExecDestroy(kv.second->exec_main);
  }
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  for (cudaEvent_t e : h->chunk_ev)
    if (e) cudaEventDestroy(e);
  if (h->small_ev) cudaEventDestroy(h->small_ev);
  for (void* p : h->allocs) cudaFree(p);
  delete h;
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* gdit_version(void) { return "gdit 0.1 (sm_100a)"; }

const char* gdit_strerror(int code) {
  switch (code) {
    case GDIT_OK: return "ok";
    case GDIT_EINVAL: return "invalid argument";
    case GDIT_ENOMEM: return "out of memory";
    case GDIT_ECUDA: return "CUDA error";
    case GDIT_EPROFILE: return "profile not prepared";
    case GDIT_ETIMEOUT: return "device wait timed out";
    case GDIT_EDEVICE: return "invalid input detected on the device";
    case GDIT_ENODEV: return "no sm_100 device";
    default: return "unknown error";
  }
}

const char* gdit_last_error(const gdit_handle* h) { return h ? h->last_error.c_str() : g_create_error.c_str(); }

int gdit_create(const gdit_config* cfg, const gdit_tensor* weights, int n_weights, gdit_handle** out) {
  if (out) *out = nullptr;
  gdit_handle* h = nullptr;
  g_create_error.clear();
  int rc = guarded(nullptr, [&] {
    REQUIRE(cfg != nullptr && out != nullptr, "cfg and out must not be NULL");
    validate_config(*cfg);
    auto W = check_weights(*cfg, weights, n_weights);   // host-only checks first
    gdit_handle::Faults faults;
    parse_faults(getenv("GDIT_FAULT"), faults);
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) throw GditError(GDIT_ENODEV, "no CUDA device");
    REQUIRE(cfg->device >= 0 && cfg->device < ndev, "device %d out of range", cfg->device);
    cudaDeviceProp prop;
    CUDA_TRY(cudaGetDeviceProperties(&prop, cfg->device));
    if (prop.major != 10) throw GditError(GDIT_ENODEV, fmt("device %d is sm_%d%d, sm_100 required", cfg->device, prop.major, prop.minor));
    CUDA_TRY(cudaSetDevice(cfg->device));
    h = new gdit_handle();
    h->cfg = *cfg;
    h->L = cfg->num_layers;
    h->D = cfg->hidden;
    h->F = cfg->mlp_hidden;
    h->Dvl = cfg->backbone_dim;
    h->A = cfg->action_dim;
    h->Sd = cfg->state_dim;
    h->H = cfg->action_horizon;
    h->C = cfg->num_embodiments;
    h->Tf = cfg->time_freq_dim;
    h->N = cfg->action_horizon + 1;
    h->Lc = cfg->num_layers / 2;
    h->num_sms = prop.multiProcessorCount;
    h->use_graph = (cfg->flags & GDIT_FLAG_NO_GRAPH) == 0;
    h->strict = (cfg->flags & GDIT_FLAG_STRICT_PROFILES) != 0;
    const char* pdl_env = getenv("GDIT_PDL");
    h->pdl = !(pdl_env && pdl_env[0] == '0');
    h->fault = faults;
    set_kernel_attrs();
    upload_model(h, W);
    alloc_workspace(h);
    CUDA_TRY(cudaDeviceSynchronize());
  });
  if (rc != GDIT_OK) {
    if (h) {
      std::string msg = g_create_error;
      free_handle(h);
      g_create_error = msg;
    }
    return rc;
  }
  *out = h;
  return GDIT_OK;
}

void gdit_destroy(gdit_handle* h) { free_handle(h); }

int gdit_get_action(gdit_handle* h, const void* backbone_features, int bb_dtype, const uint8_t* vl_mask,
                    const float* state, const int32_t* embodiment_id, const float* init_noise, int num_steps,
                    float* out_actions, int batch, int seq, void* cuda_stream) {
  if (!h) return GDIT_EINVAL;
  return guarded(h, [&] {
    check_call(h, backbone_features, bb_dtype, vl_mask, state, embodiment_id, init_noise, num_steps, out_actions,
               batch, seq);
    run_call(h, backbone_features, bb_dtype, vl_mask, state, embodiment_id, init_noise, num_steps, out_actions, batch,
             seq, (cudaStream_t)cuda_stream);
  });
}

int gdit_get_action_vl(gdit_handle* h, const void* backbone_features, int bb_dtype, const uint8_t* vl_mask,
                       const uint8_t* image_mask, const float* state, const int32_t* embodiment_id,
                       const float* init_noise, int num_steps, float* out_actions, int batch, int seq,
                       void* cuda_stream) {
  if (!h) return GDIT_EINVAL;
  return guarded(h, [&] {
    check_call(h, backbone_features, bb_dtype, vl_mask, state, embodiment_id, init_noise, num_steps, out_actions,
               batch, seq);
    run_call(h, backbone_features, bb_dtype, vl_mask, state, embodiment_id, init_noise, num_steps, out_actions, batch,
             seq, (cudaStream_t)cuda_stream, image_mask);
  });
}

int gdit_get_action_host(gdit_handle* h, const void* backbone_features, int bb_dtype, const uint8_t* vl_mask,
                         const float* state, const int32_t* embodiment_id, const float* init_noise, int num_steps,
                         float* out_actions, int batch, int seq, void* cuda_stream) {
  if (!h) return GDIT_EINVAL;
  return guarded(h, [&] {
    check_call(h, backbone_features, GDIT_BF16, vl_mask, state, embodiment_id, init_noise, num_steps, out_actions,
               batch, seq);
    REQUIRE(bb_dtype == GDIT_F32 || bb_dtype == GDIT_BF16, "bb_dtype must be GDIT_F32 or GDIT_BF16");
    CUDA_TRY(cudaSetDevice(h->cfg.device));
    cudaStream_t s = (cudaStream_t)cuda_stream;
    const size_t Bm = h->cfg.max_batch, Sm = h->cfg.max_backbone_seq;
    const size_t esz = bb_dtype == GDIT_BF16 ? 2 : 4;
    if (h->st_mask == nullptr) {
      h->st_mask = h->dalloc<uint8_t>(Bm * Sm);
      h->st_state = h->dalloc<float>(Bm * h->Sd);
      h->st_ids = h->dalloc<int32_t>(Bm);
      h->st_noise = h->dalloc<float>(Bm * h->H * h->A);
      h->st_out = h->dalloc<float>(Bm * h->H * h->A);
    }
    const size_t sample_bytes = (size_t)seq * h->Dvl * esz;
    const size_t fbytes = (size_t)batch * sample_bytes;
    if (h->st_feats_bytes < fbytes) {
      const size_t cap = Bm * Sm * h->Dvl * esz;
      h->st_feats = h->dalloc<uint8_t>(std::max(cap, fbytes));
      h->st_feats_bytes = std::max(cap, fbytes);
    }
    if (h->copy_stream == nullptr) {
      CUDA_TRY(cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking));
      for (cudaEvent_t& e : h->chunk_ev) CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
      CUDA_TRY(cudaEventCreateWithFlags(&h->small_ev, cudaEventDisableTiming));
    }
    compute_tables(h, num_steps, s);
    Profile& p = get_profile(h, batch, seq, num_steps, bb_dtype == GDIT_BF16, !h->strict);
    const size_t ha = (size_t)batch * h->H * h->A;
    // The small inputs first, on the copy stream ahead of the features:
    // routing needs the masks and ids.  Host-to-device copies of both streams
    // go through the same copy engine, so a small copy queued on the compute
    // stream could land only after every feature chunk, holding the routing
    // (and so every chunk's projection) until the whole upload had finished.
    // Every earlier use of the staging buffers ended with the previous call's
    // synchronize.
    CUDA_TRY(cudaMemcpyAsync(h->st_mask, vl_mask, (size_t)batch * seq, cudaMemcpyHostToDevice, h->copy_stream));
    CUDA_TRY(cudaMemcpyAsync(h->st_ids, embodiment_id, (size_t)batch * 4, cudaMemcpyHostToDevice, h->copy_stream));
    CUDA_TRY(cudaMemcpyAsync(h->st_state, state, (size_t)batch * h->Sd * 4, cudaMemcpyHostToDevice,
                             h->copy_stream));
    CUDA_TRY(cudaMemcpyAsync(h->st_noise, init_noise, ha * 4, cudaMemcpyHostToDevice, h->copy_stream));
    CUDA_TRY(cudaEventRecord(h->small_ev, h->copy_stream));
    CUDA_TRY(cudaStreamWaitEvent(s, h->small_ev, 0));
    IoPtrs io{h->st_feats, h->st_mask, h->st_state, h->st_ids, h->st_noise, h->st_out, nullptr};
    set_io_kernel<<<1, 1, 0, s>>>(h->io, io);
    CUDA_TRY(cudaGetLastError());
    launch_k(s, h->pdl, route_kernel, dim3(1), dim3(kRouteThreads), 0, (const IoPtrs*)h->io, batch, seq, h->C,
             h->perm, h->seg, h->vofs, h->kspan, h->bad, h->status);
    // The features in sample chunks on the copy stream; each chunk is packed
    // and projected to K/V on the compute stream once it has landed, while
    // the next chunk is still being copied.  (With vlln weights the whole
    // batch is one chunk: the LayerNorm runs over all packed rows.)
    const int nch = h->w.vlln_g != nullptr ? 1 : std::min(kHostChunks, batch);
    for (int c = 0; c < nch; ++c) {
      const int b0 = (int)((long long)c * batch / nch), b1 = (int)((long long)(c + 1) * batch / nch);
      CUDA_TRY(cudaMemcpyAsync(static_cast<uint8_t*>(h->st_feats) + (size_t)b0 * sample_bytes,
                               static_cast<const uint8_t*>(backbone_features) + (size_t)b0 * sample_bytes,
                               (size_t)(b1 - b0) * sample_bytes, cudaMemcpyHostToDevice, h->copy_stream));
      CUDA_TRY(cudaEventRecord(h->chunk_ev[c], h->copy_stream));
    }
    for (int c = 0; c < nch; ++c) {
      const int b0 = (int)((long long)c * batch / nch), b1 = (int)((long long)(c + 1) * batch / nch);
      CUDA_TRY(cudaStreamWaitEvent(s, h->chunk_ev[c], 0));
      launch_pack(h, s, bb_dtype == GDIT_BF16, seq, b0, b1 - b0);
      if (h->w.vlln_g != nullptr) launch_vlln(h, s, batch, seq);
      GemmArgs kv = p.kv.args;   // packed rows [vofs[b0], vofs[b1])
      kv.m_begin_dev = h->vofs + b0;
      kv.m_dev = h->vofs + b1;
      launch_gemm(p.kv, kv, s, h->pdl);
    }
    if (p.exec_main != nullptr)
      CUDA_TRY(cudaGraphLaunch(p.exec_main, s));
    else
      enqueue_forward(h, p, s, nullptr, false);
    h->last_stream = s;
    h->last_B = batch;
    CUDA_TRY(cudaMemcpyAsync(out_actions, h->st_out, ha * 4, cudaMemcpyDeviceToHost, s));
    CUDA_TRY(cudaStreamSynchronize(s));
  });
}

int gdit_prepare(gdit_handle* h, int batch, int seq, int num_steps, int bb_dtype, void* cuda_stream) {
  if (!h) return GDIT_EINVAL;
  return guarded(h, [&] {
    REQUIRE(num_steps >= 1 && num_steps <= 64, "num_steps must be in [1, 64]");
    REQUIRE(batch >= 1 && batch <= h->cfg.max_batch, "batch out of range");
    REQUIRE(seq >= 1 && seq <= h->cfg.max_backbone_seq, "seq out of range");
    REQUIRE(bb_dtype == GDIT_F32 || bb_dtype == GDIT_BF16, "bad bb_dtype");
    CUDA_TRY(cudaSetDevice(h->cfg.device));
    compute_tables(h, num_steps, (cudaStream_t)cuda_stream);
    get_profile(h, batch, seq, num_steps, bb_dtype == GDIT_BF16, true);
  });
}

int gdit_sync_status(gdit_handle* h) {
  if (!h) return GDIT_EINVAL;
  unsigned st = 0;
  int rc = guarded(h, [&] {
    CUDA_TRY(cudaSetDevice(h->cfg.device));
    CUDA_TRY(cudaStreamSynchronize(h->last_stream));
    CUDA_TRY(cudaMemcpy(&st, h->status, sizeof(unsigned), cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemset(h->status, 0, sizeof(unsigned)));
    if (st & DEV_ERR_TIMEOUT) CUDA_TRY(cudaMemset(h->counters, 0, sizeof(int) * kCounters));
  });
  if (rc != GDIT_OK) return rc;
  if (st & DEV_ERR_TIMEOUT) {
    h->last_error = "a device-side wait timed out";
    return GDIT_ETIMEOUT;
  }
  if (st & DEV_ERR_BAD_ID) {
    h->last_error = "embodiment_id out of range (those samples are NaN)";
    return GDIT_EDEVICE;
  }
  if (st & DEV_ERR_INDEX) {
    h->last_error = "range-checked build: an index derived from the inputs was out of range (the access was skipped)";
    return GDIT_EDEVICE;
  }
  return GDIT_OK;
}

int gdit_is_checked(void) { return GDIT_CHECKED ? 1 : 0; }

int gdit_check_canaries(gdit_handle* h, long long* corrupted_bytes) {
  if (!h) return GDIT_EINVAL;
  return guarded(h, [&] {
    REQUIRE(corrupted_bytes != nullptr, "NULL corrupted_bytes");
    REQUIRE(GDIT_CHECKED, "not a range-checked build (libgdit_checked.so has the guard bands)");
    CUDA_TRY(cudaSetDevice(h->cfg.device));
    CUDA_TRY(cudaDeviceSynchronize());
    std::vector<uint8_t> band(kGuardBytes);
    long long bad = 0;
    for (const gdit_handle::Guarded& g : h->guarded_allocs) {
      for (const uint8_t* src : {g.base, g.base + kGuardBytes + g.bytes}) {
        CUDA_TRY(cudaMemcpy(band.data(), src, kGuardBytes, cudaMemcpyDeviceToHost));
        for (uint8_t v : band) bad += v != kGuardByte;
      }
    }
    *corrupted_bytes = bad;
  });
}

int gdit_debug_poke_guard(gdit_handle* h, int which) {
  if (!h) return GDIT_EINVAL;
  return guarded(h, [&] {
    REQUIRE(GDIT_CHECKED, "not a range-checked build");
    REQUIRE(which >= 0 && which < (int)h->guarded_allocs.size(), "allocation %d of %d", which,
            (int)h->guarded_allocs.size());
    CUDA_TRY(cudaSetDevice(h->cfg.device));
    const gdit_handle::Guarded& g = h->guarded_allocs[(size_t)which];
    // the first byte after the buffer: what a one-element overrun would write
    CUDA_TRY(cudaMemset(g.base + kGuardBytes + g.bytes, (int)(uint8_t)~kGuardByte, 1));
  });
}

int gdit_debug_routing(gdit_handle* h, int32_t* perm, int32_t* seg, int32_t* vofs) {
  if (!h) return GDIT_EINVAL;
  return guarded(h, [&] {
    REQUIRE(perm && seg && vofs, "NULL output");
    REQUIRE(h->last_B > 0, "no call has run on this handle");
    CUDA_TRY(cudaSetDevice(h->cfg.device));
    CUDA_TRY(cudaStreamSynchronize(h->last_stream));
    CUDA_TRY(cudaMemcpy(perm, h->perm, sizeof(int) * h->last_B, cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemcpy(seg, h->seg, sizeof(int) * (h->C + 1), cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemcpy(vofs, h->vofs, sizeof(int) * (h->last_B + 1), cudaMemcpyDeviceToHost));
  });
}

// One thread waits on an mbarrier that nothing arrives at, through the same
// bounded wait every kernel uses, with a short limit.
__global__ void wait_expiry_kernel(unsigned* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, status, limit_ns);
}

int gdit_debug_small_plan(const gdit_config* cfg, int batch, int num_steps, int num_sms, int* group_ctas,
                          int* grouped) {
  g_create_error.clear();
  return guarded(nullptr, [&] {
    REQUIRE(cfg && group_ctas && grouped, "NULL argument");
    validate_config(*cfg);
    REQUIRE(batch >= 1 && num_steps >= 1 && num_sms >= 1, "batch %d, num_steps %d, num_sms %d", batch, num_steps,
            num_sms);
    int g = 0;
    bool gr = false;
    const bool small = plan_small(*cfg, batch, num_steps, num_sms, g, gr);
    *group_ctas = small ? g : 0;
    *grouped = small ? (gr ? 1 : 0) : 0;
  });
}

int gdit_debug_skinny_plan(long long M, int N, int K, int num_sms, int* mt, int* nu, int* stages, int* ctas,
                           int* smem_bytes) {
  g_create_error.clear();
  return guarded(nullptr, [&] {
    REQUIRE(mt && nu && stages && ctas && smem_bytes, "NULL output");
    REQUIRE(num_sms >= 1, "num_sms %d", num_sms);
    REQUIRE(skinny_shape_ok(M, N, K), "M %lld, N %d, K %d: not a skinny-M shape (M <= %lld, N %% 8, K %% 64)", M, N, K,
            kSkinnyMaxRows);
    int m = 0, u = 0, st = 0;
    REQUIRE(plan_skinny(M, N, K, num_sms, m, u, st), "no skinny-M plan fits one round over %d SMs", num_sms);
    *mt = m;
    *nu = u;
    *stages = st;
    *ctas = (int)(((M + 16LL * m - 1) / (16LL * m)) * ((N / 8 + u - 1) / u));
    *smem_bytes = sk_smem_bytes(m, u, st);
  });
}

int gdit_debug_wait_expiry(int device, unsigned long long limit_ns) {
  return guarded(nullptr, [&] {
    REQUIRE(limit_ns >= 1000ull && limit_ns <= 1000000000ull, "limit_ns %llu outside [1 us, 1 s]", limit_ns);
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess || n == 0) throw GditError(GDIT_ENODEV, "no CUDA device");
    REQUIRE(device >= 0 && device < n, "device %d of %d", device, n);
    CUDA_TRY(cudaSetDevice(device));
    unsigned* st = nullptr;
    CUDA_TRY(cudaMalloc(&st, sizeof(unsigned)));
    unsigned host = 0;
    cudaError_t e = cudaMemset(st, 0, sizeof(unsigned));
    if (e == cudaSuccess) {
      wait_expiry_kernel<<<1, 32>>>(st, limit_ns);
      e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(&host, st, sizeof(unsigned), cudaMemcpyDeviceToHost);
    cudaFree(st);
    CUDA_TRY(e);
    if (host & DEV_ERR_TIMEOUT) throw GditError(GDIT_ETIMEOUT, "the bounded wait expired and reported it");
  });
}

int gdit_debug_kv(gdit_handle* h, int layer, float* k_out, float* v_out, int* total_valid) {
  if (!h) return GDIT_EINVAL;
  return guarded(h, [&] {
    REQUIRE(total_valid != nullptr, "total_valid is NULL");
    REQUIRE(layer >= 0 && layer < h->L && layer % 2 == 0, "layer %d is not a cross-attention layer", layer);
    REQUIRE(h->last_B > 0, "no call has run on this handle");
    CUDA_TRY(cudaSetDevice(h->cfg.device));
    CUDA_TRY(cudaStreamSynchronize(h->last_stream));
    int tot = 0;
    CUDA_TRY(cudaMemcpy(&tot, h->vofs + h->last_B, sizeof(int), cudaMemcpyDeviceToHost));
    *total_valid = tot;
    if (k_out == nullptr && v_out == nullptr) return;
    const int D = h->D, dh = h->cfg.head_dim, nh = h->cfg.num_heads;
    // layer block: [K | V][head][token (max_tok)][head_dim]
    std::vector<uint16_t> buf((size_t)2 * nh * h->max_tok * dh);
    CUDA_TRY(cudaMemcpy(buf.data(), h->kv + (size_t)(layer / 2) * h->max_tok * 2 * D, buf.size() * 2,
                        cudaMemcpyDeviceToHost));
    for (int r = 0; r < tot; ++r)
      for (int c = 0; c < D; ++c) {
        const int hd = c / dh, d = c % dh;
        if (k_out) k_out[(size_t)r * D + c] = bf16_to_f32(buf[((size_t)hd * h->max_tok + r) * dh + d]);
        if (v_out) v_out[(size_t)r * D + c] = bf16_to_f32(buf[((size_t)(nh + hd) * h->max_tok + r) * dh + d]);
      }
  });
}

int gdit_profile_get_action(gdit_handle* h, const void* backbone_features, int bb_dtype, const uint8_t* vl_mask,
                            const float* state, const int32_t* embodiment_id, const float* init_noise, int num_steps,
                            float* out_actions, int batch, int seq, void* cuda_stream, gdit_kernel_stat* stats,
                            int max_stats) {
  if (!h) return GDIT_EINVAL;
  int count = 0;
  Recorder rec;
  int rc = guarded(h, [&] {
    REQUIRE(stats != nullptr && max_stats > 0, "stats buffer required");
    check_call(h, backbone_features, bb_dtype, vl_mask, state, embodiment_id, init_noise, num_steps, out_actions,
               batch, seq);
    CUDA_TRY(cudaSetDevice(h->cfg.device));
    cudaStream_t s = (cudaStream_t)cuda_stream;
    compute_tables(h, num_steps, s);
    Profile& p = get_profile(h, batch, seq, num_steps, bb_dtype == GDIT_BF16, true);
    IoPtrs io{backbone_features, vl_mask, state, embodiment_id, init_noise, out_actions};
    set_io_kernel<<<1, 1, 0, s>>>(h->io, io);
    CUDA_TRY(cudaGetLastError());
    CUDA_TRY(cudaStreamSynchronize(s));
    enqueue_forward(h, p, s, &rec);
    h->last_stream = s;
    h->last_B = batch;
    CUDA_TRY(cudaStreamSynchronize(s));
    // algorithmic work, now that the routing is known
    std::vector<int> seg(h->C + 1), vofs(batch + 1);
    CUDA_TRY(cudaMemcpy(seg.data(), h->seg, sizeof(int) * (h->C + 1), cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemcpy(vofs.data(), h->vofs, sizeof(int) * (batch + 1), cudaMemcpyDeviceToHost));
    int used = 0;
    for (int c = 0; c < h->C; ++c) used += seg[c + 1] > seg[c];
    const double tok = vofs[batch];
    std::vector<KStat> agg(rec.names.size());
    for (size_t i = 0; i < rec.names.size(); ++i) agg[i].name = rec.names[i];
    const int N = h->N, D = h->D;
    for (auto& e : rec.evs) {
      float ms = 0.0f;
      CUDA_TRY(cudaEventElapsedTime(&ms, e.a, e.b));
      KStat& k = agg[e.cls];
      k.launches += 1;
      k.ms += ms;
      double fl = e.flops, by = e.bytes;
      if (e.op != nullptr) {
        const GemmArgs& a = e.op->args;
        double m = a.M;
        double wb = (double)e.op->weight_bytes;
        if (e.op->rows_kind == 1) m = tok;
        if (e.op->rows_kind == 2) wb *= used;
        fl = 2.0 * m * a.N * a.K;
        by = wb + m * a.K * 2.0 + m * a.N * e.op->out_bytes * (a.epi == EPI_RESID_F32 || a.epi == EPI_EULER ? 2 : 1);
      }
      if (rec.names[e.cls] == "attn_cross") {
        fl = 4.0 * N * tok * D;
        by = tok * 2.0 * D * 2.0 + 2.0 * batch * N * D * 2.0;
      } else if (rec.names[e.cls] == "attn_self") {
        fl = 4.0 * batch * (double)N * N * D;
        by = batch * (double)N * 3 * D * 2.0 + batch * (double)N * D * 2.0;
      }
      k.flops += fl;
      k.bytes += by;
      cudaEventDestroy(e.a);
      cudaEventDestroy(e.b);
    }
    rec.evs.clear();
    for (auto& k : agg) {
      if (count >= max_stats) break;
      gdit_kernel_stat& o = stats[count++];
      std::memset(&o, 0, sizeof(o));
      std::snprintf(o.name, sizeof(o.name), "%s", k.name.c_str());
      o.launches = k.launches;
      o.total_ms = k.ms;
      o.flops = k.flops;
      o.bytes = k.bytes;
    }
  });
  for (auto& e : rec.evs) {
    cudaEventDestroy(e.a);
    cudaEventDestroy(e.b);
  }
  return rc == GDIT_OK ? count : rc;
}

int gdit_test_gemm(const void* A, const void* B, const float* bias, float* C, int M, int N, int K, int bn, int splits,
                   void* cuda_stream) {
  const bool tma_out = getenv("GDIT_TEST_TMA_OUT") != nullptr;   // unit-test knob: exercise the TMA-store epilogue
  const bool pair = getenv("GDIT_TEST_PAIR") != nullptr;         // unit-test knob: the CTA-pair kernel (with TMA store)
  // unit-test knob: the skinny-M kernel, "mt,nu" (a forced plan, items may
  // exceed the SMs) or "0,0" (the planner's choice)
  const char* skinny = getenv("GDIT_TEST_SKINNY");
  g_create_error.clear();
  return guarded(nullptr, [&] {
    REQUIRE(A && B && C, "NULL matrix");
    REQUIRE(M >= 1 && N >= 32 && N % 32 == 0 && K >= 8 && K % 8 == 0, "need M >= 1, N %% 32 == 0, K %% 8 == 0");
    REQUIRE(bn == 32 || bn == 64 || bn == 128 || bn == 256, "bn must be 32, 64, 128 or 256");
    const int nkb = (K + kBK - 1) / kBK;
    REQUIRE(splits >= 1 && splits <= nkb, "splits must be in [1, %d]", nkb);
    set_kernel_attrs();
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    int sms = 0;
    CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    cudaStream_t s = (cudaStream_t)cuda_stream;
    float* ws = nullptr;
    int* counters = nullptr;
    unsigned* err = nullptr;
    const long long nt = (N + bn - 1) / bn, mt = (M + kBM - 1) / kBM;
    CUDA_TRY(cudaMalloc(&err, sizeof(unsigned)));
    CUDA_TRY(cudaMemset(err, 0, sizeof(unsigned)));
    if (splits > 1) {
      CUDA_TRY(cudaMalloc(&ws, sizeof(float) * (size_t)splits * M * N));
      CUDA_TRY(cudaMalloc(&counters, sizeof(int) * (size_t)(mt * nt)));
      CUDA_TRY(cudaMemset(counters, 0, sizeof(int) * (size_t)(mt * nt)));
    }
    GemmOp op;
    op.args = default_args();
    op.args.M = M;
    op.args.N = N;
    op.args.K = K;
    op.args.splits = splits;
    op.args.ws = ws;
    op.args.counters = counters;
    op.args.epi = EPI_F32;
    op.args.bias = bias;
    op.args.out = C;
    op.args.ldo = N;
    op.args.err = err;
    op.bn = bn;
    op.ta = make_tmap(A, M, K, K, kBM);
    op.tb = make_tmap(B, N, K, K, bn);
    op.to = op.ta;
    op.grid = (int)std::min<long long>(mt * nt * splits, sms);
    if (tma_out && splits == 1) {
      op.to = make_out_tmap(C, true, M, N, N);
      op.args.tma_out = 1;
      if (pair && (bn == 128 || bn == 256)) {
        op.pair = true;
        op.ta = make_tmap(A, M, K, K, 128);
        op.tb = make_tmap(B, N, K, K, bn / 2);
        const long long pt = ((M + kPairBM - 1) / kPairBM) * nt;
        op.grid = (int)(2 * std::min<long long>(pt, sms / 2));
      }
    }
    if (skinny != nullptr) {
      REQUIRE(splits == 1, "the skinny-M kernel does not split K");
      op.a_ptr = A;
      op.b_ptr = B;
      int mt = 0, nu = 0;
      REQUIRE(std::sscanf(skinny, "%d,%d", &mt, &nu) == 2, "GDIT_TEST_SKINNY is \"mt,nu\"");
      if (mt == 0) {
        enable_skinny(op, sms);
        REQUIRE(op.sk_mt > 0, "no skinny-M plan for M %d, N %d, K %d", M, N, K);
      } else {
        REQUIRE(mt == 1 || mt == 2 || mt == 3 || mt == 5, "mt must be 1, 2, 3 or 5");
        REQUIRE(nu >= 1 && nu <= sk_max_units(mt), "nu must be in [1, %d]", sk_max_units(mt));
        REQUIRE(N % 8 == 0 && K % 64 == 0, "the skinny-M kernel needs N %% 8 == 0 and K %% 64 == 0");
        const int st = std::min(8, (kSkSmemMax - 1024 - sk_red_bytes(mt, nu) - 64) / sk_stage_bytes(mt, nu));
        REQUIRE(st >= 2, "mt %d, nu %d do not fit shared memory", mt, nu);
        op.sk_mt = mt;
        op.sk_nu = nu;
        op.sk_stages = st;
        op.ta = make_tmap(A, M, K, K, 16 * mt);
        op.tb = make_tmap(B, N, K, K, 8 * nu);
        const long long items = ((M + 16LL * mt - 1) / (16LL * mt)) * ((N / 8 + nu - 1) / nu);
        op.grid = (int)std::min<long long>(items, sms);
      }
    }
    launch_gemm(op, op.args, s, false);
    CUDA_TRY(cudaStreamSynchronize(s));
    unsigned e = 0;
    CUDA_TRY(cudaMemcpy(&e, err, sizeof(unsigned), cudaMemcpyDeviceToHost));
    cudaFree(err);
    if (ws) cudaFree(ws);
    if (counters) cudaFree(counters);
    if (e) throw GditError(GDIT_ETIMEOUT, "GEMM wait timed out");
  });
}

}  // extern "C"

// ====================================================================== no-allocation GEMM
//
// A variant of the split-K GEMM for callers that must not allocate device
// memory at call time.  A robot's control loop is the typical case: cudaMalloc
// and cudaFree can synchronise the whole device and take unbounded time, and
// deployments with a fixed memory budget route every buffer through their own
// pool.  Such callers pass inputs and outputs; the split-K partial sums, the
// per-tile arrival counters and the status word live in the fixed array below,
// which every GPU that loads this library holds until the process exits.
namespace {

constexpr long long kStaticPartialFloats = 1ll << 20;   // 4 MiB of split-K partials
constexpr int kStaticCounters = 4096;                   // output tiles per call

struct StaticScratch {
  unsigned status;
  unsigned pad[63];
  int counters[kStaticCounters];
  float partials[kStaticPartialFloats];
};

static __device__ __align__(256) StaticScratch g_static_scratch;

// Device address of g_static_scratch, looked up once per device.
std::mutex g_static_mu;
StaticScratch* g_static_ptr[64] = {};

StaticScratch* static_scratch_for_current_device() {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  REQUIRE(dev >= 0 && dev < 64, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void* p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_static_scratch));
    g_static_ptr[dev] = static_cast<StaticScratch*>(p);
  }
  return g_static_ptr[dev];
}

}  // namespace

extern "C" int gdit_gemm_static_scratch(const void* A, const void* B, const float* bias, float* C, int M, int N,
                                        int K, int bn, int splits, void* cuda_stream) {
  g_create_error.clear();
  return guarded(nullptr, [&] {
    REQUIRE(A && B && C, "NULL matrix");
    REQUIRE(M >= 1 && N >= 32 && N % 32 == 0 && K >= 8 && K % 8 == 0, "need M >= 1, N %% 32 == 0, K %% 8 == 0");
    REQUIRE(bn == 32 || bn == 64 || bn == 128 || bn == 256, "bn must be 32, 64, 128 or 256");
    const int nkb = (K + kBK - 1) / kBK;
    REQUIRE(splits >= 1 && splits <= nkb, "splits must be in [1, %d]", nkb);
    const long long nt = (N + bn - 1) / bn, mt = (M + kBM - 1) / kBM;
    REQUIRE(mt * nt <= kStaticCounters, "%lld output tiles exceed the fixed scratch's %d tile counters", mt * nt,
            kStaticCounters);
    REQUIRE(splits == 1 || (long long)splits * M * N <= kStaticPartialFloats,
            "split-K partials need %lld floats; the fixed scratch holds %lld (reduce splits, M or N)",
            (long long)splits * M * N, kStaticPartialFloats);
    set_kernel_attrs();
    StaticScratch* sc = static_scratch_for_current_device();
    cudaStream_t s = (cudaStream_t)cuda_stream;
    int dev = 0, sms = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    // the status word and the tile counters must start at zero
    CUDA_TRY(cudaMemsetAsync(&sc->status, 0, sizeof(unsigned), s));
    CUDA_TRY(cudaMemsetAsync(sc->counters, 0, sizeof(int) * (size_t)(mt * nt), s));
    GemmOp op;
    op.args = default_args();
    op.args.M = M;
    op.args.N = N;
    op.args.K = K;
    op.args.splits = splits;
    op.args.ws = sc->partials;
    op.args.counters = sc->counters;
    op.args.epi = EPI_F32;
    op.args.bias = bias;
    op.args.out = C;
    op.args.ldo = N;
    op.args.err = &sc->status;
    op.bn = bn;
    op.ta = make_tmap(A, M, K, K, kBM);
    op.tb = make_tmap(B, N, K, K, bn);
    op.to = op.ta;
    op.grid = (int)std::min<long long>(mt * nt * splits, sms);
    launch_gemm(op, op.args, s, false);
    unsigned e = 0;
    CUDA_TRY(cudaMemcpyAsync(&e, &sc->status, sizeof(unsigned), cudaMemcpyDeviceToHost, s));
    CUDA_TRY(cudaStreamSynchronize(s));
    if (e) throw GditError(GDIT_ETIMEOUT, "GEMM wait timed out");
  });
}
