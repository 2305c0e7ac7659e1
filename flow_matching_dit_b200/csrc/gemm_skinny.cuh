// GEMM for few token rows: out = epilogue(X W^T + b), X [M, K] bf16 with M up
// to a few hundred, W [N, K] bf16 (the DiT linears of the Isaac-GR00T
// architecture page, "Transformer block structure", at batches of a few
// samples: M = B (H + 1) rows).
//
// There every weight byte meets only M rows: the work is a weight stream plus
// one read of X per CTA.  The tensor-core GEMM's 128-row tiles would put a
// 1024-wide linear on 8 to 16 column tiles, most SMs idle.  Here the output is
// cut into items -- a block of 16 MT rows times nu units of 8 output features
// (nu runtime, at most sk_max_units(MT)) -- spread over every SM:
//
//   * a CTA streams its item's weight rows (8 nu rows, contiguous in W) and
//     activation rows through a ring of K-chunks of 256 columns: per chunk four
//     TMA boxes (64 columns, 128-byte swizzle) of each, on one mbarrier per
//     stage (one copy per row was tried first: 70-odd 256-byte copies per
//     chunk made a 1024-wide linear at 136 rows take 50 us); the weight boxes
//     of the first chunks (and an L2 request for the rest of the first item's
//     rows) are issued before the dependency wait, so they stream while the
//     previous kernel finishes;
//   * the 8 warps take two k-steps of each chunk each (bf16 mma.sync
//     m16n8k16: the rows as A, the weight rows as B) into MT x nu accumulator
//     fragments;
//   * at the end of an item the warps' partial sums are added in a fixed
//     order through shared memory (4 + 4 warps, then 4 partials per output)
//     and the epilogue (bias, GELU / ReLU, bf16 or f32 store, or the f32
//     residual add), one accumulator fragment per warp at a time, writes each
//     output once: the result does not depend on scheduling.
#pragma once

#include "attention.cuh"   // mma_bf16_16816, ldmatrix_x4
#include "gemm_tc.cuh"     // Epi kinds, gelu_erf
#include "ptx.cuh"

namespace gdit {

constexpr int kSkWarps = 8;
constexpr int kSkThreads = 32 * kSkWarps;
constexpr int kSkKC = 256;                       // K columns per chunk (four 64-column boxes): two k-steps per warp
constexpr int kSkBoxes = kSkKC / 64;
constexpr int kSkSmemMax = 227 * 1024 - 1024;    // dynamic shared memory budget
static_assert(kSkKC == 32 * kSkWarps, "two k-steps of a chunk per warp");

// Units an item may hold for MT row tiles: MT x units accumulator fragments
// (4 registers each) per thread.
__host__ __device__ constexpr int sk_max_units(int mt) { return mt == 1 ? 16 : (mt == 2 ? 16 : (mt == 3 ? 12 : 7)); }

struct SkinnyArgs {
  const __nv_bfloat16* W;   // [N, K] row-major (the L2 request; the copies go through the maps)
  const float* bias;        // [N] or nullptr
  void* out;                // [M, ldo]: bf16 or f32 by epi
  long long ldo;
  int M, N, K;
  int epi;                  // EPI_BF16, EPI_GELU_BF16, EPI_RELU_BF16, EPI_F32 or EPI_RESID_F32
  int nu;                   // units of 8 features per item (<= sk_max_units(MT))
  int stages;               // ring depth
  unsigned* err;
};

// Shared memory (from a 1024-byte boundary): `stages` chunks of [activation
// boxes of columns 0-63, 64-127, 128-191, 192-255 | weight boxes of the
// same], 128-byte rows (16 MT activation rows, 8 nu weight rows: every box a
// multiple of 1024 bytes), the cross-warp partial sums (4 sets of MT x nu
// fragments, 32 lanes x 4 floats each), the stage barriers.
__host__ __device__ inline int sk_stage_bytes(int mt, int nu) { return kSkBoxes * (16 * mt + 8 * nu) * 128; }
__host__ __device__ inline int sk_red_bytes(int mt, int nu) { return 4 * mt * nu * 32 * 16; }
__host__ __device__ inline int sk_smem_bytes(int mt, int nu, int stages) {
  return 1024 + stages * sk_stage_bytes(mt, nu) + sk_red_bytes(mt, nu) + stages * 8;
}

template <int MT>
__global__ void __launch_bounds__(kSkThreads, 1)
    gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const SkinnyArgs a) {
  constexpr int NUM = sk_max_units(MT);
  constexpr int ROWS = 16 * MT;
  constexpr int XB = ROWS * 128;   // one activation box
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ int s_fail;
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);   // the 128-byte swizzle repeats every 1024 bytes
  const int S = a.stages, nu = a.nu;
  const int WB = 8 * nu * 128;     // one weight box
  const int stage_b = sk_stage_bytes(MT, nu);
  float4* red = reinterpret_cast<float4*>(smem + S * stage_b);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * stage_b + sk_red_bytes(MT, nu));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int nrb = (a.M + ROWS - 1) / ROWS;
  const int units = a.N / 8;
  const int nub = (units + nu - 1) / nu;
  const int items = nrb * nub;
  const int nch = (a.K + kSkKC - 1) / kSkKC;   // (boxes past K read zeros)
  // this CTA's items: blockIdx.x, blockIdx.x + gridDim.x, ... (grid <= items)
  const int my_items = (int)blockIdx.x < items ? (items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total = my_items * nch;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
    s_fail = 0;
  }
  __syncthreads();

  // chunk q of this CTA: item (row block rb, unit block ub; consecutive CTAs
  // share a unit block) and K-chunk q mod nch
  auto item_of = [&](int q, int& r0, int& rows, int& u0, int& nuv) {
    const int it = (int)blockIdx.x + (q / nch) * (int)gridDim.x;
    const int rb = it % nrb, ub = it / nrb;
    r0 = rb * ROWS;
    rows = min(ROWS, a.M - r0);
    u0 = ub * nu;
    nuv = min(nu, units - u0);
  };
  // thread 0: the weight boxes (with the stage's byte count: whole boxes,
  // rows past the matrix zero-filled) and/or the activation boxes of chunk q
  // into stage q mod S
  auto issue = [&](int q, bool wpart, bool xpart) {
    int r0, rows, u0, nuv;
    item_of(q, r0, rows, u0, nuv);
    const int c = q % nch;
    uint8_t* st = smem + (q % S) * stage_b;
    uint64_t* bar = &full[q % S];
    if (wpart) {
      mbar_arrive_expect_tx(bar, (uint32_t)stage_b);
      for (int b = 0; b < kSkBoxes; ++b) tma_load_2d(st + kSkBoxes * XB + b * WB, &tmW, bar, c * kSkKC + 64 * b, u0 * 8);
    }
    if (xpart)
      for (int b = 0; b < kSkBoxes; ++b) tma_load_2d(st + b * XB, &tmX, bar, c * kSkKC + 64 * b, r0);
  };

  // The weights depend on no earlier kernel: their rows for the first chunks
  // go out before the dependency wait, with an L2 request for the rest of the
  // first item's weight rows.
  const int pre = min(total, S);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
    for (int q = 0; q < pre; ++q) issue(q, true, false);
    if (my_items > 0) {
      int r0, rows, u0, nuv;
      item_of(0, r0, rows, u0, nuv);
      l2_prefetch(a.W + (long long)u0 * 8 * a.K, (uint32_t)(8 * nuv) * (uint32_t)a.K * 2u);
    }
  }
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0)
    for (int q = 0; q < pre; ++q) issue(q, false, true);

  float acc[MT][NUM][4];
#pragma unroll
  for (int t = 0; t < MT; ++t)
#pragma unroll
    for (int j = 0; j < NUM; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[t][j][e] = 0.0f;

  // this warp's two k-steps in a chunk: box (warp / 2), 16-byte column
  // pieces 4 (warp % 2) .. + 3 (swizzled: piece p of row r at (p ^ (r % 8)) * 16)
  const int box = warp >> 1;
  const int pa = (warp & 1) * 4 + (lane >> 4);   // A, k-step i: piece pa + 2i (lanes 16-31: columns 8-15)
  const int pb = (warp & 1) * 4 + (lane >> 3);   // B: lanes 8i .. 8i + 7 address piece +i (two k-steps, x4)
  int r0 = 0, rows = 1, u0 = 0, nuv = 0;
  int q = 0;
  for (; q < total; ++q) {
    const int s = q % S, c = q % nch;
    if (c == 0) item_of(q, r0, rows, u0, nuv);
    if (!mbar_wait(&full[s], (uint32_t)(q / S) & 1u, a.err)) s_fail = 1;
    if (s_fail == 0) {
      const uint8_t* st = smem + s * stage_b;
      uint32_t af[2][MT][4];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          // rows past the matrix are zero (their sums are never stored)
          const int ar = t * 16 + (lane & 15);
          ldmatrix_x4(af[i][t][0], af[i][t][1], af[i][t][2], af[i][t][3],
                      st + box * XB + ar * 128 + (((pa + 2 * i) ^ (ar & 7)) << 4));
        }
      const uint8_t* wb = st + kSkBoxes * XB + box * WB + (lane & 7) * 128 + ((pb ^ (lane & 7)) << 4);
#pragma unroll
      for (int j = 0; j < NUM; ++j) {
        if (j < nuv) {
          uint32_t b[4];
          ldmatrix_x4(b[0], b[1], b[2], b[3], wb + j * 8 * 128);
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            mma_bf16_16816(acc[t][j], af[0][t][0], af[0][t][1], af[0][t][2], af[0][t][3], b[0], b[1]);
            mma_bf16_16816(acc[t][j], af[1][t][0], af[1][t][1], af[1][t][2], af[1][t][3], b[2], b[3]);
          }
        }
      }
    }
    if (c == nch - 1) {
      // item done: warps 4-7 hand their sums to warps 0-3, which store the
      // four partial sets; each output then adds its four partials in order
      if (warp >= 4) {
#pragma unroll
        for (int t = 0; t < MT; ++t)
#pragma unroll
          for (int j = 0; j < NUM; ++j)
            if (j < nuv)
              red[(((warp - 4) * MT + t) * nu + j) * 32 + lane] =
                  make_float4(acc[t][j][0], acc[t][j][1], acc[t][j][2], acc[t][j][3]);
      }
      __syncthreads();
      if (warp < 4) {
#pragma unroll
        for (int t = 0; t < MT; ++t)
#pragma unroll
          for (int j = 0; j < NUM; ++j)
            if (j < nuv) {
              float4& p = red[((warp * MT + t) * nu + j) * 32 + lane];
              const float4 o = p;
              p = make_float4(acc[t][j][0] + o.x, acc[t][j][1] + o.y, acc[t][j][2] + o.z, acc[t][j][3] + o.w);
            }
      }
      __syncthreads();
      // fragment (t, j) on warp (t nu + j) mod 8: lane l holds rows
      // 16 t + l / 4 and + 8, columns 8 j + 2 (l mod 4) and + 1
      for (int f = warp; f < MT * nuv; f += kSkWarps) {
        const int t = f / nuv, j = f - t * nuv;
        float4 p = red[(t * nu + j) * 32 + lane];
#pragma unroll
        for (int w = 1; w < 4; ++w) {
          const float4 o = red[((w * MT + t) * nu + j) * 32 + lane];
          p.x += o.x; p.y += o.y; p.z += o.z; p.w += o.w;
        }
        const int col = (u0 + j) * 8 + 2 * (lane & 3);
        if (a.bias != nullptr) {
          const float2 b = __ldg(reinterpret_cast<const float2*>(a.bias + col));
          p.x += b.x; p.y += b.y; p.z += b.x; p.w += b.y;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int m = t * 16 + (lane >> 2) + 8 * h;
          if (m >= rows) continue;
          float v0 = h ? p.z : p.x, v1 = h ? p.w : p.y;
          const long long o = (long long)(r0 + m) * a.ldo + col;
          if (a.epi == EPI_RESID_F32) {
            float2* op = reinterpret_cast<float2*>(reinterpret_cast<float*>(a.out) + o);
            const float2 old = *op;
            *op = make_float2(old.x + v0, old.y + v1);
          } else if (a.epi == EPI_F32) {
            *reinterpret_cast<float2*>(reinterpret_cast<float*>(a.out) + o) = make_float2(v0, v1);
          } else {
            if (a.epi == EPI_GELU_BF16) {
              v0 = gelu_erf(v0);
              v1 = gelu_erf(v1);
            } else if (a.epi == EPI_RELU_BF16) {
              v0 = fmaxf(v0, 0.0f);
              v1 = fmaxf(v1, 0.0f);
            }
            *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(a.out) + o) = pack_bf16x2(v0, v1);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int j = 0; j < NUM; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[t][j][e] = 0.0f;
    }
    // every warp is done with stage s (and with the partial sums)
    __syncthreads();
    if (s_fail != 0) break;
    if (threadIdx.x == 0 && q + S < total) {
      fence_proxy_async_smem();   // this CTA's reads of the stage precede the copies into it
      issue(q + S, true, true);
    }
  }
  // after a timeout: the copies still in flight (chunks q .. q + S - 1) land
  // before the CTA exits
  if (q < total && threadIdx.x == 0) {
    const unsigned long long t0 = globaltimer_ns();
    for (int i = q; i < min(total, q + S); ++i)
      while (!mbar_try_wait(&full[i % S], (uint32_t)(i / S) & 1u) && globaltimer_ns() - t0 < 10000000ull) {
      }
  }
}

}  // namespace gdit
