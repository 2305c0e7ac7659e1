// The whole K-step Euler loop of one sample (B = 1, N = H + 1 <= 32 tokens)
// as one persistent kernel (Isaac-GR00T architecture page, "Inference
// (denoising)": action encoder -> 32 DiT blocks -> action decoder -> Euler
// update, K times).
//
// At B = 1 every linear is a weight stream (17 tokens against a 1024-wide
// weight matrix), and the per-kernel fixed cost of separate launches (launch,
// TMEM allocation, pipeline fill, tail) dominates the HBM time of each matrix.
// Here one launch runs all phases.  A phase is either
//   a GEMM phase: out = epilogue(X W^T), the 16-feature units of W spread over
//   the CTAs, each unit's K split over the CTA's 8 warps (bf16 mma.sync
//   m16n8k16, weights as the 16-row A operand, tokens as B), reduced in shared
//   memory.  W and X move in chunks of up to 1024 columns through 2-slot rings
//   of padded shared memory, copied by all 256 threads with cp.async (one
//   memory round trip per chunk, no serial issue); the first two W chunks of a
//   phase are requested before the phase waits for its inputs, and the bias
//   and the old residual tile come with the X chunk.  X is a bf16 activation
//   in global memory, or LN(h) / AdaLN(h) computed by the CTA from h rows
//   staged in shared memory, or
//   an attention phase: one CTA per head, the 8 warps split the keys
//   (the routine of attention.cuh).
// Phases are ordered by arrival counters in global memory: the CTAs that work
// in phase p wait until every CTA that worked in phase p-1 has arrived (each
// of those waited for p-2, so the order is transitive), then arrive on p.
// Before waiting, a CTA requests its next weight slices into L2
// (cp.async.bulk.prefetch), so weight streaming overlaps the wait.  Every
// wait is bounded; on expiry the status word records a timeout and all CTAs
// return.
#pragma once

#include "attention.cuh"
#include "gemm_tc.cuh"   // Epi kinds, gelu_erf, swish_f
#include "ptx.cuh"

namespace gdit {

constexpr int kSmallThreads = 256;
constexpr int kSmallWarps = 8;
constexpr int kSmallMaxTok = 32;
constexpr int kSmallMaxD = 1024;
constexpr int kSmallMaxLayers = 64;
constexpr int kSmallKC = 1024;    // widest K chunk moved through shared memory
constexpr int kSmallKCP = kSmallKC + 8;   // padded row (conflict-free fragment loads)

// shared-memory layout of a GEMM phase (bytes)
constexpr int kSmW = 0;                                          // 2 x [16][KCP] bf16
constexpr int kSmX = kSmW + 2 * 16 * kSmallKCP * 2;              // 2 x [32][KCP] bf16
constexpr int kSmRed = kSmX + 2 * kSmallMaxTok * kSmallKCP * 2;  // [8][32][17] f32 (warp, token, feature)
constexpr int kRedLd = 17;                                       // padded feature stride
constexpr int kSmHold = kSmRed + kSmallWarps * kSmallMaxTok * kRedLd * 4;   // 2 x [32][16] f32 (old h)
constexpr int kSmBias = kSmHold + 2 * kSmallMaxTok * 16 * 4;     // 2 x [16] f32
constexpr int kSmStat = kSmBias + 2 * 16 * 4;                    // [32][2] f32
constexpr int kSmGemmEnd = kSmStat + kSmallMaxTok * 2 * 4;
// LN stages the f32 h rows over X slot 1 and the reduction buffer (both free
// then): rows * D * 4 bytes must fit (the host checks it before choosing this loop)
constexpr int kSmHStage = kSmX + kSmallMaxTok * kSmallKCP * 2;
constexpr int kSmHStageBytes = kSmHold - kSmHStage;

struct SmallLayer {
  const __nv_bfloat16* wq;   // [nq, D]: Q (cross) or Q|K|V (self)
  const float* bq;
  const __nv_bfloat16* wo;
  const float* bo;
  const float* ln3g;
  const float* ln3b;
  const __nv_bfloat16* wff1;
  const float* bff1;
  const __nv_bfloat16* wff2;
  const float* bff2;
  const __nv_bfloat16* kv;   // cross layers: this layer's block of the head-major K/V cache
};

struct SmallPlan {
  int D, F, A, H, N, nh, dh, L, K, C;
  float eps, scale_log2;
  long long max_tok;
  // activations
  float* h;
  float* x;
  __nv_bfloat16* xb;
  __nv_bfloat16 *abf, *zbf, *qkv, *o, *f, *ybf, *rbf;
  const float* sfeat;
  const int* seg;
  const int* vofs;
  // per-K tables: AdaLN [K][L+1][2D], timestep term of the action encoder's W2 [K][C][D]
  const float* ada;
  const float* tw2;
  // weights (category-specific ones as [C][out][in])
  const __nv_bfloat16 *wa1t, *wa2at, *wa3t, *wd1t, *wd2t, *proj_w;
  const float *ba1, *ba3, *bd1, *bd2, *proj_b;
  SmallLayer layers[kSmallMaxLayers];
  int* counters;             // one per phase, zero at launch
  struct SmallPhase* phases; // descriptor of every phase, written by small_describe_kernel
  unsigned* err;
};

struct SmallGemm {
  const __nv_bfloat16* W;
  int N, K;
  const float* bias;         // [N] or nullptr
  const float* vec;          // swish: additive term [N] (bias included)
  int epi;
  int x_mode;                // 0: X from global bf16; 1: LN(h) into shared memory
  const __nv_bfloat16* X;
  int ldx;
  int ln_mode;               // 0: AdaLN (1 + p0) and p1; 1: affine p0, p1
  const float* p0;
  const float* p1;
  int h_row_off;             // first row of h normalised
  int rows;                  // tokens
  void* out;
  int ldo;
  int out_row_off;
  __nv_bfloat16* out2;
  float alpha;
  const float* state_row;    // EPI_F32 into h: also write h row 0 from this vector
};

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void l2_prefetch(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- phase ordering

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Thread 0 waits (acquire) until `target` CTAs have arrived on `phase`.
__device__ __forceinline__ bool small_wait(const SmallPlan& P, int phase, int target) {
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    int ok = 1;
    if (phase >= 0 && target > 0) {
      const int* c = P.counters + phase;
      if (ld_acquire(c) < target) {
        const unsigned long long t0 = globaltimer_ns();
        while (ld_acquire(c) < target) {
          if (*reinterpret_cast<volatile unsigned*>(P.err) & DEV_ERR_TIMEOUT) { ok = 0; break; }
          if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
            atomicOr(P.err, DEV_ERR_TIMEOUT);
            ok = 0;
            break;
          }
        }
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// All threads' writes of the phase, then one release increment.
__device__ __forceinline__ void small_arrive(const SmallPlan& P, int phase) {
  __syncthreads();
  if (threadIdx.x == 0) red_release_add(P.counters + phase, 1);
}

__device__ __forceinline__ int gemm_units(const SmallGemm& g) { return g.N / 16; }
__device__ __forceinline__ int workers(int units) { return units < (int)gridDim.x ? units : (int)gridDim.x; }

__device__ __forceinline__ void prefetch_gemm_weights(const SmallGemm& g) {
  if (threadIdx.x != 0) return;
  const uint32_t bytes = 16u * (uint32_t)g.K * 2u;
  for (int u = blockIdx.x; u < gemm_units(g); u += gridDim.x) l2_prefetch(g.W + (size_t)u * 16 * g.K, bytes);
}

// ---------------------------------------------------------------- GEMM phase

__device__ __forceinline__ int small_kc(const SmallGemm& g) { return g.K < kSmallKC ? g.K : kSmallKC; }
__device__ __forceinline__ int small_nchunks(const SmallGemm& g) { return g.K / small_kc(g); }
__device__ __forceinline__ int small_my_units(const SmallGemm& g) {
  const int u = gemm_units(g);
  return (int)blockIdx.x < u ? (u - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
}
__device__ __forceinline__ int small_items(const SmallGemm& g) { return small_my_units(g) * small_nchunks(g); }
__device__ __forceinline__ int small_unit(const SmallGemm& g, int t) {
  return (int)blockIdx.x + (t / small_nchunks(g)) * (int)gridDim.x;
}

// Item t's W chunk (16 rows x kc) -> ring slot t & 1: lane 0 of warp 0 arms the
// slot's mbarrier with the byte count, then lanes 0..15 each issue one row as
// a bulk async copy (the copy engine, not the load/store queue).
__device__ __forceinline__ void small_copy_w(const SmallGemm& g, int t, uint8_t* smem, uint64_t* wbar) {
  if (threadIdx.x >= 32) return;
  const int kc = small_kc(g), c = t % small_nchunks(g);
  const int slot = t & 1;
  if (threadIdx.x == 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&wbar[slot], 16u * (uint32_t)kc * 2u);
  }
  __syncwarp();
  if (threadIdx.x < 16) {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(smem + kSmW) + slot * 16 * kSmallKCP + threadIdx.x * kSmallKCP;
    const __nv_bfloat16* src = g.W + ((size_t)small_unit(g, t) * 16 + threadIdx.x) * g.K + (size_t)c * kc;
    bulk_g2s(dst, src, (uint32_t)kc * 2u, &wbar[slot]);
  }
}

// cp.async of item t's X chunk (rows x kc), and at a unit's first chunk its
// bias and (residual epilogue) its old h tile.
__device__ __forceinline__ void small_copy_x(const SmallGemm& g, int t, uint8_t* smem, bool ln) {
  const int kc = small_kc(g), nch = small_nchunks(g), c = t % nch;
  if (!ln) {
    const int pieces = kc / 8;
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(smem + kSmX) + (t & 1) * kSmallMaxTok * kSmallKCP;
    const __nv_bfloat16* src = g.X + (size_t)c * kc;
    for (int i = threadIdx.x; i < g.rows * pieces; i += kSmallThreads) {
      const int r = i / pieces, q = i - r * pieces;
      cp_async16(dst + r * kSmallKCP + q * 8, src + (size_t)r * g.ldx + q * 8, true);
    }
  }
  if (c == 0) {
    const int f0 = small_unit(g, t) * 16;
    const int ub = (t / nch) & 1;
    const float* bsrc = g.epi == EPI_SWISH_VEC_BF16 ? g.vec : g.bias;
    if (bsrc != nullptr && threadIdx.x < 4)
      cp_async16(reinterpret_cast<float*>(smem + kSmBias) + ub * 16 + threadIdx.x * 4, bsrc + f0 + threadIdx.x * 4, true);
    if (g.epi == EPI_RESID_F32 || g.epi == EPI_EULER) {
      float* hold = reinterpret_cast<float*>(smem + kSmHold) + ub * kSmallMaxTok * 16;
      for (int i = threadIdx.x; i < g.rows * 4; i += kSmallThreads) {
        const int r = i >> 2, q = i & 3;
        cp_async16(hold + r * 16 + q * 4,
                   reinterpret_cast<const float*>(g.out) + (size_t)(g.out_row_off + r) * g.ldo + f0 + q * 4, true);
      }
    }
  }
}

// Request the first (up to two) W chunks of a phase: done before the phase
// waits for its inputs, since weights depend on no earlier phase.
__device__ __forceinline__ void small_prefetch_w(const SmallGemm& g, uint8_t* smem, uint64_t* wbar) {
  const int n = small_items(g);
  for (int t = 0; t < 2 && t < n; ++t) small_copy_w(g, t, smem, wbar);
}

// LN(h rows) -> bf16 X slot 0: rows staged in shared memory (one round trip);
// per-row mean and E[x^2] in one pass over the staged row.
__device__ __forceinline__ void small_ln_to_smem(const SmallGemm& g, const SmallPlan& P, uint8_t* smem) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = P.D, d4 = D / 4;
  float* hs = reinterpret_cast<float*>(smem + kSmHStage);
  for (int i = threadIdx.x; i < g.rows * d4; i += kSmallThreads) {
    const int r = i / d4, q = i - r * d4;
    cp_async16(hs + (size_t)r * D + q * 4, P.h + (size_t)(g.h_row_off + r) * D + q * 4, true);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  float* st = reinterpret_cast<float*>(smem + kSmStat);
  for (int r = warp; r < g.rows; r += kSmallWarps) {
    const float4* row = reinterpret_cast<const float4*>(hs + (size_t)r * D);
    float s0 = 0.0f, s1 = 0.0f, q0 = 0.0f, q1 = 0.0f;
    for (int c = lane; c < d4; c += 32) {
      const float4 v = row[c];
      s0 += v.x + v.y;
      s1 += v.z + v.w;
      q0 += v.x * v.x + v.y * v.y;
      q1 += v.z * v.z + v.w * v.w;
    }
    float sum = s0 + s1, sq = q0 + q1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
    }
    if (lane == 0) {
      const float mean = sum / (float)D;
      st[r * 2] = mean;
      st[r * 2 + 1] = rsqrtf(fmaxf(sq / (float)D - mean * mean, 0.0f) + P.eps);
    }
  }
  __syncthreads();
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem + kSmX);
  for (int c4 = threadIdx.x; c4 < d4; c4 += kSmallThreads) {
    const float4 a = reinterpret_cast<const float4*>(g.p0)[c4];
    const float4 b = reinterpret_cast<const float4*>(g.p1)[c4];
    for (int r = 0; r < g.rows; ++r) {
      const float4 v = reinterpret_cast<const float4*>(hs + (size_t)r * D)[c4];
      const float mean = st[r * 2], rstd = st[r * 2 + 1];
      float y0 = (v.x - mean) * rstd, y1 = (v.y - mean) * rstd, y2 = (v.z - mean) * rstd, y3 = (v.w - mean) * rstd;
      if (g.ln_mode == 0) {
        y0 = y0 * (1.0f + a.x) + b.x;
        y1 = y1 * (1.0f + a.y) + b.y;
        y2 = y2 * (1.0f + a.z) + b.z;
        y3 = y3 * (1.0f + a.w) + b.w;
      } else {
        y0 = y0 * a.x + b.x;
        y1 = y1 * a.y + b.y;
        y2 = y2 * a.z + b.z;
        y3 = y3 * a.w + b.w;
      }
      uint2 w;
      w.x = pack_bf16x2(y0, y1);
      w.y = pack_bf16x2(y2, y3);
      *reinterpret_cast<uint2*>(xs + (size_t)r * kSmallKCP + 4 * c4) = w;
    }
  }
  __syncthreads();
}

__device__ __forceinline__ void small_epilogue(const SmallGemm& g, int n, int tok, float v, float bias,
                                               float hold) {
  if (g.epi == EPI_SWISH_VEC_BF16) {
    v = swish_f(v + bias);
  } else {
    v += bias;
  }
  const size_t idx = (size_t)(g.out_row_off + tok) * g.ldo + n;
  switch (g.epi) {
    case EPI_BF16:
    case EPI_SWISH_VEC_BF16:
      reinterpret_cast<__nv_bfloat16*>(g.out)[idx] = __float2bfloat16_rn(v);
      break;
    case EPI_GELU_BF16:
      reinterpret_cast<__nv_bfloat16*>(g.out)[idx] = __float2bfloat16_rn(gelu_erf(v));
      break;
    case EPI_RELU_BF16:
      reinterpret_cast<__nv_bfloat16*>(g.out)[idx] = __float2bfloat16_rn(fmaxf(v, 0.0f));
      break;
    case EPI_F32:
      reinterpret_cast<float*>(g.out)[idx] = v;
      break;
    case EPI_RESID_F32:
      reinterpret_cast<float*>(g.out)[idx] = hold + v;
      break;
    default: {   // EPI_EULER
      const float xn = hold + g.alpha * v;
      reinterpret_cast<float*>(g.out)[idx] = xn;
      g.out2[(size_t)tok * g.ldo + n] = __float2bfloat16_rn(xn);
    }
  }
}

// One GEMM phase.  W chunks: item t waits on mbarrier slot t & 1 for its
// (wuse)-th completion, where wuse counts this CTA's earlier uses of the slot
// over the whole loop.  X chunks (and the bias / old-h tiles): cp.async groups,
// the X groups of items 0 and 1 (or the LN staging) first, then one group per
// later item; each item waits until at most one younger group is pending.
__device__ __forceinline__ void small_gemm_phase(const SmallGemm& g, const SmallPlan& P, uint8_t* smem,
                                                 uint64_t* wbar, uint32_t* wuse) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, tig = lane & 3;
  const __nv_bfloat16* wsm = reinterpret_cast<const __nv_bfloat16*>(smem + kSmW);
  const __nv_bfloat16* xsm = reinterpret_cast<const __nv_bfloat16*>(smem + kSmX);
  float* red = reinterpret_cast<float*>(smem + kSmRed);
  const float* holds = reinterpret_cast<const float*>(smem + kSmHold);
  const float* biases = reinterpret_cast<const float*>(smem + kSmBias);
  const int nch = small_nchunks(g), kc = small_kc(g);
  const int n_items = small_items(g);
  const bool ln = g.x_mode == 1;   // LN phases have K = D <= kSmallKC: one chunk per unit, X in slot 0
  for (int t = 0; t < 2; ++t) {
    if (t < n_items) small_copy_x(g, t, smem, ln);
    cp_async_commit();
  }
  if (ln) small_ln_to_smem(g, P, smem);   // waits for every group so far
  const int ks = kc / 16;
  const int ks0 = warp * ks / kSmallWarps, ks1 = (warp + 1) * ks / kSmallWarps;
  const int nt_act = (g.rows + 7) / 8;
  float acc[4][4];
  for (int t = 0; t < n_items; ++t) {
    const int c = t % nch;
    if (c == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    }
    cp_async_wait<1>();
    if (!mbar_wait(&wbar[t & 1], wuse[t & 1] & 1u, P.err)) {
      // a timed-out copy: leave the phase (the loop returns at its next wait)
      __syncthreads();
      return;
    }
    ++wuse[t & 1];
    __syncthreads();
    // ldmatrix addressing: lane l supplies row (l & 15) of the tile, column half (l >> 4)
    const int lr = lane & 15, lh = (lane >> 4) * 8;
    const __nv_bfloat16* wtile = wsm + (size_t)(t & 1) * 16 * kSmallKCP + lr * kSmallKCP + lh;
    const __nv_bfloat16* xtile = xsm + (size_t)(ln ? 0 : (t & 1)) * kSmallMaxTok * kSmallKCP;
    for (int k16 = ks0; k16 < ks1; ++k16) {
      const int k = k16 * 16;
      // A (16 weight rows x 16 k): matrices (rows 0-7 | 8-15) x (k 0-7 | 8-15) -> a0 a1 a2 a3
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(a0, a1, a2, a3, wtile + k);
      // B for token tiles (0,1) and (2,3): rows = tokens, k contiguous -> (b0, b1) per tile
      uint32_t b[4][2];
#pragma unroll
      for (int pair = 0; pair < 2; ++pair) {
        if (pair * 2 < nt_act) {
          // lanes 0-7: tokens 16p+0..7 k 0-7; 8-15: same tokens k 8-15; 16-23: tokens 16p+8..15 k 0-7; 24-31: k 8-15
          const int tok = pair * 16 + ((lane >> 4) << 3) + (lane & 7);
          const int kh = ((lane >> 3) & 1) * 8;
          ldmatrix_x4(b[pair * 2][0], b[pair * 2][1], b[pair * 2 + 1][0], b[pair * 2 + 1][1],
                      xtile + (size_t)tok * kSmallKCP + k + kh);
        }
      }
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
        if (nt < nt_act) mma_bf16_16816(acc[nt], a0, a1, a2, a3, b[nt][0], b[nt][1]);
    }
    __syncthreads();   // slot t & 1 consumed
    if (c == nch - 1) {
      // unit done: reduce the 8 warps' partials, epilogue
      const int f0 = small_unit(g, t) * 16;
      const int ub = (t / nch) & 1;
      float* rw = red + warp * kSmallMaxTok * kRedLd;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int tok = nt * 8 + tig * 2;
        rw[tok * kRedLd + gr] = acc[nt][0];
        rw[(tok + 1) * kRedLd + gr] = acc[nt][1];
        rw[tok * kRedLd + gr + 8] = acc[nt][2];
        rw[(tok + 1) * kRedLd + gr + 8] = acc[nt][3];
      }
      __syncthreads();
      const bool has_bias = (g.epi == EPI_SWISH_VEC_BF16 ? g.vec : g.bias) != nullptr;
      for (int idx = threadIdx.x; idx < 16 * g.rows; idx += kSmallThreads) {
        const int tok = idx >> 4, fi = idx & 15;   // consecutive threads: consecutive features of a row
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kSmallWarps; ++w) v += red[(w * kSmallMaxTok + tok) * kRedLd + fi];
        small_epilogue(g, f0 + fi, tok, v, has_bias ? biases[ub * 16 + fi] : 0.0f,
                       holds[(ub * kSmallMaxTok + tok) * 16 + fi]);
      }
      if (g.state_row != nullptr && threadIdx.x < 16)
        reinterpret_cast<float*>(g.out)[f0 + threadIdx.x] = g.state_row[f0 + threadIdx.x];
      __syncthreads();   // red and the unit's tiles are reused
    }
    // item t + 2 reuses slot t & 1 and, at a unit start, the tiles of unit t
    if (t + 2 < n_items) {
      small_copy_w(g, t + 2, smem, wbar);
      small_copy_x(g, t + 2, smem, ln);
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------- attention phase (one CTA per head)

template <int DH>
__device__ __forceinline__ void small_attention_phase(const AttnArgs& a, int head, uint8_t* smem) {
  using SM = AttnSmem<2, DH>;
  constexpr int NW = kSmallWarps;
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sKV = sQ + SM::Q_ELEMS;
  float* sO = reinterpret_cast<float*>(smem + (SM::Q_ELEMS + NW * SM::RING_ELEMS) * 2);
  float* sML = sO + NW * 32 * DH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, tig = lane & 3;
  int k_begin, n_keys;
  attn_key_range(a, 0, k_begin, n_keys);
  attn_load_q<2, DH>(a, 0, head, sQ, threadIdx.x, kSmallThreads);
  __syncthreads();
  float o[2][DH / 8][4];
  float mrow[2][2], lrow[2][2];
  attn_init<2, DH>(o, mrow, lrow);
  attn_stream_chunks<2, DH>(a, head, k_begin, n_keys, warp, NW, sQ, sKV + warp * SM::RING_ELEMS, o, mrow, lrow);
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float l = lrow[mt][hr];
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      const int row = mt * 16 + gr + hr * 8;
      if (tig == 0) {
        sML[(warp * 32 + row) * 2 + 0] = mrow[mt][hr];
        sML[(warp * 32 + row) * 2 + 1] = l;
      }
      float* orow = sO + (warp * 32 + row) * DH;
#pragma unroll
      for (int nd = 0; nd < DH / 8; ++nd) {
        orow[nd * 8 + tig * 2 + 0] = o[mt][nd][hr * 2 + 0];
        orow[nd * 8 + tig * 2 + 1] = o[mt][nd][hr * 2 + 1];
      }
    }
  }
  __syncthreads();
  __nv_bfloat16* obase = a.out + head * DH;
  for (int i = threadIdx.x; i < a.n_tok * (DH / 2); i += kSmallThreads) {
    const int row = i / (DH / 2);
    const int d = (i - row * (DH / 2)) * 2;
    float mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mt = fmaxf(mt, sML[(w * 32 + row) * 2]);
    float r0 = 0.0f, r1 = 0.0f;
    if (mt != -INFINITY) {
      float l = 0.0f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = sML[(w * 32 + row) * 2];
        const float f = (mw == -INFINITY) ? 0.0f : exp2f(mw - mt);
        l += f * sML[(w * 32 + row) * 2 + 1];
        r0 += f * sO[(w * 32 + row) * DH + d];
        r1 += f * sO[(w * 32 + row) * DH + d + 1];
      }
      const float inv = 1.0f / l;
      r0 *= inv;
      r1 *= inv;
    }
    *reinterpret_cast<uint32_t*>(obase + (size_t)row * a.out_ld + d) = pack_bf16x2(r0, r1);
  }
  __syncthreads();   // shared memory is reused by the next phase
}

template <int DH>
struct SmallSmem {
  static constexpr int GEMM = kSmGemmEnd;
  static constexpr int ATTN = (AttnSmem<2, DH>::Q_ELEMS + kSmallWarps * AttnSmem<2, DH>::RING_ELEMS) * 2 +
                              kSmallWarps * 32 * DH * 4 + kSmallWarps * 32 * 2 * 4;
  static constexpr int TOTAL = GEMM > ATTN ? GEMM : ATTN;
};

// ---------------------------------------------------------------- the loop

struct SmallPhase {
  int kind;          // 0 GEMM, 1 attention
  SmallGemm g;
  AttnArgs a;
};

// Phase `idx` of Euler step k (per step: 3 action-encoder GEMMs, 5 phases per
// DiT block, norm_out + proj_out, 2 decoder GEMMs).
__device__ __forceinline__ void small_describe(const SmallPlan& P, int c, int k, int idx, SmallPhase& ph) {
  const int D = P.D, H = P.H, N = P.N, A = P.A, C = P.C, L = P.L;
  memset(&ph, 0, sizeof(ph));
  SmallGemm& g = ph.g;
  const float* ada_k = P.ada + (size_t)k * (L + 1) * 2 * D;
  g.rows = N;
  if (idx < 3) {
    g.rows = H;
    g.ldo = D;
    if (idx == 0) {          // a = x W1[c] + b1
      g.W = P.wa1t + (size_t)c * D * A; g.N = D; g.K = A; g.bias = P.ba1 + (size_t)c * D; g.epi = EPI_BF16;
      g.X = P.xb; g.ldx = A; g.out = P.abf;
    } else if (idx == 1) {   // z = swish(a W2[c][action half] + (phi(td) W2[c][timestep half] + b2))
      g.W = P.wa2at + (size_t)c * D * D; g.N = D; g.K = D; g.vec = P.tw2 + ((size_t)k * C + c) * D;
      g.epi = EPI_SWISH_VEC_BF16; g.X = P.abf; g.ldx = D; g.out = P.zbf;
    } else {                 // h[1..H] = z W3[c] + b3; h[0] = state features
      g.W = P.wa3t + (size_t)c * D * D; g.N = D; g.K = D; g.bias = P.ba3 + (size_t)c * D; g.epi = EPI_F32;
      g.X = P.zbf; g.ldx = D; g.out = P.h; g.out_row_off = 1; g.state_row = P.sfeat;
    }
    return;
  }
  const int j = idx - 3;
  if (j < 5 * L) {
    const int l = j / 5, part = j % 5;
    const SmallLayer& Ly = P.layers[l];
    const bool self = (l % 2) == 1;
    switch (part) {
      case 0: {              // AdaLN + Q (cross) or QKV (self)
        const int nq = self ? 3 * D : D;
        g.W = Ly.wq; g.N = nq; g.K = D; g.bias = Ly.bq; g.epi = EPI_BF16; g.x_mode = 1; g.ln_mode = 0;
        g.p0 = ada_k + (size_t)l * 2 * D; g.p1 = g.p0 + D; g.out = P.qkv; g.ldo = nq;
        break;
      }
      case 1: {              // attention
        ph.kind = 1;
        AttnArgs& a = ph.a;
        a.n_tok = N;
        a.num_heads = P.nh;
        a.num_items = P.nh;
        a.out = P.o;
        a.out_ld = D;
        a.scale_log2 = P.scale_log2;
        if (self) {
          a.q = P.qkv; a.q_ld = 3 * D; a.k = P.qkv + D; a.v = P.qkv + 2 * D; a.kv_ld = 3 * D;
          a.kv_head_stride = P.dh; a.kofs = nullptr;
        } else {
          a.q = P.qkv; a.q_ld = D; a.k = Ly.kv; a.v = Ly.kv + (size_t)P.nh * P.max_tok * P.dh; a.kv_ld = P.dh;
          a.kv_head_stride = P.max_tok * P.dh; a.kofs = P.vofs;
        }
        break;
      }
      case 2:                // h += O(attn) + b
        g.W = Ly.wo; g.N = D; g.K = D; g.bias = Ly.bo; g.epi = EPI_RESID_F32; g.X = P.o; g.ldx = D;
        g.out = P.h; g.ldo = D;
        break;
      case 3:                // f = GELU(LN3(h) W1^T + b1)
        g.W = Ly.wff1; g.N = P.F; g.K = D; g.bias = Ly.bff1; g.epi = EPI_GELU_BF16; g.x_mode = 1; g.ln_mode = 1;
        g.p0 = Ly.ln3g; g.p1 = Ly.ln3b; g.out = P.f; g.ldo = P.F;
        break;
      default:               // h += f W2^T + b2
        g.W = Ly.wff2; g.N = D; g.K = P.F; g.bias = Ly.bff2; g.epi = EPI_RESID_F32; g.X = P.f; g.ldx = P.F;
        g.out = P.h; g.ldo = D;
    }
    return;
  }
  const int t = j - 5 * L;
  g.rows = H;
  if (t == 0) {              // y = AdaLN_out(h[1..H]) W_out^T + b  (the state row is not decoded)
    g.W = P.proj_w; g.N = D; g.K = D; g.bias = P.proj_b; g.epi = EPI_BF16; g.x_mode = 1; g.ln_mode = 0;
    g.p0 = ada_k + (size_t)L * 2 * D; g.p1 = g.p0 + D; g.h_row_off = 1; g.out = P.ybf; g.ldo = D;
  } else if (t == 1) {       // r = ReLU(y W1[c] + b1)
    g.W = P.wd1t + (size_t)c * D * D; g.N = D; g.K = D; g.bias = P.bd1 + (size_t)c * D; g.epi = EPI_RELU_BF16;
    g.X = P.ybf; g.ldx = D; g.out = P.rbf; g.ldo = D;
  } else {                   // x += (1/K) (r W2[c] + b2); bf16 copy of x for the next step
    g.W = P.wd2t + (size_t)c * A * D; g.N = A; g.K = D; g.bias = P.bd2 + (size_t)c * A; g.epi = EPI_EULER;
    g.X = P.rbf; g.ldx = D; g.out = P.x; g.ldo = A; g.out2 = P.xb; g.alpha = 1.0f / (float)P.K;
  }
}

__device__ __forceinline__ int small_phase_workers(const SmallPhase& ph) {
  return ph.kind == 1 ? ph.a.num_heads : workers(gemm_units(ph.g));
}

__device__ __forceinline__ void small_prefetch(const SmallPhase& ph, const SmallPlan& P, uint8_t* smem,
                                               uint64_t* wbar) {
  if (ph.kind == 0) {
    small_prefetch_w(ph.g, smem, wbar);
    prefetch_gemm_weights(ph.g);
  } else if (ph.a.kofs != nullptr && threadIdx.x == 0 && (int)blockIdx.x < ph.a.num_heads) {
    // K and V of this CTA's head: contiguous rows of the head-major cache
    const uint32_t bytes = (uint32_t)P.vofs[1] * (uint32_t)P.dh * 2u;
    if (bytes > 0) {
      l2_prefetch(ph.a.k + (size_t)blockIdx.x * ph.a.kv_head_stride, bytes);
      l2_prefetch(ph.a.v + (size_t)blockIdx.x * ph.a.kv_head_stride, bytes);
    }
  }
}

__device__ __forceinline__ int small_category(const SmallPlan& P) {
  int c = 0;   // category of the single sample (an out-of-range id was routed to 0)
  for (int i = 0; i < P.C; ++i)
    if (P.seg[i] == 0 && P.seg[i + 1] == 1) c = i;
  return c;
}

// One thread per phase: the descriptor table of the whole loop.
__global__ void small_describe_kernel(const SmallPlan* __restrict__ plan) {
  const SmallPlan& P = *plan;
  pdl_wait();
  pdl_launch_dependents();
  const int per_step = 5 * P.L + 6;
  const int total = per_step * P.K;
  const int gp = blockIdx.x * blockDim.x + threadIdx.x;
  if (gp >= total) return;
  small_describe(P, small_category(P), gp / per_step, gp % per_step, P.phases[gp]);
}

// all threads: descriptor gp -> shared slot
__device__ __forceinline__ void small_load_phase(const SmallPlan& P, int gp, SmallPhase* dst) {
  static_assert(sizeof(SmallPhase) % 4 == 0, "descriptor copied as words");
  const uint32_t* src = reinterpret_cast<const uint32_t*>(P.phases + gp);
  uint32_t* d = reinterpret_cast<uint32_t*>(dst);
  for (int i = threadIdx.x; i < (int)(sizeof(SmallPhase) / 4); i += kSmallThreads) d[i] = src[i];
}

template <int DH>
__global__ void __launch_bounds__(kSmallThreads, 1) small_loop_kernel(const SmallPlan* __restrict__ plan) {
  extern __shared__ __align__(16) uint8_t smem[];
  // phase descriptors in shared memory: slot gp & 1 holds the current phase,
  // the other slot the next one
  __shared__ __align__(16) SmallPhase s_ph[2];
  __shared__ __align__(8) uint64_t s_wbar[2];
  const SmallPlan& P = *plan;
  const int per_step = 5 * P.L + 6;
  const int total = per_step * P.K;
  if (threadIdx.x == 0) {
    mbar_init(&s_wbar[0], 1);
    mbar_init(&s_wbar[1], 1);
    fence_mbar_init();
  }
  small_load_phase(P, 0, &s_ph[0]);
  __syncthreads();
  uint32_t wuse[2] = {0u, 0u};   // completed uses of each W slot's mbarrier (same in every thread)
  small_prefetch(s_ph[0], P, smem, s_wbar);
  if (threadIdx.x == 0)
    for (int la = 1; la < 3 && la < total; ++la)
      if (P.phases[la].kind == 0) prefetch_gemm_weights(P.phases[la].g);
  int prev_workers = 0;
  for (int gp = 0; gp < total; ++gp) {
    const SmallPhase& cur = s_ph[gp & 1];
    SmallPhase& nxt = s_ph[(gp + 1) & 1];
    const bool has_next = gp + 1 < total;
    if (has_next) small_load_phase(P, gp + 1, &nxt);
    __syncthreads();
    const int w = small_phase_workers(cur);
    bool ok = true;
    if ((int)blockIdx.x < w) {
      ok = small_wait(P, gp - 1, prev_workers);
      if (ok) {
        if (cur.kind == 0)
          small_gemm_phase(cur.g, P, smem, s_wbar, wuse);
        else
          small_attention_phase<DH>(cur.a, blockIdx.x, smem);
        small_arrive(P, gp);
      }
    }
    if (!ok) {
      cp_async_wait<0>();   // requested chunks land before the CTA exits
      const unsigned long long t0 = globaltimer_ns();
      for (int i = 0; i < 2; ++i)
        while (!mbar_try_wait(&s_wbar[i], wuse[i] & 1u) && globaltimer_ns() - t0 < 10000000ull) {
        }
      return;
    }
    if (has_next) small_prefetch(nxt, P, smem, s_wbar);
    // weights of the phase three ahead -> L2, so the shared-memory prefetch
    // issued at the end of the next-but-one phase finds them there
    if (threadIdx.x == 0 && gp + 3 < total && P.phases[gp + 3].kind == 0) prefetch_gemm_weights(P.phases[gp + 3].g);
    prev_workers = w;
    __syncthreads();   // every thread is done with s_ph[gp & 1] before it is rewritten
  }
}

}  // namespace gdit
