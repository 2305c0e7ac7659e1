// Persistent bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA, with the action head's epilogues fused in.
//
//   C[m, n] = sum_k A[m, k] * B[n, k]      (A: activations, B: weights, both K-major)
//
// Used for every dense contraction of the action head: the cross-attention
// K/V projection of the backbone features, the Q/QKV, O, FF1, FF2 and
// proj_out linears of the DiT blocks (Isaac-GR00T architecture page,
// "Transformer block structure"), and the CategorySpecificLinear layers of the
// state encoder, action encoder and action decoder ("Embodiment-specific
// projectors"), which run grouped: rows are sorted by embodiment and each
// group multiplies by its own category's weights.
//
// CTA = 10 warps: warp 0 issues TMA loads into a STAGES-deep shared-memory
// ring, warp 1 allocates TMEM and one thread issues tcgen05.mma (128 x BN x 16
// per instruction) into one of two TMEM accumulators, warps 2-9 drain the
// other accumulator through tcgen05.ld and run the epilogue: two warps per
// 32-lane TMEM quarter, taking alternate column chunks, so that on each SM
// sub-partition one epilogue warp computes while the other waits on memory.  Tiles are
// 128 x BN (BN in {32, 64, 128, 256}) with 64-wide K blocks in the 128-byte
// swizzled layout.  Split-K is deterministic: every split writes an f32
// partial, and the last split to finish (per-tile counter) sums the partials
// in split order and runs the epilogue.  Dense GEMMs with a plain output
// store through TMA: each epilogue warp stages 32 rows x 128 bytes in a
// 128-byte-swizzled shared buffer (conflict-free 16-byte stores) and one lane
// issues a bulk tensor store, or a bulk reduce-add (f32) for the residual
// adds, so the residual is never read back.
#pragma once

#include "ptx.cuh"

namespace gdit {

enum Epi : int {
  EPI_BF16 = 0,            // out(bf16) = acc + bias
  EPI_GELU_BF16 = 1,       // out(bf16) = gelu(acc + bias)           (FF1)
  EPI_RELU_BF16 = 2,       // out(bf16) = relu(acc + bias)           (CategorySpecificMLP layer 1)
  EPI_SWISH_VEC_BF16 = 3,  // out(bf16) = swish(acc + vec[g])        (action encoder W2)
  EPI_F32 = 4,             // out(f32)  = acc + bias
  EPI_RESID_F32 = 5,       // out(f32) += acc + bias                 (residual adds)
  EPI_EULER = 6,           // x = out + alpha * (acc + bias); out = x; out2(bf16) = x   (velocity -> Euler)
};

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kGemmThreads = 64 + kEpiThreads;
constexpr int kMaxGroups = 64;

struct GemmArgs {
  int M;                    // rows of A (dense) or row capacity (grouped)
  int N, K;
  const int* m_dev;         // dense: optional device row count (<= M)
  const int* m_begin_dev;   // dense with m_dev: optional first row (device): rows [*m_begin_dev, *m_dev)
  int num_groups;           // 0 = dense
  const int* seg;           // grouped: [num_groups + 1] sample offsets (device)
  int rows_per_sample;      // grouped: rows of A per sample
  int b_group_rows;         // grouped: rows of B per group (= N)
  int splits;               // split-K factor
  float* ws;                // split-K partials [splits][M][N]
  int* counters;            // split-K per-unit arrival counters (zero between launches)
  int epi;
  const float* bias;
  long long bias_gstride;   // bias of group g at bias + g * bias_gstride
  const float* vec;
  long long vec_gstride;
  void* out;
  long long ldo;
  __nv_bfloat16* out2;
  long long ldo2;
  float alpha;
  int in_group, in_skip, out_group, out_off;   // output row = (m / in_group) * out_group + m % in_group - in_skip + out_off
  int nblk;                 // > 0: columns blocked by nblk, block j at out + j * blk_stride
  long long blk_stride;
  int head_cols;            // > 0 (with nblk): inside a block, column c goes to sub-matrix c / head_cols,
  long long head_stride;    //   stored [rows][head_cols] at block + (c / head_cols) * head_stride

  int tma_out;              // 1: output through the TMA map (dense, one split, plain [M, N] layout)
  int out3d;                // with tma_out: the map is 3-D [N / 64][rows][64] (head-major K/V cache; bf16)
  unsigned* err;

};

template <int BN>
struct GemmCfg {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int STG_BYTES = kEpiWarps * 4096;   // per epilogue warp: one 32 x 128-byte staging box
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + STG_BYTES + 256;
  static constexpr uint32_t IDESC = idesc_bf16_f32(kBM, BN);
};

struct GemmSched {
  int units;          // output tiles (without the split factor)
  int nt;             // column tiles
  int mt;             // dense: row tiles
  int rows;           // dense: end of the valid rows
  int m_begin;        // dense: first row
  int uprefix[kMaxGroups + 1];
  int rstart[kMaxGroups];
  int rend[kMaxGroups];
};

struct TileInfo {
  int g, m0, m_end, n_idx, kb0, kb1, unit, split;   // n_idx: column tile index
};

__device__ __forceinline__ void gemm_decode(const GemmArgs& a, const GemmSched& s, int t, TileInfo& ti) {
  const int u = t / a.splits;
  ti.split = t - u * a.splits;
  ti.unit = u;
  int m_idx, n_idx;
  if (a.num_groups == 0) {
    constexpr int GM = 16;   // row-tile groups for L2 reuse of the B tiles
    const int group_size = GM * s.nt;
    const int gid = u / group_size;
    const int first_m = gid * GM;
    const int gm = min(s.mt - first_m, GM);
    const int r = u - gid * group_size;
    m_idx = first_m + r % gm;
    n_idx = r / gm;
    ti.g = 0;
    ti.m0 = s.m_begin + m_idx * kBM;
    ti.m_end = s.rows;
  } else {
    int g = 0;
    while (g + 1 < a.num_groups && s.uprefix[g + 1] <= u) ++g;
    const int r = u - s.uprefix[g];
    const int mt_g = (s.rend[g] - s.rstart[g] + kBM - 1) / kBM;
    m_idx = r % mt_g;
    n_idx = r / mt_g;
    ti.g = g;
    ti.m0 = s.rstart[g] + m_idx * kBM;
    ti.m_end = s.rend[g];
  }
  ti.n_idx = n_idx;
  const int nkb = (a.K + kBK - 1) / kBK;
  ti.kb0 = (int)(((long long)ti.split * nkb) / a.splits);
  ti.kb1 = (int)(((long long)(ti.split + 1) * nkb) / a.splits);
}

template <int BN>
__device__ __forceinline__ void gemm_build_sched(const GemmArgs& a, GemmSched& sched) {
  sched.nt = (a.N + BN - 1) / BN;
  if (a.num_groups == 0) {
    int rows = a.M;
    if (a.m_dev != nullptr) rows = min(rows, *a.m_dev);
    rows = max(rows, 0);
    const int begin = (a.m_dev != nullptr && a.m_begin_dev != nullptr) ? min(max(*a.m_begin_dev, 0), rows) : 0;
    sched.rows = rows;
    sched.m_begin = begin;
    sched.mt = (rows - begin + kBM - 1) / kBM;
    sched.units = sched.mt * sched.nt;
  } else {
    int u = 0;
    for (int g = 0; g < a.num_groups; ++g) {
      const int rs = a.seg[g] * a.rows_per_sample;
      const int re = a.seg[g + 1] * a.rows_per_sample;
      sched.rstart[g] = rs;
      sched.rend[g] = re;
      sched.uprefix[g] = u;
      u += ((re - rs + kBM - 1) / kBM) * sched.nt;
    }
    sched.uprefix[a.num_groups] = u;
    sched.units = u;
  }
}

// erf by approximation 7.1.28 of Abramowitz & Stegun, Handbook of
// Mathematical Functions (1964): erf(z) = 1 - 1 / (1 + a1 z + ... + a6 z^6)^16
// for z >= 0, |error| <= 3e-7, far below bf16 resolution.  One reciprocal and
// no exponential (one special-function op per element instead of two).  For
// z >= 4 erf(z) rounds to 1 in fp32; clamping there keeps the 16th power finite.
__device__ __forceinline__ float erf_as(float x) {
  const float z = fminf(fabsf(x), 4.0f);
  float p = fmaf(4.30638e-5f, z, 2.765672e-4f);
  p = fmaf(p, z, 1.520143e-4f);
  p = fmaf(p, z, 9.2705272e-3f);
  p = fmaf(p, z, 4.22820123e-2f);
  p = fmaf(p, z, 7.05230784e-2f);
  p = fmaf(p, z, 1.0f);
  p *= p;   // p^2
  p *= p;   // p^4
  p *= p;   // p^8
  p *= p;   // p^16
  return copysignf(1.0f - __fdividef(1.0f, p), x);
}

// exact (erf) GELU: x * Phi(x)
__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.0f + erf_as(x * 0.70710678118654752f)); }

// Packed pairs of f32 (sm_100 f32x2 arithmetic: one instruction for both
// lanes, each rounded to nearest like its scalar form).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_splat(float c) { return f2_pack(c, c); }

// gelu_erf of two values at once: the same operations in the same order as
// gelu_erf (so the same results, bit for bit), the multiply-adds and
// multiplies as f32x2 instructions, about half the instructions per value.
__device__ __forceinline__ void gelu_erf2(float& x0, float& x1) {
  const uint64_t x = f2_pack(x0, x1);
  float u0, u1;
  f2_unpack(f2_mul(x, f2_splat(0.70710678118654752f)), u0, u1);
  const uint64_t z = f2_pack(fminf(fabsf(u0), 4.0f), fminf(fabsf(u1), 4.0f));
  uint64_t p = f2_fma(f2_splat(4.30638e-5f), z, f2_splat(2.765672e-4f));
  p = f2_fma(p, z, f2_splat(1.520143e-4f));
  p = f2_fma(p, z, f2_splat(9.2705272e-3f));
  p = f2_fma(p, z, f2_splat(4.22820123e-2f));
  p = f2_fma(p, z, f2_splat(7.05230784e-2f));
  p = f2_fma(p, z, f2_splat(1.0f));
  p = f2_mul(p, p);
  p = f2_mul(p, p);
  p = f2_mul(p, p);
  p = f2_mul(p, p);
  float p0, p1;
  f2_unpack(p, p0, p1);
  const float e0 = copysignf(1.0f - __fdividef(1.0f, p0), u0);
  const float e1 = copysignf(1.0f - __fdividef(1.0f, p1), u1);
  const uint64_t r = f2_mul(f2_mul(f2_splat(0.5f), x), f2_add(f2_splat(1.0f), f2_pack(e0, e1)));
  f2_unpack(r, x0, x1);
}
__device__ __forceinline__ float swish_f(float x) { return x / (1.0f + __expf(-x)); }

// Epilogue of 32 consecutive columns [n, n + 32) of row m (group g).
__device__ __forceinline__ void gemm_epilogue32(const GemmArgs& a, int g, int m, int n, float (&v)[32]) {
  const int gi = m / a.in_group;
  const int ri = m - gi * a.in_group;
  if (ri < a.in_skip) return;
  const long long orow = (long long)gi * a.out_group + (ri - a.in_skip) + a.out_off;
  long long col = n;
  long long blk_off = 0;
  long long ldo = a.ldo;
  if (a.nblk > 0) {
    const int blk = n / a.nblk;
    col = n - (long long)blk * a.nblk;
    blk_off = (long long)blk * a.blk_stride;
    if (a.head_cols > 0) {   // head-major: 32 columns never straddle a sub-matrix (head_cols % 32 == 0)
      const long long hh = col / a.head_cols;
      blk_off += hh * a.head_stride;
      col -= hh * a.head_cols;
      ldo = a.head_cols;
    }
  }
  const int epi = a.epi;
  if (epi == EPI_SWISH_VEC_BF16) {
    const float4* vp = reinterpret_cast<const float4*>(a.vec + (long long)g * a.vec_gstride + n);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 b = vp[j];
      v[4 * j + 0] = swish_f(v[4 * j + 0] + b.x);
      v[4 * j + 1] = swish_f(v[4 * j + 1] + b.y);
      v[4 * j + 2] = swish_f(v[4 * j + 2] + b.z);
      v[4 * j + 3] = swish_f(v[4 * j + 3] + b.w);
    }
  } else if (a.bias != nullptr) {
    const float4* bp = reinterpret_cast<const float4*>(a.bias + (long long)g * a.bias_gstride + n);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 b = bp[j];
      v[4 * j + 0] += b.x;
      v[4 * j + 1] += b.y;
      v[4 * j + 2] += b.z;
      v[4 * j + 3] += b.w;
    }
  }
  if (epi == EPI_GELU_BF16) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = gelu_erf(v[j]);
  } else if (epi == EPI_RELU_BF16) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.0f);
  }
  if (epi <= EPI_SWISH_VEC_BF16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + blk_off + orow * ldo + col;
    uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
      w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
      w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
      w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
      o4[j] = w;
    }
    return;
  }
  float* o = reinterpret_cast<float*>(a.out) + blk_off + orow * ldo + col;
  float4* o4 = reinterpret_cast<float4*>(o);
  if (epi == EPI_F32) {
#pragma unroll
    for (int j = 0; j < 8; ++j) o4[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  } else if (epi == EPI_RESID_F32) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float4 r = o4[j];
      r.x += v[4 * j];
      r.y += v[4 * j + 1];
      r.z += v[4 * j + 2];
      r.w += v[4 * j + 3];
      o4[j] = r;
    }
  } else {  // EPI_EULER
    uint4* x2 = reinterpret_cast<uint4*>(a.out2 + orow * a.ldo2 + col);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float4 r = o4[j];
      r.x += a.alpha * v[4 * j];
      r.y += a.alpha * v[4 * j + 1];
      r.z += a.alpha * v[4 * j + 2];
      r.w += a.alpha * v[4 * j + 3];
      o4[j] = r;
      v[4 * j] = r.x;
      v[4 * j + 1] = r.y;
      v[4 * j + 2] = r.z;
      v[4 * j + 3] = r.w;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
      w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
      w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
      w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
      x2[j] = w;
    }
  }
}

// TMA-store epilogue of one accumulator tile on one epilogue warp: TMEM lanes
// of this warp's quarter (taddr), i.e. output rows [ym, ym + 32), column
// chunks half, half + 2, ... of [n0, n0 + BN); f32 boxes hold 32 columns,
// bf16 boxes 64.  Each chunk is staged in one of this warp's NBOX 4 KB boxes
// (128-byte swizzle, conflict-free 16-byte stores; `seq` counts the warp's
// chunks, so consecutive chunks alternate boxes) and one lane issues a bulk
// tensor store, or a bulk reduce-add for the residual adds.  Both TMEM loads
// of a 64-column chunk are issued before one wait.
template <int BN, int NBOX>
__device__ __forceinline__ void gemm_epilogue_tma(const GemmArgs& a, const CUtensorMap* tmO, uint8_t* boxes,
                                                  uint32_t taddr, int n0, int ym, int half, int lane, int& seq) {
  const bool f32out = a.epi == EPI_RESID_F32 || a.epi == EPI_F32;
  const int ccols = f32out ? 32 : 64;
  const int rs = lane & 7;   // swizzle phase of this thread's row
#pragma unroll 1
  for (int cs = half; cs < BN / ccols; cs += 2, ++seq) {
    const int n = n0 + cs * ccols;
    uint8_t* box = boxes + (seq % NBOX) * 4096;
    float v[64];
    {
      uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
      uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
      tmem_ld32(taddr + cs * ccols, lo);
      if (!f32out) tmem_ld32(taddr + cs * ccols + 32, hi);
      tmem_ld_wait();
    }
    // the store NBOX chunks ago has finished reading this box
    if (lane == 0) bulk_wait_read<NBOX - 1>();
    __syncwarp();
    if (f32out) {
      if (a.bias != nullptr) {
        const float4* bp = reinterpret_cast<const float4*>(a.bias + n);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 b = __ldg(bp + j);
          f2_unpack(f2_add(f2_pack(v[4 * j], v[4 * j + 1]), f2_pack(b.x, b.y)), v[4 * j], v[4 * j + 1]);
          f2_unpack(f2_add(f2_pack(v[4 * j + 2], v[4 * j + 3]), f2_pack(b.z, b.w)), v[4 * j + 2], v[4 * j + 3]);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(box + lane * 128 + ((j ^ rs) << 4)) =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
      if (a.bias != nullptr) {
        const float4* bp = reinterpret_cast<const float4*>(a.bias + n);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float4 b = __ldg(bp + j);
          f2_unpack(f2_add(f2_pack(v[4 * j], v[4 * j + 1]), f2_pack(b.x, b.y)), v[4 * j], v[4 * j + 1]);
          f2_unpack(f2_add(f2_pack(v[4 * j + 2], v[4 * j + 3]), f2_pack(b.z, b.w)), v[4 * j + 2], v[4 * j + 3]);
        }
      }
      if (a.epi == EPI_GELU_BF16) {
#pragma unroll
        for (int j = 0; j < 64; j += 2) gelu_erf2(v[j], v[j + 1]);
      } else if (a.epi == EPI_RELU_BF16) {
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = fmaxf(v[j], 0.0f);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
        w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
        w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
        w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
        *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ rs) << 4)) = w;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (a.epi == EPI_RESID_F32)
        tma_reduce_add_2d(tmO, box, n, ym);
      else if (a.out3d)
        tma_store_3d(tmO, box, 0, ym, n >> 6);   // 64 columns: one head block
      else
        tma_store_2d(tmO, box, n, ym);
      bulk_commit();
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const GemmArgs a) {
  using Cfg = GemmCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  __shared__ GemmSched sched;
  __shared__ uint32_t tmem_holder;
  __shared__ int s_last;
  __shared__ volatile int s_abort;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* stg = smem + STAGES * Cfg::STAGE_BYTES;   // 1024-aligned staging boxes
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + Cfg::STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiThreads);
    }
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (a.tma_out) tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  // The schedule of a dense GEMM with a fixed row count depends on nothing an
  // earlier kernel writes, and neither do the weights (operand B): their first
  // stages are requested before waiting for the previous kernel, so weight
  // streaming overlaps its tail.  A, seg, m_dev and residuals are read after.
  const bool early = a.num_groups == 0 && a.m_dev == nullptr;
  int pre = 0;   // stages whose B tile was issued before the wait (first tile only)
  if (threadIdx.x == 0) {
    if (early) gemm_build_sched<BN>(a, sched);
    if (early && (int)blockIdx.x < sched.units * a.splits) {
      TileInfo ti;
      gemm_decode(a, sched, blockIdx.x, ti);
      pre = min(ti.kb1 - ti.kb0, STAGES);
      const int brow = ti.g * a.b_group_rows + ti.n_idx * BN;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], Cfg::STAGE_BYTES);
        tma_load_2d(sB + i * Cfg::B_BYTES, &tmB, &full[i], (ti.kb0 + i) * kBK, brow);
      }
    }
  }
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0 && !early) gemm_build_sched<BN>(a, sched);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  const int total = sched.units * a.splits;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        TileInfo ti;
        gemm_decode(a, sched, t, ti);
        const int brow = ti.g * a.b_group_rows + ti.n_idx * BN;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (pre > 0) {
            // stage armed and its B tile requested before the dependency wait
            tma_load_2d(sA + stage * Cfg::A_BYTES, &tmA, &full[stage], kb * kBK, ti.m0);
            --pre;
          } else {
            if (!mbar_wait(&empty[stage], phase ^ 1u, a.err)) { ok = false; s_abort = 1; break; }
            if (s_abort) { ok = false; break; }
            mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
            tma_load_2d(sA + stage * Cfg::A_BYTES, &tmA, &full[stage], kb * kBK, ti.m0);
            tma_load_2d(sB + stage * Cfg::B_BYTES, &tmB, &full[stage], kb * kBK, brow);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (ok) {
        // Producer tail: wait until the MMA warp has released every stage, so
        // no tcgen05.commit arrival is still pending when the CTA exits.
        for (int i = 0; i < STAGES; ++i) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, a.err)) break;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      } else {
        // Let the loads already in flight land before the CTA can exit.
        const unsigned long long t0 = globaltimer_ns();
        for (int i = 0; i < min(issued, STAGES); ++i) {
          if (--stage < 0) { stage = STAGES - 1; phase ^= 1u; }
          while (!mbar_try_wait(&full[stage], phase) && globaltimer_ns() - t0 < 10000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        TileInfo ti;
        gemm_decode(a, sched, t, ti);
        const int buf = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[buf], aphase ^ 1u, a.err)) { s_abort = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * BN;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, a.err) || s_abort) { ok = false; s_abort = 1; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            umma_bf16(d, smem_desc_sw128(a_addr + k * 32), smem_desc_sw128(b_addr + k * 32), Cfg::IDESC,
                      (kb > ti.kb0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        umma_commit(&tfull[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;   // column chunks half, half + 2, ... of the tile
    const int row = q * 32 + lane;
    int it = 0;
    int eseq = 0;   // TMA-store chunks of this warp
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      TileInfo ti;
      gemm_decode(a, sched, t, ti);
      const int buf = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      int ready = 0;
      if (lane == 0) ready = mbar_wait(&tfull[buf], aphase, a.err) && !s_abort;
      ready = __shfl_sync(0xffffffffu, ready, 0);   // keep the warp converged for tcgen05.ld
      if (!ready) { s_abort = 1; break; }
      tc_fence_after();
      const int m = ti.m0 + row;
      const bool row_ok = m < ti.m_end;
      const int n0 = ti.n_idx * BN;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
      if (a.tma_out) {
        // rows [m0 + 32q, +32) of the tile
        gemm_epilogue_tma<BN, 1>(a, &tmO, stg + (warp - 2) * 4096, taddr, n0, ti.m0 + q * 32, half, lane, eseq);
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
      } else if (a.splits == 1) {
#pragma unroll 1
        for (int c = half; c < BN / 32; c += 2) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          const int n = n0 + c * 32;
          if (row_ok && n < a.N) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            gemm_epilogue32(a, ti.g, m, n, v);
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
      } else {
        // write this split's partial, then the last split reduces in split order
        float* wsp = a.ws + ((long long)ti.split * a.M + m) * a.N;
#pragma unroll 1
        for (int c = half; c < BN / 32; c += 2) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          const int n = n0 + c * 32;
          if (row_ok && n < a.N) {
            float4* w4 = reinterpret_cast<float4*>(wsp + n);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              w4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                  __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
        __threadfence();
        named_bar_sync(1, kEpiThreads);
        if (threadIdx.x == 64) {
          const int old = atomicAdd(&a.counters[ti.unit], 1);
          s_last = (old == a.splits - 1);
          if (s_last) a.counters[ti.unit] = 0;
        }
        named_bar_sync(1, kEpiThreads);
        if (s_last) {
          __threadfence();
          if (row_ok) {
#pragma unroll 1
            for (int c = half; c < BN / 32; c += 2) {
              const int n = n0 + c * 32;
              if (n >= a.N) break;
              float v[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = 0.0f;
              for (int s = 0; s < a.splits; ++s) {
                const float4* p4 = reinterpret_cast<const float4*>(a.ws + ((long long)s * a.M + m) * a.N + n);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float4 x = __ldcg(p4 + j);
                  v[4 * j] += x.x;
                  v[4 * j + 1] += x.y;
                  v[4 * j + 2] += x.z;
                  v[4 * j + 3] += x.w;
                }
              }
              gemm_epilogue32(a, ti.g, m, n, v);
            }
          }
        }
        named_bar_sync(1, kEpiThreads);   // s_last is reused by the next tile
      }
    }
    if (a.tma_out && lane == 0) bulk_wait<0>();   // stores complete before the CTA exits
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ====================================================================== CTA-pair GEMM
//
// Dense GEMMs with a plain TMA-store output (the DiT linears at large batch)
// run on CTA pairs: a cluster of two CTAs on two SMs owns a 256 x BN output
// tile.  Each CTA loads its 128 rows of A and its BN/2 rows of B (weights)
// into its own shared memory; one thread of the even CTA issues
// tcgen05.mma.cta_group::2 (256 x BN x 16), which reads both CTAs' operands
// and leaves each CTA's 128 accumulator rows in that CTA's TMEM.  Per SM and
// k-block that is 16 KB of A and BN/2 x 128 bytes of B from L2, a third less
// than the 128 x BN tile of one CTA for the same tensor work; the 1-CTA tile
// is bound by that L2-to-shared-memory traffic.
//
// Protocol: the stage barriers `full` live in the even CTA (both CTAs' TMA
// loads count their bytes there); `empty` and `tfull` live in both CTAs and
// the MMA thread's commits arrive on both; `tempty` lives in the even CTA and
// counts one arrival per epilogue warp of both CTAs.  Both CTAs walk the same
// tile sequence.  Every wait is bounded; both CTAs always reach the final
// cluster barrier, after which TMEM is released.

constexpr int kPairBM = 256;

template <int BN>
struct GemmPairCfg {
  static constexpr int A_BYTES = 128 * kBK * 2;
  static constexpr int B_BYTES = (BN / 2) * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;              // per CTA
  static constexpr int NBOX = 2;                                     // staging boxes per epilogue warp
  static constexpr int STG_BYTES = kEpiWarps * NBOX * 4096;
  static constexpr int STAGES = (227 * 1024 - 1024 - STG_BYTES - 256) / STAGE_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + STG_BYTES + 256;
  static constexpr uint32_t IDESC = idesc_bf16_f32(kPairBM, BN);
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Tile t of a pair GEMM: 256-row block m_idx, column tile n_idx (row blocks
// grouped by 8 so that consecutive tiles reuse the same weight columns in L2).
__device__ __forceinline__ void gemm_pair_decode(int t, int mt, int nt, int& m0, int& n_idx) {
  constexpr int GM = 8;
  const int group_size = GM * nt;
  const int gid = t / group_size;
  const int first_m = gid * GM;
  const int gm = min(mt - first_m, GM);
  const int r = t - gid * group_size;
  m0 = (first_m + r % gm) * kPairBM;
  n_idx = r / gm;
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO, const GemmArgs a) {
  using Cfg = GemmPairCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int s_abort;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::A_BYTES;
  uint8_t* stg = smem + STAGES * Cfg::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + Cfg::STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);
    }
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  // both CTAs' barriers exist before either CTA signals the other's
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  const uint32_t full_l = mapa_shared(&full[0], 0);       // the even CTA's stage barriers
  const uint32_t tempty_l = mapa_shared(&tempty[0], 0);   // the even CTA's accumulator-free barriers

  int mt = (a.M + kPairBM - 1) / kPairBM;
  const int nt = (a.N + BN - 1) / BN;
  int total = mt * nt;
  const int cid = blockIdx.x >> 1;
  const int ncl = gridDim.x >> 1;
  const int nkb = (a.K + kBK - 1) / kBK;

  // The weights depend on no earlier kernel: the first tile's B stages are
  // requested before the dependency wait (with host-side rows only: a
  // device-side row range is known after it).
  int pre = 0;
  if (warp == 0 && lane == 0 && cid < total && a.m_dev == nullptr) {
    int m0, n_idx;
    gemm_pair_decode(cid, mt, nt, m0, n_idx);
    pre = min(nkb, STAGES);
    const int brow = n_idx * BN + (int)rank * (BN / 2);
    for (int i = 0; i < pre; ++i) {
      if (leader) mbar_arrive_expect_tx(&full[i], 2 * Cfg::STAGE_BYTES);
      tma_load_2d_pair(sB + i * Cfg::B_BYTES, &tmB, full_l + 8u * i, i * kBK, brow);
    }
  }
  pdl_wait();
  pdl_launch_dependents();
  __syncthreads();
  // rows [mb, me): all M, or the device-side range an earlier kernel wrote
  int mb = 0;
  if (a.m_dev != nullptr) {
    const int me = min(__ldcg(a.m_dev), a.M);
    mb = a.m_begin_dev != nullptr ? max(__ldcg(a.m_begin_dev), 0) : 0;
    mt = me > mb ? (me - mb + kPairBM - 1) / kPairBM : 0;
    total = mt * nt;
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = cid; t < total && ok; t += ncl) {
        int m0, n_idx;
        gemm_pair_decode(t, mt, nt, m0, n_idx);
        m0 += mb;
        const int arow = m0 + (int)rank * 128;
        const int brow = n_idx * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < nkb; ++kb) {
          if (pre > 0) {
            tma_load_2d_pair(sA + stage * Cfg::A_BYTES, &tmA, full_l + 8u * stage, kb * kBK, arow);
            --pre;
          } else {
            if (!mbar_wait(&empty[stage], phase ^ 1u, a.err)) { ok = false; s_abort = 1; break; }
            if (s_abort) { ok = false; break; }
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * Cfg::STAGE_BYTES);
            tma_load_2d_pair(sA + stage * Cfg::A_BYTES, &tmA, full_l + 8u * stage, kb * kBK, arow);
            tma_load_2d_pair(sB + stage * Cfg::B_BYTES, &tmB, full_l + 8u * stage, kb * kBK, brow);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Tail: every stage released by the MMA commits (which arrive on this
      // CTA's empty barriers), so none is pending when the CTA exits.
      const unsigned long long t0 = globaltimer_ns();
      for (int i = 0; i < min(issued, STAGES); ++i) {
        while (!mbar_try_wait(&empty[stage], phase ^ 1u) && globaltimer_ns() - t0 < 10000000ull) {
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = cid; t < total && ok; t += ncl, ++it) {
        const int buf = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[buf], aphase ^ 1u, a.err)) { s_abort = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * BN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, a.err) || s_abort) { ok = false; s_abort = 1; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16_pair(d, smem_desc_sw128(a_addr + k * 32), smem_desc_sw128(b_addr + k * 32), Cfg::IDESC,
                           (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        umma_commit_pair(&tfull[buf], 0x3);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9, both CTAs)
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    int it = 0;
    int eseq = 0;   // TMA-store chunks of this warp
    for (int t = cid; t < total; t += ncl, ++it) {
      int m0, n_idx;
      gemm_pair_decode(t, mt, nt, m0, n_idx);
      m0 += mb;
      const int buf = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      int ready = 0;
      if (lane == 0) ready = mbar_wait(&tfull[buf], aphase, a.err) && !s_abort;
      ready = __shfl_sync(0xffffffffu, ready, 0);
      if (!ready) { s_abort = 1; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
      gemm_epilogue_tma<BN, Cfg::NBOX>(a, &tmO, stg + (warp - 2) * Cfg::NBOX * 4096, taddr, n_idx * BN,
                                       m0 + (int)rank * 128 + q * 32, half, lane, eseq);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_l + 8u * buf);
    }
    if (lane == 0) bulk_wait<0>();   // stores complete before the CTA exits
  }
  __syncthreads();
  // neither CTA leaves while the other may still read its shared memory or
  // signal its barriers
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace gdit
