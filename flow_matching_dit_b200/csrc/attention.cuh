// Multi-head attention of the action tokens ("Transformer block structure"
// and "AlternateVLDiT variant", Isaac-GR00T architecture page):
//   cross layers (even): the N = H + 1 state/action tokens of a sample attend to
//     that sample's valid backbone tokens, whose K/V were projected once per call;
//   self layers (odd): the N tokens attend to each other (no mask).
// out_h = softmax(q_h k_h^T / sqrt(head_dim)) v_h per head, heads concatenated;
// a sample with no key gets a zero output.
//
// A warp streams 16-key chunks of K and V through a 3-deep cp.async ring in
// shared memory and keeps an online (base-2) softmax.  Scores and P*V use bf16
// mma.sync m16n8k16 with f32 accumulation: the op is bound by the K/V reads
// (about 17 FLOP per byte at N = 17), which this path keeps up with; queries
// are padded to 16-row tiles.  Two schedules share that routine:
//   attention_split_kernel: one CTA per (sample, head), the 4 warps split the
//     keys (flash-decoding inside the CTA) and combine through shared memory;
//     for few samples with long key lists.
//   attention_warp_kernel: every warp owns one (sample, head) and all its keys;
//     for many samples, and for self-attention (N keys).
#pragma once

#include "ptx.cuh"

namespace gdit {

constexpr int kAttnThreads = 128;
constexpr bool kKvEvictFirst = true;   // L2 priority of the streamed cross K/V (see attn_stream_chunks)

struct AttnArgs {
  const __nv_bfloat16* q;
  long long q_ld;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  long long kv_ld;          // row stride of K and V
  long long kv_head_stride; // offset between heads of K (and of V)
  const int* kspan;     // cross: keys of sample b are rows [kspan[2b], kspan[2b+1]); nullptr: self (rows of q's sample)
  int n_tok;            // queries (tokens) per sample
  int num_heads;
  int num_items;        // samples * heads
  __nv_bfloat16* out;
  long long out_ld;
  float scale_log2;     // log2(e) / sqrt(head_dim)
  const uint8_t* kflag; // cross: image flag of each packed key (used when ksel >= 0)
  int ksel;             // -1: every key; 0: keys with flag 0 (text); 1: flag 1 (image)
  long long kv_rows;    // cross: rows of a head's block of the K/V cache (the key spans must lie inside)
  unsigned* status;     // range-checked builds: where a key span outside the block is recorded
};

// MT: 16-row query tiles (queries padded to 16 * MT); DH: head dim (32 or 64).
// Shared-memory rows hold DH + 8 bf16 so fragment loads are bank-conflict free.
template <int MT, int DH, int RING_ = 3>
struct AttnSmem {
  static constexpr int ROW = DH + 8;
  static constexpr int Q_ELEMS = MT * 16 * ROW;
  static constexpr int CHUNK_ELEMS = 16 * ROW;                    // 16 keys x DH dims (padded)
  static constexpr int RING = RING_;                              // chunks in flight per warp
  static constexpr int RING_ELEMS = RING * 2 * CHUNK_ELEMS;       // (K, V) per slot
  // split schedule: one Q tile, 4 rings, per-warp partials
  static constexpr int SPLIT_O_BYTES = 4 * MT * 16 * DH * 4;
  static constexpr int SPLIT_ML_BYTES = 4 * MT * 16 * 2 * 4;
  static constexpr int SPLIT_TOTAL = (Q_ELEMS + 4 * RING_ELEMS) * 2 + SPLIT_O_BYTES + SPLIT_ML_BYTES;
  // warp schedule: a Q tile and a ring per warp
  static constexpr int WARP_TOTAL = 4 * (Q_ELEMS + RING_ELEMS) * 2;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t n = valid ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(n) : "memory");
}
// Same, with an L2 eviction-priority hint (a createpolicy value).
__device__ __forceinline__ void cp_async16_hint(void* smem, const void* gmem, bool valid, uint64_t policy) {
  const uint32_t n = valid ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(n), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// 2^x by the PTX ex2.approx instruction (one special-function op; relative
// error of a few ulp, far below bf16 resolution).  Arguments here are <= 0
// (scores minus their running maximum); -inf gives 0.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void attn_key_range(const AttnArgs& a, int b, int& k_begin, int& n_keys) {
  if (a.kspan != nullptr) {
    k_begin = a.kspan[2 * b];
    n_keys = a.kspan[2 * b + 1] - k_begin;
    if constexpr (GDIT_CHECKED) {   // a span outside the block is not followed: no keys
      if (!checked_in_range(n_keys, 0, a.kv_rows + 1, a.status) ||
          !checked_in_range(k_begin, 0, a.kv_rows - n_keys + 1, a.status)) {
        k_begin = 0;
        n_keys = 0;
      }
    }
  } else {
    k_begin = b * a.n_tok;
    n_keys = a.n_tok;
  }
}

// Q rows of (b, h) -> shared tile [MT*16][DH+8]; rows >= n_tok are zero.
// Thread t of `nthreads` cooperating threads copies every nthreads-th piece.
template <int MT, int DH>
__device__ __forceinline__ void attn_load_q(const AttnArgs& a, int b, int h, __nv_bfloat16* sQ, int t, int nthreads) {
  constexpr int ROW = DH + 8;
  constexpr int PIECES = DH / 8;   // 16-byte pieces per row
  const __nv_bfloat16* qbase = a.q + (long long)b * a.n_tok * a.q_ld + h * DH;
  for (int i = t; i < MT * 16 * PIECES; i += nthreads) {
    const int r = i / PIECES, c = (i % PIECES) * 8;
    uint4 val = make_uint4(0, 0, 0, 0);
    // L2 load: queries are rewritten every layer by other CTAs of a persistent loop
    if (r < a.n_tok) val = __ldcg(reinterpret_cast<const uint4*>(qbase + (long long)r * a.q_ld + c));
    *reinterpret_cast<uint4*>(sQ + r * ROW + c) = val;
  }
}

template <int MT, int DH>
__device__ __forceinline__ void attn_init(float (&o)[MT][DH / 8][4], float (&mrow)[MT][2], float (&lrow)[MT][2]) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int nd = 0; nd < DH / 8; ++nd)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[mt][nd][j] = 0.0f;
    mrow[mt][0] = mrow[mt][1] = -INFINITY;
    lrow[mt][0] = lrow[mt][1] = 0.0f;
  }
}

// One 16-key chunk (keys key0 .. key0 + 15 of the list [k_begin, k_begin +
// n_keys)) folded into (o, mrow, lrow) with an online softmax (base 2).  The
// chunk's K and V rows sit in shared memory: kaddr(r, c) / vaddr(r, c) give
// the address of 16-byte column chunk c of row r (0..15) of the chunk.  Keys
// past n_keys (and, with a.ksel >= 0, keys of the other kind) get -inf; their
// V rows must hold finite values.
template <int MT, int DH, typename KAddr, typename VAddr>
__device__ __forceinline__ void attn_fold_chunk(const AttnArgs& a, int key0, int k_begin, int n_keys,
                                                const __nv_bfloat16* sQ, KAddr kaddr, VAddr vaddr,
                                                float (&o)[MT][DH / 8][4], float (&mrow)[MT][2],
                                                float (&lrow)[MT][2]) {
  constexpr int ROW = DH + 8;
  const int lane = threadIdx.x & 31;
  const int tig = lane & 3;    // thread in group
  // the keys of this lane's score columns that the layer keeps (bit nt * 2 + j)
  uint32_t keep = 0xFu;
  if (a.ksel >= 0) {
    keep = 0u;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int key = key0 + nt * 8 + tig * 2 + j;
        if (key < n_keys && (int)__ldg(a.kflag + k_begin + key) == a.ksel) keep |= 1u << (nt * 2 + j);
      }
  }

  // S = Q K^T for 16 keys (two n-tiles of 8).  Even and odd k-steps go to
  // separate accumulators: a dependent chain of mma.sync is bound by its
  // latency, and this halves the chain.
  float s[MT][2][4], s1[MT][2][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s[mt][nt][j] = 0.0f;
        s1[mt][nt][j] = 0.0f;
      }
#pragma unroll
  for (int ks = 0; ks < DH / 16; ++ks) {
    // K fragments of both 8-key tiles in one ldmatrix: lanes 0-7 keys 0-7
    // (k 0-7), 8-15 keys 0-7 (k 8-15), 16-23 keys 8-15 (k 0-7), 24-31 keys 8-15 (k 8-15)
    uint32_t kb[2][2];
    ldmatrix_x4(kb[0][0], kb[0][1], kb[1][0], kb[1][1],
                kaddr((lane & 7) + ((lane >> 4) << 3), ks * 2 + ((lane >> 3) & 1)));
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      // Q fragments: lane supplies row (lane & 15) of the tile, k half (lane >> 4)
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(a0, a1, a2, a3, sQ + (mt * 16 + (lane & 15)) * ROW + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
        mma_bf16_16816((ks & 1) ? s1[mt][nt] : s[mt][nt], a0, a1, a2, a3, kb[nt][0], kb[nt][1]);
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[mt][nt][j] += s1[mt][nt][j];

  // online softmax (base 2); masked keys get -inf.  Row groups of 8 with no
  // query (past n_tok: zero Q rows, never stored) are skipped.
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {   // hr 0: row g, hr 1: row g + 8
      if (mt * 16 + hr * 8 >= a.n_tok) continue;
      float x[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int key = key0 + nt * 8 + tig * 2 + j;
          x[nt * 2 + j] = (key < n_keys && ((keep >> (nt * 2 + j)) & 1u)) ? s[mt][nt][hr * 2 + j] * a.scale_log2
                                                                           : -INFINITY;
        }
      float cm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
      const float m_old = mrow[mt][hr];
      const float m_new = fmaxf(m_old, cm);
      const float alpha = (m_new == -INFINITY) ? 1.0f : ex2_approx(m_old - m_new);
      float psum = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = (m_new == -INFINITY) ? 0.0f : ex2_approx(x[j] - m_new);
        x[j] = p;
        psum += p;
      }
      mrow[mt][hr] = m_new;
      lrow[mt][hr] = lrow[mt][hr] * alpha + psum;
#pragma unroll
      for (int nd = 0; nd < DH / 8; ++nd) {
        o[mt][nd][hr * 2 + 0] *= alpha;
        o[mt][nd][hr * 2 + 1] *= alpha;
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        s[mt][nt][hr * 2 + 0] = x[nt * 2 + 0];
        s[mt][nt][hr * 2 + 1] = x[nt * 2 + 1];
      }
    }
  }

  // O += P V : P (16 x 16 keys) from the score accumulators, V via ldmatrix.trans
#pragma unroll
  for (int nd2 = 0; nd2 < DH / 16; ++nd2) {   // pairs of 8-wide dim tiles
    uint32_t vb0, vb1, vb2, vb3;
    const int r = lane & 7;
    const int mtx = lane >> 3;          // matrix 0..3: (keys 0-7 | 8-15) x (dims nd | nd+1)
    ldmatrix_x4_trans(vb0, vb1, vb2, vb3, vaddr((mtx & 1) * 8 + r, nd2 * 2 + (mtx >> 1)));
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const uint32_t a0 = pack_bf16x2(s[mt][0][0], s[mt][0][1]);
      const uint32_t a1 = pack_bf16x2(s[mt][0][2], s[mt][0][3]);
      const uint32_t a2 = pack_bf16x2(s[mt][1][0], s[mt][1][1]);
      const uint32_t a3 = pack_bf16x2(s[mt][1][2], s[mt][1][3]);
      mma_bf16_16816(o[mt][nd2 * 2 + 0], a0, a1, a2, a3, vb0, vb1);
      mma_bf16_16816(o[mt][nd2 * 2 + 1], a0, a1, a2, a3, vb2, vb3);
    }
  }
}

// One warp: chunks c0, c0 + cstep, ... of the keys [k_begin, k_begin + n_keys)
// of head h, folded into (o, mrow, lrow) with an online softmax.
template <int MT, int DH, int RING_ = 3>
__device__ __forceinline__ void attn_stream_chunks(const AttnArgs& a, int h, int k_begin, int n_keys, int c0,
                                                   int cstep, const __nv_bfloat16* sQ, __nv_bfloat16* ring,
                                                   float (&o)[MT][DH / 8][4], float (&mrow)[MT][2],
                                                   float (&lrow)[MT][2]) {
  using SM = AttnSmem<MT, DH, RING_>;
  constexpr int ROW = SM::ROW;
  constexpr int PIECES = DH / 8;
  const int lane = threadIdx.x & 31;
  const int n_chunks = (n_keys + 15) >> 4;
  const __nv_bfloat16* kbase = a.k + h * a.kv_head_stride;
  const __nv_bfloat16* vbase = a.v + h * a.kv_head_stride;

  // each lane copies DH/16 x 16 bytes of K and of V per chunk: piece i is row
  // r0 + i * RSTEP, column c (fixed per lane); full chunks skip the per-row
  // validity test
  constexpr int RSTEP = 32 / PIECES;
  const int r0 = lane / PIECES, c = (lane % PIECES) * 8;
  // The cross layers' K/V cache is read once per step and is larger than L2
  // at large batch: its lines go first, so that the activations the next
  // GEMMs read (and the outputs they write) stay in L2.  Self-attention
  // reads activation rows: normal priority.
  const uint64_t kv_policy = a.kspan != nullptr && kKvEvictFirst ? policy_evict_first() : policy_evict_normal();
  auto issue = [&](int chunk, int slot) {
    __nv_bfloat16* dk = ring + slot * 2 * SM::CHUNK_ELEMS;
    __nv_bfloat16* dv = dk + SM::CHUNK_ELEMS;
    if (chunk * 16 + 16 <= n_keys) {
      const long long off = (long long)(k_begin + chunk * 16 + r0) * a.kv_ld + c;
      const long long step = (long long)RSTEP * a.kv_ld;
#pragma unroll
      for (int i = 0; i < DH / 16; ++i) {
        cp_async16_hint(dk + (r0 + i * RSTEP) * ROW + c, kbase + off + i * step, true, kv_policy);
        cp_async16_hint(dv + (r0 + i * RSTEP) * ROW + c, vbase + off + i * step, true, kv_policy);
      }
    } else {
#pragma unroll
      for (int i = 0; i < DH / 16; ++i) {
        const int r = r0 + i * RSTEP;
        const int key = chunk * 16 + r;
        const bool valid = key < n_keys;
        const long long row = (long long)(k_begin + (valid ? key : 0));
        cp_async16_hint(dk + r * ROW + c, kbase + row * a.kv_ld + c, valid, kv_policy);
        cp_async16_hint(dv + r * ROW + c, vbase + row * a.kv_ld + c, valid, kv_policy);
      }
    }
  };

  int my_n = 0;
  for (int c = c0; c < n_chunks; c += cstep) ++my_n;
#pragma unroll
  for (int p = 0; p < SM::RING - 1; ++p) {
    if (p < my_n) issue(c0 + cstep * p, p);
    cp_async_commit();
  }

  for (int it = 0; it < my_n; ++it) {
    const int chunk = c0 + cstep * it;
    {
      const int nxt = it + SM::RING - 1;
      if (nxt < my_n) issue(c0 + cstep * nxt, nxt % SM::RING);
      cp_async_commit();
    }
    cp_async_wait<SM::RING - 1>();
    __syncwarp();
    const __nv_bfloat16* sk = ring + (it % SM::RING) * 2 * SM::CHUNK_ELEMS;
    const __nv_bfloat16* sv = sk + SM::CHUNK_ELEMS;
    // padded rows of ROW elements: 16-byte column chunk cc of key row r
    attn_fold_chunk<MT, DH>(
        a, chunk * 16, k_begin, n_keys, sQ,
        [&](int r, int cc) { return sk + r * ROW + cc * 8; },
        [&](int r, int cc) { return sv + r * ROW + cc * 8; }, o, mrow, lrow);
    __syncwarp();   // the slot is refilled by a later issue
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------- split schedule
template <int MT, int DH>
__global__ void __launch_bounds__(kAttnThreads) attention_split_kernel(const AttnArgs a) {
  using SM = AttnSmem<MT, DH>;
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sKV = sQ + SM::Q_ELEMS;
  float* sO = reinterpret_cast<float*>(smem + (SM::Q_ELEMS + 4 * SM::RING_ELEMS) * 2);
  float* sML = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sO) + SM::SPLIT_O_BYTES);

  const int b = blockIdx.x / a.num_heads;
  const int h = blockIdx.x - b * a.num_heads;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int tig = lane & 3;

  pdl_wait();
  pdl_launch_dependents();
  int k_begin, n_keys;
  attn_key_range(a, b, k_begin, n_keys);
  attn_load_q<MT, DH>(a, b, h, sQ, threadIdx.x, kAttnThreads);
  __syncthreads();

  float o[MT][DH / 8][4];
  float mrow[MT][2], lrow[MT][2];
  attn_init<MT, DH>(o, mrow, lrow);
  attn_stream_chunks<MT, DH>(a, h, k_begin, n_keys, warp, 4, sQ, sKV + warp * SM::RING_ELEMS, o, mrow, lrow);

  // per-warp partial results -> shared memory
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float l = lrow[mt][hr];
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      const int row = mt * 16 + g + hr * 8;
      if (tig == 0) {
        sML[(warp * MT * 16 + row) * 2 + 0] = mrow[mt][hr];
        sML[(warp * MT * 16 + row) * 2 + 1] = l;
      }
      float* orow = sO + (warp * MT * 16 + row) * DH;
#pragma unroll
      for (int nd = 0; nd < DH / 8; ++nd) {
        orow[nd * 8 + tig * 2 + 0] = o[mt][nd][hr * 2 + 0];
        orow[nd * 8 + tig * 2 + 1] = o[mt][nd][hr * 2 + 1];
      }
    }
  }
  __syncthreads();

  // combine the 4 warps and write bf16 rows
  __nv_bfloat16* obase = a.out + (long long)b * a.n_tok * a.out_ld + h * DH;
  for (int i = threadIdx.x; i < a.n_tok * (DH / 2); i += kAttnThreads) {
    const int row = i / (DH / 2);
    const int d = (i - row * (DH / 2)) * 2;
    float mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mt = fmaxf(mt, sML[(w * MT * 16 + row) * 2]);
    float r0 = 0.0f, r1 = 0.0f;
    if (mt != -INFINITY) {
      float l = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = sML[(w * MT * 16 + row) * 2];
        const float f = (mw == -INFINITY) ? 0.0f : exp2f(mw - mt);
        l += f * sML[(w * MT * 16 + row) * 2 + 1];
        r0 += f * sO[(w * MT * 16 + row) * DH + d];
        r1 += f * sO[(w * MT * 16 + row) * DH + d + 1];
      }
      const float inv = 1.0f / l;
      r0 *= inv;
      r1 *= inv;
    }
    *reinterpret_cast<uint32_t*>(obase + (long long)row * a.out_ld + d) = pack_bf16x2(r0, r1);
  }
}

// ---------------------------------------------------------------- warp schedule
// Ring depth of the warp schedule: two chunks in flight per warp keep a warp's
// shared memory at 13.8 KB (DH 64), so 16 warps fit an SM.
constexpr int kWarpRing = 2;

// Persistent: warp w of CTA c takes items c * 4 + w, + 4 * gridDim.x, ...; the
// host sizes the grid so that every warp gets the same number of items.
template <int MT, int DH>
__global__ void __launch_bounds__(kAttnThreads, MT == 2 ? 4 : 2) attention_warp_kernel(const AttnArgs a) {
  using SM = AttnSmem<MT, DH, kWarpRing>;
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int tig = lane & 3;
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem) + warp * (SM::Q_ELEMS + SM::RING_ELEMS);
  __nv_bfloat16* ring = sQ + SM::Q_ELEMS;

  pdl_wait();
  pdl_launch_dependents();
  for (int item = blockIdx.x * 4 + warp; item < a.num_items; item += gridDim.x * 4) {
    const int b = item / a.num_heads;
    const int h = item - b * a.num_heads;
    int k_begin, n_keys;
    attn_key_range(a, b, k_begin, n_keys);
    attn_load_q<MT, DH>(a, b, h, sQ, lane, 32);
    __syncwarp();

    float o[MT][DH / 8][4];
    float mrow[MT][2], lrow[MT][2];
    attn_init<MT, DH>(o, mrow, lrow);
    attn_stream_chunks<MT, DH, kWarpRing>(a, h, k_begin, n_keys, 0, 1, sQ, ring, o, mrow, lrow);

    __nv_bfloat16* obase = a.out + (long long)b * a.n_tok * a.out_ld + h * DH;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        float l = lrow[mt][hr];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int row = mt * 16 + g + hr * 8;
        if (row >= a.n_tok) continue;
        const float inv = l > 0.0f ? 1.0f / l : 0.0f;   // no key: zero output
#pragma unroll
        for (int nd = 0; nd < DH / 8; ++nd)
          *reinterpret_cast<uint32_t*>(obase + (long long)row * a.out_ld + nd * 8 + tig * 2) =
              pack_bf16x2(o[mt][nd][hr * 2 + 0] * inv, o[mt][nd][hr * 2 + 1] * inv);
      }
    }
    __syncwarp();   // the Q tile is rewritten by the next item
  }
}

}  // namespace gdit
