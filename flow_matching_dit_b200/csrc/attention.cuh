// Multi-head attention of the action tokens ("Transformer block structure"
// and "AlternateVLDiT variant", Isaac-GR00T architecture page):
//   cross layers (even): the N = H + 1 state/action tokens of a sample attend to
//     that sample's valid backbone tokens, whose K/V were projected once per call;
//   self layers (odd): the N tokens attend to each other (no mask).
// out_h = softmax(q_h k_h^T / sqrt(head_dim)) v_h per head, heads concatenated; a
// sample with no key gets a zero output.
//
// One CTA per (sample, head); its 4 warps split the keys in chunks of 16
// (flash-decoding inside the CTA) and keep an online softmax, then combine
// through shared memory.  Scores and P*V use bf16 mma.sync m16n8k16 with f32
// accumulation: the op is bound by the K/V reads (about 17 FLOP per byte at
// N = 17), which this path keeps up with; queries are padded to 16-row tiles.
#pragma once

#include "ptx.cuh"

namespace gdit {

constexpr int kAttnThreads = 128;

struct AttnArgs {
  const __nv_bfloat16* q;
  long long q_ld;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  long long kv_ld;
  const int* kofs;      // cross: keys of sample b are rows [kofs[b], kofs[b+1]); nullptr: self (rows of q's sample)
  int n_tok;            // queries (tokens) per sample
  int num_heads;
  __nv_bfloat16* out;
  long long out_ld;
  float scale_log2;     // log2(e) / sqrt(head_dim)
};

// MT: 16-row query tiles (queries padded to 16 * MT); DH: head dim (32 or 64).
// Shared-memory rows hold DH + 8 bf16 so fragment loads are bank-conflict free.
template <int MT, int DH>
struct AttnSmem {
  static constexpr int ROW = DH + 8;
  static constexpr int Q_BYTES = MT * 16 * ROW * 2;
  static constexpr int CHUNK_BYTES = 16 * ROW * 2;                // 16 keys x DH dims (padded)
  static constexpr int RING = 3;                                  // chunks in flight per warp
  static constexpr int KV_BYTES = 4 * RING * 2 * CHUNK_BYTES;     // 4 warps x ring x (K, V)
  static constexpr int O_BYTES = 4 * MT * 16 * DH * 4;
  static constexpr int ML_BYTES = 4 * MT * 16 * 2 * 4;
  static constexpr int TOTAL = Q_BYTES + KV_BYTES + O_BYTES + ML_BYTES;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t n = valid ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

template <int MT, int DH>
__global__ void __launch_bounds__(kAttnThreads) attention_kernel(const AttnArgs a) {
  using SM = AttnSmem<MT, DH>;
  constexpr int kRowPad = SM::ROW;
  constexpr int kHeadDim = DH;
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sKV = reinterpret_cast<__nv_bfloat16*>(smem + SM::Q_BYTES);
  float* sO = reinterpret_cast<float*>(smem + SM::Q_BYTES + SM::KV_BYTES);
  float* sML = reinterpret_cast<float*>(smem + SM::Q_BYTES + SM::KV_BYTES + SM::O_BYTES);

  const int b = blockIdx.x / a.num_heads;
  const int h = blockIdx.x - b * a.num_heads;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;     // row group of the mma fragments
  const int tig = lane & 3;    // thread in group

  pdl_wait();

  int k_begin, k_end;
  if (a.kofs != nullptr) {
    k_begin = a.kofs[b];
    k_end = a.kofs[b + 1];
  } else {
    k_begin = b * a.n_tok;
    k_end = k_begin + a.n_tok;
  }
  const int n_keys = k_end - k_begin;

  // ---- queries -> shared memory (rows >= n_tok are zero)
  const __nv_bfloat16* qbase = a.q + (long long)b * a.n_tok * a.q_ld + h * kHeadDim;
  constexpr int PIECES = DH / 8;   // 16-byte pieces per row
  for (int i = threadIdx.x; i < MT * 16 * PIECES; i += kAttnThreads) {
    const int r = i / PIECES, c = (i % PIECES) * 8;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < a.n_tok) val = *reinterpret_cast<const uint4*>(qbase + (long long)r * a.q_ld + c);
    *reinterpret_cast<uint4*>(sQ + r * kRowPad + c) = val;
  }
  __syncthreads();

  float o[MT][DH / 8][4];
  float mrow[MT][2], lrow[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int nd = 0; nd < DH / 8; ++nd)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[mt][nd][j] = 0.0f;
    mrow[mt][0] = mrow[mt][1] = -INFINITY;
    lrow[mt][0] = lrow[mt][1] = 0.0f;
  }

  const int n_chunks = (n_keys + 15) >> 4;
  __nv_bfloat16* ring = sKV + warp * SM::RING * 2 * (16 * kRowPad);
  const __nv_bfloat16* kbase = a.k + h * kHeadDim;
  const __nv_bfloat16* vbase = a.v + h * kHeadDim;

  // each lane copies DH/16 x 16 bytes of K and of V per chunk
  auto issue = [&](int chunk, int slot) {
    __nv_bfloat16* dk = ring + slot * 2 * (16 * kRowPad);
    __nv_bfloat16* dv = dk + 16 * kRowPad;
#pragma unroll
    for (int i = 0; i < DH / 16; ++i) {
      const int idx = lane + 32 * i;      // 16 rows x PIECES pieces
      const int r = idx / PIECES, c = (idx % PIECES) * 8;
      const int key = chunk * 16 + r;
      const bool valid = key < n_keys;
      const long long row = (long long)(k_begin + (valid ? key : 0));
      cp_async16(dk + r * kRowPad + c, kbase + row * a.kv_ld + c, valid);
      cp_async16(dv + r * kRowPad + c, vbase + row * a.kv_ld + c, valid);
    }
  };

  // chunks of this warp: warp, warp + 4, ...
  int my_n = 0;
  for (int c = warp; c < n_chunks; c += 4) ++my_n;
#pragma unroll
  for (int p = 0; p < SM::RING - 1; ++p) {
    if (p < my_n) issue(warp + 4 * p, p);
    cp_async_commit();
  }

  for (int it = 0; it < my_n; ++it) {
    const int chunk = warp + 4 * it;
    {
      const int nxt = it + SM::RING - 1;
      if (nxt < my_n) issue(warp + 4 * nxt, nxt % SM::RING);
      cp_async_commit();
    }
    cp_async_wait<SM::RING - 1>();
    __syncwarp();
    const __nv_bfloat16* sk = ring + (it % SM::RING) * 2 * (16 * kRowPad);
    const __nv_bfloat16* sv = sk + 16 * kRowPad;

    // S = Q K^T for 16 keys (two n-tiles of 8)
    float s[MT][2][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[mt][nt][j] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < DH / 16; ++ks) {
      uint32_t kb[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const __nv_bfloat16* kr = sk + (nt * 8 + g) * kRowPad + ks * 16 + tig * 2;
        kb[nt][0] = *reinterpret_cast<const uint32_t*>(kr);
        kb[nt][1] = *reinterpret_cast<const uint32_t*>(kr + 8);
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const __nv_bfloat16* qr = sQ + (mt * 16 + g) * kRowPad + ks * 16 + tig * 2;
        const uint32_t a0 = *reinterpret_cast<const uint32_t*>(qr);
        const uint32_t a1 = *reinterpret_cast<const uint32_t*>(qr + 8 * kRowPad);
        const uint32_t a2 = *reinterpret_cast<const uint32_t*>(qr + 8);
        const uint32_t a3 = *reinterpret_cast<const uint32_t*>(qr + 8 * kRowPad + 8);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma_bf16_16816(s[mt][nt], a0, a1, a2, a3, kb[nt][0], kb[nt][1]);
      }
    }

    // online softmax (base 2); masked keys get -inf
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {   // hr 0: row g, hr 1: row g + 8
        float x[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int key = chunk * 16 + nt * 8 + tig * 2 + j;
            x[nt * 2 + j] = key < n_keys ? s[mt][nt][hr * 2 + j] * a.scale_log2 : -INFINITY;
          }
        float cm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
        const float m_old = mrow[mt][hr];
        const float m_new = fmaxf(m_old, cm);
        const float alpha = (m_new == -INFINITY) ? 1.0f : exp2f(m_old - m_new);
        float psum = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float p = (m_new == -INFINITY) ? 0.0f : exp2f(x[j] - m_new);
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
      const __nv_bfloat16* vp = sv + ((mtx & 1) * 8 + r) * kRowPad + (nd2 * 2 + (mtx >> 1)) * 8;
      ldmatrix_x4_trans(vb0, vb1, vb2, vb3, vp);
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
    __syncwarp();   // the slot is refilled by a later issue
  }
  cp_async_wait<0>();

  // ---- per-warp partial results -> shared memory
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
      float* orow = sO + (warp * MT * 16 + row) * kHeadDim;
#pragma unroll
      for (int nd = 0; nd < DH / 8; ++nd) {
        orow[nd * 8 + tig * 2 + 0] = o[mt][nd][hr * 2 + 0];
        orow[nd * 8 + tig * 2 + 1] = o[mt][nd][hr * 2 + 1];
      }
    }
  }
  __syncthreads();

  // ---- combine the 4 warps and write bf16 rows
  __nv_bfloat16* obase = a.out + (long long)b * a.n_tok * a.out_ld + h * kHeadDim;
  for (int i = threadIdx.x; i < a.n_tok * (kHeadDim / 2); i += kAttnThreads) {
    const int row = i / (kHeadDim / 2);
    const int d = (i - row * (kHeadDim / 2)) * 2;
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
        r0 += f * sO[(w * MT * 16 + row) * kHeadDim + d];
        r1 += f * sO[(w * MT * 16 + row) * kHeadDim + d + 1];
      }
      const float inv = 1.0f / l;
      r0 *= inv;
      r1 *= inv;
    }
    *reinterpret_cast<uint32_t*>(obase + (long long)row * a.out_ld + d) = pack_bf16x2(r0, r1);
  }
}

}  // namespace gdit
