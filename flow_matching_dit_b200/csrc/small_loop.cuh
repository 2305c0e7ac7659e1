// The whole K-step Euler loop of one sample (B = 1, N = H + 1 tokens) as one
// persistent kernel (Isaac-GR00T architecture page, "Inference (denoising)":
// action encoder -> 32 DiT blocks -> action decoder -> Euler update, K times).
//
// At B = 1 every linear is a weight stream: 17 tokens against a weight matrix
// of 1-8 MB.  Separate launches would pay launch, pipeline fill and tail per
// matrix, so one cooperative launch runs every phase, and weights never wait
// for activations:
//
//   * a phase is a GEMM (out = epilogue(X W^T)) or an attention;
//   * a GEMM's output features are cut into units of 8 (N / 8 units, unit u on
//     CTA u mod grid), so at B = 1 a 1024-wide linear keeps 128 CTAs busy and
//     the 4096-wide FF1 all of them;
//   * one producer warp per CTA walks the phase table ahead of the compute
//     warps and streams this CTA's weight chunks (8 rows x up to 1024 columns,
//     one bulk copy per row into padded rows) into a ring of shared-memory
//     slots, gated only by free slots: while the compute warps wait for the
//     previous phase, the next phases' weights are already arriving; it also
//     asks L2 for the chunks of the phase after next;
//   * the 8 compute warps take the phase's activations X from L2 (bf16 rows,
//     or LN / AdaLN of the f32 residual rows computed by the CTA), split K
//     among themselves (bf16 mma.sync m16n8k16: tokens as the A operand,
//     weight rows as B), reduce through shared memory and run the epilogue
//     (bias, GELU / ReLU / swish, residual add, Euler update);
//   * a cross-attention phase runs one head per CTA (the streaming routine of
//     the attention kernels, keys split over the 8 warps); self-attention (17
//     keys) is computed inside the self layer's O phase by every CTA of it,
//     from its own copy of the QKV rows, so that phase needs no X load.
//
// A batch of 2-4 samples runs the same loop with the grid cut into one group
// of CTAs per sample (148 / B each): each group has its own phase table,
// counters and rows, and streams all the weights itself (the groups read the
// same weights, mostly from L2).  A CTA then has up to 4 x B units of 8
// features in a linear and takes them in passes of up to four.  At B = 2 a
// call takes 5.3 ms against 8.8 ms for the per-layer kernels; from B = 5 on
// the per-layer kernels are faster (9.1 against 9.0 ms at B = 5, 12.4 against
// 9.3 ms at B = 8: a CTA's weight stream, not the shared phase cost, then sets
// the time).
//
// Phases are ordered by arrival counters in global memory: the CTAs that work
// in phase p wait until every CTA that worked in phase p-1 has arrived (each
// of those waited for p-2, so the order is transitive), then arrive on p.
// Every wait is bounded; on expiry the status word records a timeout, every
// warp gives up, and the producer lets its copies land before the CTA exits.
#pragma once

#include "attention.cuh"
#include "gemm_tc.cuh"   // Epi kinds, gelu_erf, swish_f
#include "ptx.cuh"

namespace gdit {

constexpr int kSmallWarps = 8;                           // compute warps
constexpr int kSmallCompute = 32 * kSmallWarps;          // compute threads
constexpr int kSmallThreads = kSmallCompute + 32;        // + the weight-producer warp
constexpr int kSmallMaxTok = 32;
constexpr int kSmallMaxD = 1024;
constexpr int kSmallMaxLayers = 64;
constexpr int kSmallKC = 1024;                           // widest weight chunk (K columns)
constexpr int kSmallUF = 8;                              // output features per unit
constexpr int kSmallMaxUnits = 4;                        // units of one CTA in one pass of a phase
constexpr int kSmallMaxGroups = 4;                       // samples run at once (one CTA group each)
constexpr int kSmallSlots = 5;                           // weight chunks resident at once
constexpr int kSmallPairPhases = 9;                      // phases of a (cross, self) layer pair
constexpr int kSlotRow = kSmallKC + 8;                   // padded slot row (elements): conflict-free ldmatrix
constexpr int kSlotBytes = kSmallUF * kSlotRow * 2;

// dynamic shared memory (bytes)
constexpr int kSmXBytes = 140800;                        // X rows / LN / attention / QKV rows / reduction
constexpr int kSmLnScratchBytes = 4096;                  // LN (mean, rstd) of each row, at the end of the X area
constexpr int kSmLnScratch = kSmXBytes - kSmLnScratchBytes;
constexpr int kLnPieces = kSmallMaxD / 8;                // LayerNorm statistics pieces of a row: one per 8 columns
static_assert(kSmallMaxTok * 8 <= kSmLnScratchBytes, "(mean, rstd) of every row fits the LN scratch");
static_assert(kSmallMaxD / 4 <= kSmallCompute, "one float4 column group per compute thread");
constexpr int kSmRing = kSmXBytes;                       // weight slots
constexpr int kSmHold = kSmRing + kSmallSlots * kSlotBytes;                       // [unit][tok][8] f32 old values
constexpr int kSmBias = kSmHold + kSmallMaxUnits * kSmallMaxTok * kSmallUF * 4;  // [unit][8] f32
constexpr int kSmallSmem = kSmBias + kSmallMaxUnits * kSmallUF * 4;
constexpr int kSmRedBytes = kSmallWarps * kSmallMaxUnits * kSmallMaxTok * kSmallUF * 4;   // over X
static_assert(kSmRedBytes <= kSmXBytes, "reduction buffer fits the X area");

// Cross attention at B = 1 (one head per CTA): the Q tile at the start of the
// X area, the 8 warps' (max, sum) after it, then up to kSmallAttnBlocks TMA
// boxes of kSmallAttnKB keys of K, followed by as many of V (1024-aligned for
// the 128-byte swizzle).
constexpr int kSmallAttnKB = 128;
constexpr int kSmallAttnBlocks = 4;
constexpr int kSmAttnML = 4864;
constexpr int kSmAttnKV = 8192;
static_assert(kSmAttnKV + 1024 + 2 * kSmallAttnBlocks * kSmallAttnKB * 128 <= kSmXBytes,
              "K/V boxes (aligned up to 1024 bytes) fit the X area");
static_assert(kSmallMaxUnits <= kSmallSlots, "one K-chunk of every unit of a phase is resident at once");
static_assert(kSmallSmem <= 227 * 1024 - 1024, "shared memory budget");

// 3 encoder GEMMs, 9 phases per (cross, self) layer pair, norm_out + proj_out
// and the 2 decoder GEMMs (the layer count is even)
__host__ __device__ constexpr int small_phases_per_step(int L) { return kSmallPairPhases * (L / 2) + 6; }

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
  // the K/V cache as a 2-D tensor [layers x {K, V} x heads x max_tok rows, head_dim]
  // for TMA boxes of kSmallAttnKB rows (swizzled like a key row)
  CUtensorMap kv_map;
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
  const int* kspan;          // [begin, end) of the sample's packed keys
  const uint8_t* kflag;      // image flag of each packed backbone token
  int text_every;            // attend_text_every_n_blocks (0: no image/text split)
  // per-K tables: AdaLN [K][L+1][2D], timestep term of the action encoder's W2 [K][C][D]
  const float* ada;
  const float* tw2;
  // weights (category-specific ones as [C][out][in])
  const __nv_bfloat16 *wa1t, *wa2at, *wa3t, *wd1t, *wd2t, *proj_w;
  const float *ba1, *ba3, *bd1, *bd2, *proj_b;
  SmallLayer layers[kSmallMaxLayers];
  int* counters;             // one arrival counter per phase, zero at launch
  struct SmallPhase* phases; // descriptor of every phase, written by small_describe_kernel
  // LayerNorm statistics of the residual rows h, in pieces: the phase that
  // writes h stores, for every row and every 8 columns of it, their (mean,
  // M2) ([kSmallMaxTok][kLnPieces]); a LayerNorm phase combines them
  float2* ln_part;
  unsigned* err;
  int groups;                // samples run at once: one plan per sample, plan[0].groups of them
  int sample;                // this plan's sample (position in the embodiment-sorted batch)
};

struct SmallGemm {
  const __nv_bfloat16* W;
  int N, K;
  const float* bias;         // [N] or nullptr
  const float* vec;          // swish: additive term [N] (bias included)
  int epi;
  int x_mode;                // 0: X from global bf16; 1: LN(h) into shared memory; 2: self-attention of the QKV rows
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

// barrier of the 8 compute warps (the producer warp never joins it)
__device__ __forceinline__ void csync() { named_bar_sync(1, kSmallCompute); }

// ---------------------------------------------------------------- phase ordering

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}


struct alignas(16) SmallPhase {
  int kind;          // 0 GEMM, 1 attention
  int kv_row;        // cross attention: first row of this layer's K block in kv_map
  SmallGemm g;
  AttnArgs a;
};

// Phase `idx` of Euler step k (per step: 3 action-encoder GEMMs, 9 phases per
// (cross, self) block pair, norm_out + proj_out, 2 decoder GEMMs).
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
  if (j < kSmallPairPhases * (L / 2)) {
    // a (cross, self) layer pair: Q, attention, O, FF1, FF2 of the cross layer,
    // then QKV, attention fused into O, FF1, FF2 of the self layer
    const int r = j % kSmallPairPhases;
    const int l = 2 * (j / kSmallPairPhases) + (r >= 5 ? 1 : 0);
    const int part = r < 5 ? r : (r == 5 ? 0 : r - 4);
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
        a.kflag = P.kflag;
        // keys of this cross layer: every valid key, or the text (0) / image (1) ones
        a.ksel = (self || P.text_every <= 0) ? -1 : (l % (2 * P.text_every) == 0 ? 0 : 1);
        if (self) {
          a.q = P.qkv; a.q_ld = 3 * D; a.k = P.qkv + D; a.v = P.qkv + 2 * D; a.kv_ld = 3 * D;
          a.kv_head_stride = P.dh; a.kspan = nullptr;
        } else {
          a.q = P.qkv; a.q_ld = D; a.k = Ly.kv; a.v = Ly.kv + (size_t)P.nh * P.max_tok * P.dh; a.kv_ld = P.dh;
          a.kv_head_stride = P.max_tok * P.dh; a.kspan = P.kspan;
          a.kv_rows = P.max_tok; a.status = P.err;
          ph.kv_row = (int)((long long)(l / 2) * 2 * P.nh * P.max_tok);
        }
        break;
      }
      case 2:                // h += O(attn) + b; self layers compute attn here, from the QKV rows
        g.W = Ly.wo; g.N = D; g.K = D; g.bias = Ly.bo; g.epi = EPI_RESID_F32; g.X = P.o; g.ldx = D;
        g.out = P.h; g.ldo = D;
        if (self) {
          g.x_mode = 2;
          AttnArgs& a = ph.a;
          a.q = P.qkv; a.q_ld = 3 * D; a.k = P.qkv + D; a.v = P.qkv + 2 * D; a.kv_ld = 3 * D;
          a.n_tok = N; a.num_heads = P.nh; a.num_items = P.nh; a.scale_log2 = P.scale_log2; a.ksel = -1;
        }
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
  const int t = j - kSmallPairPhases * (L / 2);
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

// The plan's scalars that the loop reads in every phase, copied into registers
// once: a field read through the plan pointer would be reloaded from global
// memory after every barrier or fence (they clobber memory), and with nearly
// all of L1 given to shared memory each reload is an L2 round trip.
struct SmallCtx {
  unsigned* err;
  int* counters;
  const float* h;
  float eps;
  const SmallPhase* phases;
  const int* vofs;
  int dh;
  int nh;
  long long max_tok;
  const CUtensorMap* kv_map;
  float2* ln_part;
  int rank;                  // this CTA's index in its group (the CTAs that run one sample's loop)
  int gsize;                 // CTAs in the group
};

// Thread 0 waits (acquire) until `target` CTAs have arrived on `phase`; the
// compute warps then continue together.  One counter per phase: a waiter
// polls a single word.  (One flag per CTA, polled as 37 16-byte words by a
// warp, measured 0.85 ms slower per call: the polls flood L2.)
__device__ __forceinline__ bool small_wait(const SmallCtx& P, int phase, int target, int* s_ok) {
  if (threadIdx.x == 0) {
    int ok = 1;
    if (phase >= 0 && target > 0) {
      const int* c = P.counters + phase;
      if (ld_acquire(c) < target) {
        const unsigned long long t0 = globaltimer_ns();
        while (ld_acquire(c) < target) {
          const unsigned long long dt = globaltimer_ns() - t0;
          if (dt > kWaitPeekNs) {
            if (*reinterpret_cast<volatile unsigned*>(P.err) & DEV_ERR_TIMEOUT) { ok = 0; break; }
            if (dt > kWaitTimeoutNs) {
              atomicOr(P.err, DEV_ERR_TIMEOUT);
              ok = 0;
              break;
            }
          }
        }
      }
    }
    *s_ok = ok;
  }
  csync();
  return *s_ok != 0;
}

// One release increment, after the barrier that ends the phase.
__device__ __forceinline__ void small_arrive(const SmallCtx& P, int phase) {
  if (threadIdx.x == 0) red_release_add(P.counters + phase, 1);
}

// ---------------------------------------------------------------- units and chunks

__device__ __forceinline__ int gemm_units(const SmallGemm& g) { return g.N / kSmallUF; }
__device__ __forceinline__ int workers(const SmallCtx& P, int units) { return units < P.gsize ? units : P.gsize; }
__device__ __forceinline__ int small_my_units(const SmallCtx& P, const SmallGemm& g) {
  const int u = gemm_units(g);
  return P.rank < u ? (u - P.rank + P.gsize - 1) / P.gsize : 0;
}
__device__ __forceinline__ int small_kc(const SmallGemm& g) { return g.K < kSmallKC ? g.K : kSmallKC; }
__device__ __forceinline__ int small_nchunks(const SmallGemm& g) { return g.K / small_kc(g); }
// unit j of this CTA (units go round robin over the group's CTAs)
__device__ __forceinline__ int small_unit(const SmallCtx& P, int j) { return P.rank + j * P.gsize; }

__device__ __forceinline__ int small_phase_workers(const SmallCtx& P, const SmallPhase& ph) {
  return ph.kind == 1 ? ph.a.num_heads : workers(P, gemm_units(ph.g));
}

// ---------------------------------------------------------------- weight producer (warp 8)

struct SmallRing {
  uint64_t full[kSmallSlots];    // producer arm + copy bytes
  uint64_t empty[kSmallSlots];   // one arrival per compute warp
};

// Streams this CTA's weight chunks of every GEMM phase, in the order the
// compute warps consume them, into the slot ring; runs ahead as far as free
// slots allow.  Lanes 0..7 each copy one weight row per chunk.  GROUPS: the
// grid may hold several groups, and a CTA more than kSmallMaxUnits units of
// a phase (else one group, one pass).  [k0, k1): the sample's packed keys.
template <bool GROUPS>
__device__ __forceinline__ void small_producer(const SmallCtx& P, int total, int k0, int k1, uint8_t* smem,
                                               SmallRing& R) {
  const int lane = threadIdx.x & 31;
  uint32_t item = 0;
  bool ok = true;
  // The weights are read once per Euler step and 0.75 GB of them pass
  // through L2 per step: with one group they are marked first to evict, so
  // that the activations, the per-step tables and the K/V cache (read every
  // step) stay in L2.  With several groups every group reads every weight
  // line within a few microseconds of the others: evict-first lines were
  // read from DRAM again (4.7 GB per call at B = 2 against 2.95 GB), so they
  // keep the normal policy (B = 4: 7.39 ms per call against 7.61 ms).
  const uint64_t stream_policy = GROUPS ? policy_evict_normal() : policy_evict_first();
  auto l2_ahead = [&](int gp) {   // the chunks of phase gp (if any) towards L2
    if (lane != 0 || gp >= total) return;
    const SmallPhase& ph = P.phases[gp];
    if (ph.kind == 0) {
      const SmallGemm& g = ph.g;
      const int nu = small_my_units(P, g);
      for (int j = 0; j < nu; ++j)
        l2_prefetch_hint(g.W + (size_t)small_unit(P, j) * kSmallUF * g.K, (uint32_t)(kSmallUF * g.K * 2),
                         stream_policy);
    } else if (ph.a.kspan != nullptr && P.rank < ph.a.num_heads) {
      // K and V of this CTA's head: the sample's contiguous rows of the head-major cache
      const uint32_t bytes = (uint32_t)(k1 - k0) * (uint32_t)P.dh * 2u;
      if (bytes > 0) {
        l2_prefetch(ph.a.k + (size_t)P.rank * ph.a.kv_head_stride + (size_t)k0 * P.dh, bytes);
        l2_prefetch(ph.a.v + (size_t)P.rank * ph.a.kv_head_stride + (size_t)k0 * P.dh, bytes);
      }
    }
  };
  l2_ahead(0);
  l2_ahead(1);
  for (int gp = 0; gp < total && ok; ++gp) {
    l2_ahead(gp + 2);
    const SmallPhase& ph = P.phases[gp];
    if (ph.kind != 0) continue;
    const SmallGemm& g = ph.g;
    const int nu_all = small_my_units(P, g), nch = small_nchunks(g), kc = small_kc(g);
    // the compute warps take the units in passes of up to kSmallMaxUnits,
    // each pass chunk by chunk: the same order here
    for (int u0 = 0; u0 < nu_all && ok; u0 += kSmallMaxUnits) {
    const int nu = GROUPS ? min(kSmallMaxUnits, nu_all - u0) : nu_all;
    for (int c = 0; c < nch && ok; ++c) {
      for (int j = 0; j < nu; ++j, ++item) {
        const int slot = (int)(item % kSmallSlots);
        const uint32_t use = item / kSmallSlots;
        int good = 1;
        if (lane == 0) {
          good = mbar_wait(&R.empty[slot], (use & 1u) ^ 1u, P.err);
          if (good) mbar_arrive_expect_tx(&R.full[slot], (uint32_t)(kSmallUF * kc * 2));
        }
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) { ok = false; break; }
        if (lane < kSmallUF) {
          uint8_t* dst = smem + kSmRing + slot * kSlotBytes + lane * kSlotRow * 2;
          const __nv_bfloat16* src =
              g.W + ((size_t)small_unit(P, u0 + j) * kSmallUF + lane) * g.K + (size_t)c * kc;
          bulk_g2s_hint(dst, src, (uint32_t)kc * 2u, &R.full[slot], stream_policy);
        }
      }
    }
    if (!GROUPS) break;
    }
  }
  // Let every copy issued land before the CTA can exit: wait for the last
  // fill of each slot (bounded; on the normal path they were all consumed).
  if (lane == 0) {
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t i = item > (uint32_t)kSmallSlots ? item - kSmallSlots : 0; i < item; ++i) {
      const int slot = (int)(i % kSmallSlots);
      const uint32_t use = i / kSmallSlots;
      while (!mbar_try_wait(&R.full[slot], use & 1u) && globaltimer_ns() - t0 < 10000000ull) {
      }
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------- GEMM phase (compute warps)

// Warp 0: the phase's bf16 activation rows (row stride ldx) by bulk copies on
// `xbar`, into shared rows of K + 8 elements.  The proxy fences order the
// other CTAs' stores (seen through the acquire) and this CTA's earlier reads
// of the area before the async-proxy copies.
__device__ __forceinline__ void small_issue_x(const SmallGemm& g, uint8_t* smem, uint64_t* xbar) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  if (lane == 0) {
    fence_proxy_async_global();
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(xbar, (uint32_t)(g.rows * g.K * 2));
  }
  __syncwarp();
  const int xrow = g.K + 8;
  for (int r = lane; r < g.rows; r += 32)
    bulk_g2s(smem + (size_t)r * xrow * 2, g.X + (size_t)r * g.ldx, (uint32_t)g.K * 2u, xbar);
}

// Bias and, for the residual and Euler epilogues, the old output values of
// this CTA's units: one cp.async group, waited for before the epilogue.
__device__ __forceinline__ void small_issue_side(const SmallGemm& g, const SmallCtx& P, int u0, int nu,
                                                 uint8_t* smem) {
  const int tid = threadIdx.x;
  const float* bsrc = g.epi == EPI_SWISH_VEC_BF16 ? g.vec : g.bias;
  if (bsrc != nullptr && tid < 2 * nu) {
    const int j = tid >> 1, q = tid & 1;
    cp_async16(reinterpret_cast<float*>(smem + kSmBias) + j * kSmallUF + q * 4,
               bsrc + small_unit(P, u0 + j) * kSmallUF + q * 4, true);
  }
  if (g.epi == EPI_RESID_F32 || g.epi == EPI_EULER) {
    float* hold = reinterpret_cast<float*>(smem + kSmHold);
    for (int i = tid; i < nu * g.rows * 2; i += kSmallCompute) {
      const int j = i / (g.rows * 2), rem = i - j * g.rows * 2, r = rem >> 1, q = rem & 1;
      cp_async16(hold + (j * kSmallMaxTok + r) * kSmallUF + q * 4,
                 reinterpret_cast<const float*>(g.out) + (size_t)(g.out_row_off + r) * g.ldo +
                     small_unit(P, u0 + j) * kSmallUF + q * 4,
                 true);
    }
  }
  cp_async_commit();
}

// Shared-memory offset of the f32 rows staged for LayerNorm (after the bf16
// output rows).
__device__ __host__ __forceinline__ int small_ln_stage_offset(int rows, int D) {
  return (rows * (D + 8) * 2 + 127) & ~127;
}
// ... and of the rows' statistics pieces, after the staged rows
__device__ __host__ __forceinline__ int small_ln_piece_offset(int rows, int D) {
  return small_ln_stage_offset(rows, D) + rows * D * 4;
}

// Warp 0: the f32 residual rows that the phase normalises and their
// statistics pieces, by bulk copies into shared memory on `xbar`.  The copy
// engine keeps the whole 90 KB in flight at once; loads through the threads'
// registers are limited by the SM's outstanding-miss capacity and took
// several L2 round trips.
__device__ __forceinline__ void small_issue_ln(const SmallGemm& g, const SmallCtx& P, uint8_t* smem,
                                               uint64_t* xbar) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  const int D = g.K;
  const uint32_t row_bytes = (uint32_t)D * 4u;
  if (lane == 0) {
    fence_proxy_async_global();
    fence_proxy_async_smem();
    const uint32_t piece_bytes = (uint32_t)(g.rows * kLnPieces * 8);
    mbar_arrive_expect_tx(xbar, (uint32_t)g.rows * row_bytes + piece_bytes);
    bulk_g2s(smem + small_ln_piece_offset(g.rows, D), P.ln_part + (size_t)g.h_row_off * kLnPieces, piece_bytes,
             xbar);
  }
  __syncwarp();
  uint8_t* st = smem + small_ln_stage_offset(g.rows, D);
  const float* h0 = P.h + (size_t)g.h_row_off * D;
  for (int r = lane; r < g.rows; r += 32)
    bulk_g2s(st + (size_t)r * row_bytes, h0 + (size_t)r * D, row_bytes, xbar);
}

// Mean and 1/std of the rows a LayerNorm phase normalises, from the pieces
// staged with them: piece i of a row is the mean m_i and the sum of squared
// deviations M2_i of its columns 8i .. 8i + 7, so the row's mean is the mean
// of the m_i and its M2 is sum(M2_i + 8 (m_i - mean)^2) (the pairwise update
// of Chan, Golub and LeVeque, applied to all pieces at once).  A warp per row
// (rows warp, warp + 8, ...), a lane per piece (and pieces 32, 64, 96 after
// it); the reductions of a warp's rows are interleaved, one shuffle level
// for all of them at a time, so their latencies overlap.
constexpr int kLnRowsPerWarp = kSmallMaxTok / kSmallWarps;
constexpr int kLnPiecesPerLane = kLnPieces / 32;
__device__ __forceinline__ void small_ln_stats(const SmallGemm& g, const SmallCtx& P, const uint8_t* smem,
                                               float2* stat) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = g.K, U = D / kSmallUF;
  const float2* pcs = reinterpret_cast<const float2*>(smem + small_ln_piece_offset(g.rows, D));
  float2 pc[kLnRowsPerWarp][kLnPiecesPerLane];
  float s[kLnRowsPerWarp], q[kLnRowsPerWarp], mean[kLnRowsPerWarp];
#pragma unroll
  for (int t = 0; t < kLnRowsPerWarp; ++t) {
    const int r = warp + t * kSmallWarps;
    s[t] = 0.0f;
#pragma unroll
    for (int k = 0; k < kLnPiecesPerLane; ++k) {
      const int i = lane + 32 * k;
      pc[t][k] = (r < g.rows && i < U) ? pcs[r * kLnPieces + i] : make_float2(0.0f, 0.0f);
      s[t] += pc[t][k].x;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int t = 0; t < kLnRowsPerWarp; ++t) s[t] += __shfl_xor_sync(0xffffffffu, s[t], o);
#pragma unroll
  for (int t = 0; t < kLnRowsPerWarp; ++t) {
    mean[t] = s[t] / (float)U;
    q[t] = 0.0f;
#pragma unroll
    for (int k = 0; k < kLnPiecesPerLane; ++k) {
      const float w = lane + 32 * k < U ? (float)kSmallUF : 0.0f;
      const float d = pc[t][k].x - mean[t];
      q[t] += pc[t][k].y + w * d * d;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int t = 0; t < kLnRowsPerWarp; ++t) q[t] += __shfl_xor_sync(0xffffffffu, q[t], o);
  if (lane == 0) {
#pragma unroll
    for (int t = 0; t < kLnRowsPerWarp; ++t) {
      const int r = warp + t * kSmallWarps;
      if (r < g.rows) stat[r] = make_float2(mean[t], rsqrtf(q[t] / (float)D + P.eps));
    }
  }
}

// LN(h rows) -> bf16 X rows, from the rows staged by small_issue_ln and the
// (mean, rstd) of small_ln_stats: thread t owns columns 4t .. 4t + 3 of every
// row, so its AdaLN ((1 + p0), p1) or affine (p0, p1) modulation is loaded
// once, from global memory, before the rows land.
__device__ __forceinline__ void small_ln_apply(const SmallGemm& g, const uint8_t* smem, uint8_t* xout,
                                               const float2* stat, float4 m0, float4 m1) {
  const int D = g.K, d4 = D / 4, xrow = D + 8, c4 = threadIdx.x;
  if (c4 >= d4) return;
  const float4* st = reinterpret_cast<const float4*>(smem + small_ln_stage_offset(g.rows, D)) + c4;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(xout) + 4 * c4;
#pragma unroll 4
  for (int r = 0; r < g.rows; ++r) {
    const float4 x = st[(size_t)r * d4];
    const float2 ms = stat[r];
    uint2 w;
    w.x = pack_bf16x2((x.x - ms.x) * ms.y * m0.x + m1.x, (x.y - ms.x) * ms.y * m0.y + m1.y);
    w.y = pack_bf16x2((x.z - ms.x) * ms.y * m0.z + m1.z, (x.w - ms.x) * ms.y * m0.w + m1.w);
    *reinterpret_cast<uint2*>(xs + (size_t)r * xrow) = w;
  }
}

// The statistics piece of 8 columns of one row, from the 8 adjacent lanes
// that hold them (lanes 8i .. 8i + 7 of a warp): their mean, then the sum of
// their squared deviations from it.  Every lane of the warp takes part.
__device__ __forceinline__ float2 small_piece8(float v) {
  float s = v;
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float m = s * 0.125f;
  const float d = v - m;
  float q = d * d;
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  return make_float2(m, q);
}

// Self-attention of all heads from the phase's own copy of the QKV rows, for
// the O projection that follows in the same phase.  The QKV rows (N tokens,
// 3D wide) sit after the X rows in the X area; the output goes to the X rows.
__device__ __forceinline__ int small_qkv_offset(int rows, int D) { return (rows * (D + 8) * 2 + 127) & ~127; }

__device__ __forceinline__ void small_issue_qkv(const AttnArgs& a, int D, uint8_t* smem, uint64_t* xbar) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  const int rows = a.n_tok, qrow = 3 * D + 8;
  if (lane == 0) {
    fence_proxy_async_global();
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(xbar, (uint32_t)(rows * 3 * D * 2));
  }
  __syncwarp();
  uint8_t* dst = smem + small_qkv_offset(rows, D);
  for (int r = lane; r < rows; r += 32)
    bulk_g2s(dst + (size_t)r * qrow * 2, a.q + (size_t)r * a.q_ld, (uint32_t)(3 * D * 2), xbar);
}

// One warp per head (heads warp, warp + 8, ...), all N <= 32 keys and both
// 16-query tiles at once: S = Q K^T (2 x 4 tiles of 16 x 8; even and odd
// k-steps into separate accumulators, so the dependent mma.sync chains are
// half as long), softmax over the valid keys (base 2), O = P V, rows divided
// by their sums.  Rows and keys past N read the last token (finite values)
// and are masked or never stored.
template <int DH>
__device__ __forceinline__ void small_self_attention_dh(const AttnArgs& a, int D, uint8_t* smem) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int N = a.n_tok, qrow = 3 * D + 8, xrow = D + 8;
  const __nv_bfloat16* qkv = reinterpret_cast<const __nv_bfloat16*>(smem + small_qkv_offset(N, D));
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem);
  for (int h = warp; h < a.num_heads; h += kSmallWarps) {
    const __nv_bfloat16* Qh = qkv + h * DH;
    const __nv_bfloat16* Kh = qkv + D + h * DH;
    const __nv_bfloat16* Vh = qkv + 2 * D + h * DH;
    float s[2][2][4][4];   // [k-step parity][query tile][key tile of 8][fragment]
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[p][mt][nt][e] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < DH / 16; ++ks) {
      uint32_t q[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int qr = min(mt * 16 + (lane & 15), N - 1);
        ldmatrix_x4(q[mt][0], q[mt][1], q[mt][2], q[mt][3], Qh + (size_t)qr * qrow + ks * 16 + (lane >> 4) * 8);
      }
      // K fragments: keys (lane & 7) + 8 (lane >> 4) of each 16-key pair, k half (lane >> 3) & 1
#pragma unroll
      for (int kp = 0; kp < 2; ++kp) {
        const int key = min(kp * 16 + (lane & 7) + ((lane >> 4) << 3), N - 1);
        uint32_t k0, k1, k2, k3;
        ldmatrix_x4(k0, k1, k2, k3, Kh + (size_t)key * qrow + ks * 16 + ((lane >> 3) & 1) * 8);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          mma_bf16_16816(s[ks & 1][mt][2 * kp], q[mt][0], q[mt][1], q[mt][2], q[mt][3], k0, k1);
          mma_bf16_16816(s[ks & 1][mt][2 * kp + 1], q[mt][0], q[mt][1], q[mt][2], q[mt][3], k2, k3);
        }
      }
    }
    // softmax over keys 0..N-1 of each query row (a row's 32 keys: 4 tiles x 4 lanes x 2)
    float inv[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        float m = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = nt * 8 + tig * 2 + e;
            const float sv = s[0][mt][nt][hr * 2 + e] + s[1][mt][nt][hr * 2 + e];
            const float x = key < N ? sv * a.scale_log2 : -INFINITY;
            s[0][mt][nt][hr * 2 + e] = x;
            m = fmaxf(m, x);
          }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        float l = 0.0f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float p = exp2f(s[0][mt][nt][hr * 2 + e] - m);
            s[0][mt][nt][hr * 2 + e] = p;
            l += p;
          }
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        inv[mt][hr] = 1.0f / l;
      }
    // O = P V over the two 16-key chunks; V fragments by ldmatrix.trans, shared by both query tiles
    float o[2][DH / 8][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nd = 0; nd < DH / 8; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[mt][nd][e] = 0.0f;
#pragma unroll
    for (int kc = 0; kc < 2; ++kc) {
      uint32_t pf[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        pf[mt][0] = pack_bf16x2(s[0][mt][2 * kc][0], s[0][mt][2 * kc][1]);
        pf[mt][1] = pack_bf16x2(s[0][mt][2 * kc][2], s[0][mt][2 * kc][3]);
        pf[mt][2] = pack_bf16x2(s[0][mt][2 * kc + 1][0], s[0][mt][2 * kc + 1][1]);
        pf[mt][3] = pack_bf16x2(s[0][mt][2 * kc + 1][2], s[0][mt][2 * kc + 1][3]);
      }
      const int r = lane & 7, mtx = lane >> 3;   // matrices: (keys 0-7 | 8-15) x (dims nd | nd + 8)
      const int key = min(kc * 16 + (mtx & 1) * 8 + r, N - 1);
#pragma unroll
      for (int nd2 = 0; nd2 < DH / 16; ++nd2) {
        uint32_t vb0, vb1, vb2, vb3;
        ldmatrix_x4_trans(vb0, vb1, vb2, vb3, Vh + (size_t)key * qrow + (nd2 * 2 + (mtx >> 1)) * 8);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          mma_bf16_16816(o[mt][nd2 * 2 + 0], pf[mt][0], pf[mt][1], pf[mt][2], pf[mt][3], vb0, vb1);
          mma_bf16_16816(o[mt][nd2 * 2 + 1], pf[mt][0], pf[mt][1], pf[mt][2], pf[mt][3], vb2, vb3);
        }
      }
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = mt * 16 + g + hr * 8;
        if (row < N) {
#pragma unroll
          for (int nd = 0; nd < DH / 8; ++nd)
            *reinterpret_cast<uint32_t*>(xs + (size_t)row * xrow + h * DH + nd * 8 + tig * 2) =
                pack_bf16x2(o[mt][nd][hr * 2] * inv[mt][hr], o[mt][nd][hr * 2 + 1] * inv[mt][hr]);
        }
      }
  }
}

__device__ __forceinline__ void small_self_attention(const AttnArgs& a, int D, uint8_t* smem) {
  if (D / a.num_heads == 64)
    small_self_attention_dh<64>(a, D, smem);
  else
    small_self_attention_dh<32>(a, D, smem);
}

// Returns the value stored (the f32 one for the residual outputs).
__device__ __forceinline__ float small_epilogue(const SmallGemm& g, int n, int tok, float v, float bias,
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
      v += hold;
      reinterpret_cast<float*>(g.out)[idx] = v;
      break;
    default: {   // EPI_EULER
      v = hold + g.alpha * v;
      reinterpret_cast<float*>(g.out)[idx] = v;
      g.out2[(size_t)tok * g.ldo + n] = __float2bfloat16_rn(v);
    }
  }
  return v;
}

// Operands of the MMA loop of one GEMM phase on one compute warp.
struct SmallMmaIn {
  const __nv_bfloat16* xa0;     // token tile 0: this lane's ldmatrix row of the X rows
  const __nv_bfloat16* xa1;     // token tile 1 (rows past the last token repeat it)
  bool two;                     // the phase has a second token tile
  int wrow;                     // this lane's ldmatrix offset in a weight slot
  int ks0, ks1;                 // this warp's k-steps (16 wide) of every chunk
  int kc, nch;                  // chunk width (K columns) and chunk count
  uint32_t base;                // the CTA's weight-chunk count before the phase
};

// The MMAs of one GEMM phase on one compute warp: for chunk c of the phase,
// wait for every unit's weight slot, then run this warp's k-steps of the
// chunk against every unit (token fragments loaded once per k-step), then
// release the slots.  A dependent chain of mma.sync is bound by the
// instruction's latency, which is long next to the few MMAs a warp issues per
// phase here: each (unit, token tile) keeps NS accumulator sets, k-step i
// going to set i % NS, so no chain is longer than kSmallMaxKs / NS.  The sets
// are summed into acc at the end.
constexpr int kSmallMaxKs = kSmallKC / 16 / kSmallWarps;   // k-steps of one warp in one chunk
template <int NU, int NS>
__device__ __forceinline__ void small_mma_units(const SmallMmaIn& in, uint8_t* smem, SmallRing& R,
                                                const SmallCtx& P, bool& ok, float (&acc)[kSmallMaxUnits][2][4]) {
  const int lane = threadIdx.x & 31;
  float a_s[NU][NS][2][4];
#pragma unroll
  for (int j = 0; j < NU; ++j)
#pragma unroll
    for (int q = 0; q < NS; ++q)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) a_s[j][q][t][e] = 0.0f;
  for (int c = 0; c < in.nch; ++c) {
    const __nv_bfloat16* wsj[NU];
#pragma unroll
    for (int j = 0; j < NU; ++j) {
      const uint32_t it = in.base + (uint32_t)(c * NU + j);
      const int slot = (int)(it % kSmallSlots);
      if (ok && !mbar_wait(&R.full[slot], (it / kSmallSlots) & 1u, P.err)) ok = false;
      wsj[j] = reinterpret_cast<const __nv_bfloat16*>(smem + kSmRing + slot * kSlotBytes) + in.wrow;
    }
    if (!ok) continue;
    const int kx = c * in.kc;
    // two k-steps at a time: the weight fragments of both in one ldmatrix.x4
    // (shared-memory instructions, not the MMAs, are what this loop waits on)
#pragma unroll
    for (int i = 0; i < kSmallMaxKs; i += 2) {
      const int s = in.ks0 + i;
      const int k = s * 16;
      if (s + 1 < in.ks1) {
        uint32_t b[NU][4];
        {
          uint32_t a[4], e[4];   // token tile 0
          ldmatrix_x4(a[0], a[1], a[2], a[3], in.xa0 + kx + k);
          ldmatrix_x4(e[0], e[1], e[2], e[3], in.xa0 + kx + k + 16);
#pragma unroll
          for (int j = 0; j < NU; ++j) {
            ldmatrix_x4(b[j][0], b[j][1], b[j][2], b[j][3], wsj[j] + k);
            mma_bf16_16816(a_s[j][i % NS][0], a[0], a[1], a[2], a[3], b[j][0], b[j][1]);
            mma_bf16_16816(a_s[j][(i + 1) % NS][0], e[0], e[1], e[2], e[3], b[j][2], b[j][3]);
          }
        }
        if (in.two) {
          uint32_t a[4], e[4];   // token tile 1
          ldmatrix_x4(a[0], a[1], a[2], a[3], in.xa1 + kx + k);
          ldmatrix_x4(e[0], e[1], e[2], e[3], in.xa1 + kx + k + 16);
#pragma unroll
          for (int j = 0; j < NU; ++j) {
            mma_bf16_16816(a_s[j][i % NS][1], a[0], a[1], a[2], a[3], b[j][0], b[j][1]);
            mma_bf16_16816(a_s[j][(i + 1) % NS][1], e[0], e[1], e[2], e[3], b[j][2], b[j][3]);
          }
        }
      } else if (s < in.ks1) {   // an odd last k-step (narrow K)
        uint32_t a[4], a1[4];
        ldmatrix_x4(a[0], a[1], a[2], a[3], in.xa0 + kx + k);
        if (in.two) ldmatrix_x4(a1[0], a1[1], a1[2], a1[3], in.xa1 + kx + k);
#pragma unroll
        for (int j = 0; j < NU; ++j) {
          uint32_t b0, b1;
          ldmatrix_x2(b0, b1, wsj[j] + k);
          mma_bf16_16816(a_s[j][i % NS][0], a[0], a[1], a[2], a[3], b0, b1);
          if (in.two) mma_bf16_16816(a_s[j][i % NS][1], a1[0], a1[1], a1[2], a1[3], b0, b1);
        }
      }
    }
    __syncwarp();
    if (lane == 0)
#pragma unroll
      for (int j = 0; j < NU; ++j) mbar_arrive(&R.empty[(in.base + (uint32_t)(c * NU + j)) % kSmallSlots]);
  }
#pragma unroll
  for (int j = 0; j < kSmallMaxUnits; ++j)
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = 0.0f;
        if (j < NU) {
#pragma unroll
          for (int q = 0; q < NS; ++q) v += a_s[j < NU ? j : 0][q][t][e];
        }
        acc[j][t][e] = v;
      }
}

// One GEMM phase on the compute warps.  Chunk `item` of the CTA's running
// count sits in slot item % kSmallSlots, filled for the (item / kSmallSlots)-th
// time; a phase's items go chunk by chunk (every unit's K-chunk 0, then 1 ...)
// and every warp releases a slot after its last read of it.
template <bool GROUPS>
__device__ __forceinline__ bool small_gemm_phase(const SmallGemm& g, const AttnArgs& att, const SmallCtx& P,
                                                 uint8_t* smem, SmallRing& R, uint32_t& item, uint64_t* xbar,
                                                 uint32_t& xuse, int* fail) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, tig = lane & 3;
  const int nu_all = small_my_units(P, g), nch = small_nchunks(g), kc = small_kc(g);
  small_issue_side(g, P, 0, GROUPS ? min(kSmallMaxUnits, nu_all) : nu_all, smem);
  bool ok = true;
  if (g.x_mode == 0) {
    small_issue_x(g, smem, xbar);
    // every thread waits for the activations itself: no barrier before the MMAs
    ok = mbar_wait(xbar, xuse & 1u, P.err);
    ++xuse;
  } else if (g.x_mode == 1) {
    small_issue_ln(g, P, smem, xbar);
    float4 m0 = make_float4(0.0f, 0.0f, 0.0f, 0.0f), m1 = m0;
    if ((int)threadIdx.x < g.K / 4) {
      const float add = g.ln_mode == 0 ? 1.0f : 0.0f;
      m0 = __ldg(reinterpret_cast<const float4*>(g.p0) + threadIdx.x);
      m1 = __ldg(reinterpret_cast<const float4*>(g.p1) + threadIdx.x);
      m0.x += add; m0.y += add; m0.z += add; m0.w += add;
    }
    float2* stat = reinterpret_cast<float2*>(smem + kSmLnScratch);
    if (!mbar_wait(xbar, xuse & 1u, P.err)) *fail = 1;
    ++xuse;
    small_ln_stats(g, P, smem, stat);   // every lane (shuffles); unused after a failed wait
    csync();                       // a failed wait is seen by every thread; stat complete
    ok = *fail == 0;
    if (ok) small_ln_apply(g, smem, smem, stat, m0, m1);
    csync();
  } else {
    small_issue_qkv(att, g.K, smem, xbar);
    ok = mbar_wait(xbar, xuse & 1u, P.err);
    ++xuse;
    if (ok) small_self_attention(att, g.K, smem);
    csync();
  }
  const int xrow = g.K + 8;
  const __nv_bfloat16* xs = reinterpret_cast<const __nv_bfloat16*>(smem);
  const int ks = kc / 16;
  const int ks0 = warp * ks / kSmallWarps, ks1 = (warp + 1) * ks / kSmallWarps;
  const bool two = g.rows > 16;
  // tile 0 (tokens 0-15): ldmatrix rows (rows past the last token repeat it:
  // their products land in accumulator rows that are never stored)
  const int ar0 = min(lane & 15, g.rows - 1);
  const __nv_bfloat16* xa0 = xs + (size_t)ar0 * xrow + (lane >> 4) * 8;
  // tile 1 (tokens 16-31) usually holds one real token; its rows past the
  // last token repeat it as well
  const int ar1 = min(16 + (lane & 15), g.rows - 1);
  const __nv_bfloat16* xa1 = xs + (size_t)ar1 * xrow + (lane >> 4) * 8;
  // weight fragments: ldmatrix.x4 over k, k + 8, k + 16, k + 24 (two k-steps;
  // lanes 0-15 also address the x2 form of one k-step)
  const int wrow = (lane & 7) * kSlotRow + (lane >> 3) * 8;
  // One pass over units u0 .. u0 + nu - 1 of this CTA (nu <= kSmallMaxUnits):
  // MMAs, the cross-warp reduction through `red`, the epilogue.
  auto pass = [&](int u0, int nu, float* red) {
    const uint32_t base = item;
    float acc[kSmallMaxUnits][2][4];
    SmallMmaIn in{xa0, xa1, two, wrow, ks0, ks1, kc, nch, base};
    switch (nu) {
      case 1: small_mma_units<1, 2>(in, smem, R, P, ok, acc); break;
      case 2: small_mma_units<2, 2>(in, smem, R, P, ok, acc); break;
      case 3: small_mma_units<3, 2>(in, smem, R, P, ok, acc); break;
      default: small_mma_units<4, 2>(in, smem, R, P, ok, acc); break;
    }
    item = base + (uint32_t)(nch * nu);
    // all warps stay together from here on, also on a timeout
    cp_async_wait<0>();   // bias / old values
    csync();
#pragma unroll
    for (int j = 0; j < kSmallMaxUnits; ++j) {
      if (j < nu) {
        float* rw = red + ((warp * kSmallMaxUnits + j) * kSmallMaxTok) * kSmallUF;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int tok = t * 16 + gr;
          rw[tok * kSmallUF + 2 * tig] = acc[j][t][0];
          rw[tok * kSmallUF + 2 * tig + 1] = acc[j][t][1];
          rw[(tok + 8) * kSmallUF + 2 * tig] = acc[j][t][2];
          rw[(tok + 8) * kSmallUF + 2 * tig + 1] = acc[j][t][3];
        }
      }
    }
    csync();
    const bool has_bias = (g.epi == EPI_SWISH_VEC_BF16 ? g.vec : g.bias) != nullptr;
    const float* biases = reinterpret_cast<const float*>(smem + kSmBias);
    const float* holds = reinterpret_cast<const float*>(smem + kSmHold);
    // a phase that writes h also leaves the LayerNorm statistics piece of
    // every (row, unit) it wrote: the 8 lanes 8i .. 8i + 7 hold one (unit,
    // row), as the CTA's outputs are walked unit by unit, row by row, column
    // by column
    const bool pieces = g.epi == EPI_F32 || g.epi == EPI_RESID_F32;
    const int per_unit = g.rows * kSmallUF, n_out = nu * per_unit;
    for (int b0 = 0; b0 < n_out; b0 += kSmallCompute) {   // the same trip count in every thread
      const int idx = b0 + (int)threadIdx.x;
      const bool mine = idx < n_out;
      const int j = mine ? idx / per_unit : 0, rem = idx - j * per_unit;
      const int tok = rem / kSmallUF, fi = rem - tok * kSmallUF;
      float r = 0.0f;
      if (mine) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kSmallWarps; ++w)
          v += red[((w * kSmallMaxUnits + j) * kSmallMaxTok + tok) * kSmallUF + fi];
        r = small_epilogue(g, small_unit(P, u0 + j) * kSmallUF + fi, tok, v,
                           has_bias ? biases[j * kSmallUF + fi] : 0.0f, holds[(j * kSmallMaxTok + tok) * kSmallUF + fi]);
      }
      if (pieces) {
        const float2 pc = small_piece8(r);
        if (mine && fi == 0 && ok)
          P.ln_part[(size_t)(g.out_row_off + tok) * kLnPieces + small_unit(P, u0 + j)] = pc;
      }
    }
    // the action encoder's output row 0 is the state row, copied (its pieces too)
    if (g.state_row != nullptr && (int)threadIdx.x < 32 * ((nu * kSmallUF + 31) / 32)) {
      const int t = threadIdx.x;
      const bool mine = t < nu * kSmallUF;
      const int n = small_unit(P, u0 + t / kSmallUF) * kSmallUF + t % kSmallUF;
      const float v = mine ? g.state_row[n] : 0.0f;
      if (mine) reinterpret_cast<float*>(g.out)[n] = v;
      const float2 pc = small_piece8(v);
      if (mine && t % kSmallUF == 0 && ok) P.ln_part[small_unit(P, u0 + t / kSmallUF)] = pc;
    }
  };
  if constexpr (!GROUPS) {
    pass(0, nu_all, reinterpret_cast<float*>(smem));   // the reduction over the X area, no longer read
  } else {
    // More than kSmallMaxUnits units: several passes.  The reduction goes
    // after the activation rows (they are read again), or, when the rows
    // fill the area (the FF2 input), over them, and they are copied in again
    // for each later pass.
    int red_off = 0;
    bool reload = false;
    if (nu_all > kSmallMaxUnits) {
      const int off = small_ln_stage_offset(g.rows, g.K);
      if (off + kSmRedBytes <= kSmLnScratch) red_off = off;
      else reload = true;
      if (reload && g.x_mode != 0) ok = false;   // computed rows cannot be copied in again (the host rules it out)
    }
    for (int u0 = 0; u0 < nu_all; u0 += kSmallMaxUnits) {
      const int nu = min(kSmallMaxUnits, nu_all - u0);
      if (u0 > 0) {   // the previous pass ended with a barrier: side area and rows are free
        small_issue_side(g, P, u0, nu, smem);
        if (reload) {
          small_issue_x(g, smem, xbar);
          if (!mbar_wait(xbar, xuse & 1u, P.err)) ok = false;
          ++xuse;
        }
      }
      pass(u0, nu, reinterpret_cast<float*>(smem + red_off));
      if (u0 + kSmallMaxUnits < nu_all) {   // another pass: its side loads and rows may overwrite these
        cp_async_wait<0>();
        csync();
      }
    }
  }
  // One barrier ends the phase: every thread's epilogue stores precede the
  // arrival (thread 0 releases right after it), the X area and the slot of
  // this phase's descriptor may be rewritten after it (every thread waited
  // for its descriptor copies first), and the failure flag is uniform.
  if (!ok) *fail = 1;
  cp_async_wait<0>();
  csync();
  return *fail == 0;
}

// ---------------------------------------------------------------- attention phase (one CTA per head)

// Byte offset of 16-byte column chunk c of key row r in a TMA box of
// head_dim-wide bf16 rows: the 128-byte swizzle for 128-byte rows (DH 64),
// the 64-byte swizzle for 64-byte rows (DH 32).
template <int DH>
__device__ __forceinline__ int small_kv_swz(int r, int c) {
  if constexpr (DH == 64)
    return r * 128 + ((c ^ (r & 7)) << 4);
  else
    return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}

// Cross attention of one head on this CTA (B = 1).  Warp 0 requests the
// head's K and V rows as 2-D TMA boxes of kSmallAttnKB keys (up to
// kSmallAttnBlocks boxes of each at a time: longer key lists take several
// passes); the box rows past the last key are zeroed once they land, so
// their products are finite and masked.  Warp w folds the 16-key chunks
// w, w + 8, ... of the resident keys into its online softmax; the 8 warps'
// partial results are combined at the end (over the K/V area).
template <int DH>
__device__ __forceinline__ bool small_cross_attention(const SmallPhase& ph, const SmallCtx& P, int head,
                                                      uint8_t* smem, uint64_t* xbar, uint32_t& xuse, int* fail) {
  constexpr int NW = kSmallWarps;
  constexpr int BOX = kSmallAttnKB * DH * 2;
  const AttnArgs& a = ph.a;
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  float* sML = reinterpret_cast<float*>(smem + kSmAttnML);
  // the swizzle pattern follows absolute shared-memory address bits: boxes
  // start on a 1024-byte boundary
  const uint32_t kv0 = smem_u32(smem + kSmAttnKV);
  uint8_t* sK = smem + kSmAttnKV + (((kv0 + 1023u) & ~1023u) - kv0);
  uint8_t* sV = sK + kSmallAttnBlocks * BOX;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, tig = lane & 3;
  int k_begin, n_keys;
  attn_key_range(a, 0, k_begin, n_keys);
  const int krow = ph.kv_row + head * (int)P.max_tok + k_begin;
  const int vrow = ph.kv_row + (P.nh + head) * (int)P.max_tok + k_begin;
  const int nblk = (n_keys + kSmallAttnKB - 1) / kSmallAttnKB;
  // K/V boxes of pass b0 (thread 0), on xbar
  auto issue_kv = [&](int b0) {
    if (threadIdx.x != 0) return;
    const int nb = min(kSmallAttnBlocks, nblk - b0);
    fence_proxy_async_smem();   // earlier reads of the area precede the copies
    mbar_arrive_expect_tx(xbar, (uint32_t)(2 * nb * BOX));
    for (int b = 0; b < nb; ++b) {
      tma_load_2d(sK + b * BOX, P.kv_map, xbar, 0, krow + (b0 + b) * kSmallAttnKB);
      tma_load_2d(sV + b * BOX, P.kv_map, xbar, 0, vrow + (b0 + b) * kSmallAttnKB);
    }
  };
  // the first pass's keys are requested before the queries are loaded: the
  // query loads (an L2 round trip) then overlap the K/V copies
  if (nblk > 0) issue_kv(0);
  attn_load_q<2, DH>(a, 0, head, sQ, threadIdx.x, kSmallCompute);
  float o[2][DH / 8][4];
  float mrow[2][2], lrow[2][2];
  attn_init<2, DH>(o, mrow, lrow);
  bool ok = true;
  for (int b0 = 0; b0 < nblk; b0 += kSmallAttnBlocks) {
    const int nb = min(kSmallAttnBlocks, nblk - b0);
    if (b0 > 0) issue_kv(b0);
    if (!mbar_wait(xbar, xuse & 1u, P.err)) *fail = 1;
    ++xuse;
    // rows past the last key (in the last box) hold other tokens or nothing
    // written yet: zero them (K and V)
    const int valid = min(n_keys - b0 * kSmallAttnKB, nb * kSmallAttnKB);
    for (int i = threadIdx.x; i < (nb * kSmallAttnKB - valid) * (DH / 8); i += kSmallCompute) {
      const int r = valid + i / (DH / 8), c = i % (DH / 8);
      const int off = (r / kSmallAttnKB) * BOX + small_kv_swz<DH>(r % kSmallAttnKB, c);
      *reinterpret_cast<uint4*>(sK + off) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sV + off) = make_uint4(0, 0, 0, 0);
    }
    csync();
    ok = *fail == 0;
    if (!ok) break;
    for (int ch = warp; ch * 16 < valid; ch += NW) {
      const int r0 = ch * 16;   // first row of the chunk among the resident keys
      attn_fold_chunk<2, DH>(
          a, b0 * kSmallAttnKB + r0, k_begin, n_keys, sQ,
          [&](int r, int c) {
            const int rr = r0 + r;
            return sK + (rr / kSmallAttnKB) * BOX + small_kv_swz<DH>(rr % kSmallAttnKB, c);
          },
          [&](int r, int c) {
            const int rr = r0 + r;
            return sV + (rr / kSmallAttnKB) * BOX + small_kv_swz<DH>(rr % kSmallAttnKB, c);
          },
          o, mrow, lrow);
    }
    csync();   // the boxes are rewritten by the next pass, or by the partial results
  }
  if (ok) {
    // per-warp partial results -> shared memory (over the K/V boxes), then the
    // combination across warps, bf16 rows of the head's output columns
    float* sO = reinterpret_cast<float*>(sK) + warp * 32 * DH;
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
        float* orow = sO + row * DH;
#pragma unroll
        for (int nd = 0; nd < DH / 8; ++nd) {
          orow[nd * 8 + tig * 2 + 0] = o[mt][nd][hr * 2 + 0];
          orow[nd * 8 + tig * 2 + 1] = o[mt][nd][hr * 2 + 1];
        }
      }
    }
    csync();
    __nv_bfloat16* obase = a.out + head * DH;
    for (int i = threadIdx.x; i < a.n_tok * (DH / 2); i += kSmallCompute) {
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
          const float* ow = reinterpret_cast<const float*>(sK) + (w * 32 + row) * DH;
          l += f * sML[(w * 32 + row) * 2 + 1];
          r0 += f * ow[d];
          r1 += f * ow[d + 1];
        }
        const float inv = 1.0f / l;
        r0 *= inv;
        r1 *= inv;
      }
      *reinterpret_cast<uint32_t*>(obase + (size_t)row * a.out_ld + d) = pack_bf16x2(r0, r1);
    }
  }
  // one barrier ends the phase: stores before the arrival, shared memory and
  // the descriptor slot free afterwards
  cp_async_wait<0>();
  csync();
  return *fail == 0;
}

template <int DH>
struct SmallSmem {
  static constexpr int TOTAL = kSmallSmem;
  static_assert(32 * (DH + 8) * 2 <= kSmAttnML && kSmAttnML + kSmallWarps * 32 * 2 * 4 <= kSmAttnKV,
                "attention Q tile and (max, sum) fit before the K/V boxes");
  static_assert(kSmallWarps * 32 * DH * 4 <= kSmallAttnBlocks * kSmallAttnKB * DH * 2,
                "the warps' partial outputs fit the K boxes");
};

__device__ __forceinline__ int small_category(const SmallPlan& P) {
  int c = 0;   // category of the plan's sample (an out-of-range id was routed to 0)
  for (int i = 0; i < P.C; ++i)
    if (P.seg[i] <= P.sample && P.sample < P.seg[i + 1]) c = i;
  return c;
}

// One thread per (sample, phase): the descriptor tables of the whole loop.
__global__ void small_describe_kernel(const SmallPlan* __restrict__ plan) {
  pdl_wait();
  pdl_launch_dependents();
  const int per_step = small_phases_per_step(plan->L);
  const int total = per_step * plan->K;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total * plan->groups) return;
  const SmallPlan& P = plan[i / total];
  const int gp = i % total;
  small_describe(P, small_category(P), gp / per_step, gp % per_step, P.phases[gp]);
}

// compute threads: descriptor gp -> shared slot, as one cp.async group (no
// stall; complete by the next wait_group 0)
__device__ __forceinline__ void small_fetch_phase(const SmallPhase* phases, int gp, SmallPhase* dst) {
  static_assert(sizeof(SmallPhase) % 16 == 0, "descriptor copied in 16-byte pieces");
  constexpr int kPieces = (int)(sizeof(SmallPhase) / 16);
  static_assert(kPieces <= kSmallCompute, "one piece per thread");
  if (threadIdx.x < kPieces)
    cp_async16(reinterpret_cast<uint8_t*>(dst) + threadIdx.x * 16,
               reinterpret_cast<const uint8_t*>(phases + gp) + threadIdx.x * 16, true);
  cp_async_commit();
}

template <int DH, bool GROUPS>
__global__ void __launch_bounds__(kSmallThreads, 1) small_loop_kernel(const SmallPlan* __restrict__ plan) {
  extern __shared__ __align__(16) uint8_t smem[];
  // phase descriptors: slot gp % 3 holds the current phase; the one two ahead
  // is fetched while the current one runs
  __shared__ __align__(16) SmallPhase s_ph[3];
  __shared__ __align__(8) SmallRing s_ring;
  __shared__ __align__(8) uint64_t s_xbar;
  __shared__ int s_ok;
  __shared__ int s_fail;
  // the grid is cut into plan->groups equal groups of CTAs, one per sample:
  // group q runs the loop of sample q on its own plan, counters and tables
  // (without GROUPS there is one group: the whole grid, one pass per phase)
  const int gsize = GROUPS ? (int)gridDim.x / plan->groups : (int)gridDim.x;
  const int group = GROUPS ? (int)blockIdx.x / gsize : 0;
  if (group >= plan->groups) return;   // (the host launches groups x gsize CTAs)
  const SmallPlan* gpl = plan + group;
  const SmallCtx P = {gpl->err,  gpl->counters, gpl->h,  gpl->eps,     gpl->phases,
                      gpl->vofs, gpl->dh,       gpl->nh, gpl->max_tok, &gpl->kv_map, gpl->ln_part,
                      (int)blockIdx.x - group * gsize, gsize};
  const int total = small_phases_per_step(gpl->L) * gpl->K;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSmallSlots; ++i) {
      mbar_init(&s_ring.full[i], 1);
      mbar_init(&s_ring.empty[i], kSmallWarps);
    }
    mbar_init(&s_xbar, 1);
    fence_mbar_init();
    s_fail = 0;
  }
  __syncthreads();
  if (threadIdx.x >= kSmallCompute) {
    // the key span was written by an earlier kernel: read once, for the L2 requests
    small_producer<GROUPS>(P, total, gpl->kspan[0], gpl->kspan[1], smem, s_ring);
    return;
  }
  small_fetch_phase(P.phases, 0, &s_ph[0]);
  if (total > 1) small_fetch_phase(P.phases, 1, &s_ph[1]);
  cp_async_wait<0>();
  csync();
  uint32_t item = 0;   // weight chunks consumed so far (same count in every compute thread)
  uint32_t xuse = 0;   // activation loads on s_xbar so far
  int prev_workers = 0;
  int slot = 0;        // gp % 3
  for (int gp = 0; gp < total; ++gp) {
    const SmallPhase& cur = s_ph[slot];
    if (gp + 2 < total) small_fetch_phase(P.phases, gp + 2, &s_ph[slot == 0 ? 2 : slot - 1]);
    const int w = small_phase_workers(P, cur);
    bool ok = true;
    if (P.rank < w) {
      ok = small_wait(P, gp - 1, prev_workers, &s_ok);
      if (ok) {
        if (cur.kind == 0)
          ok = small_gemm_phase<GROUPS>(cur.g, cur.a, P, smem, s_ring, item, &s_xbar, xuse, &s_fail);
        else
          ok = small_cross_attention<DH>(cur, P, P.rank, smem, &s_xbar, xuse, &s_fail);
        if (ok) small_arrive(P, gp);
      }
    }
    if (!ok) {
      cp_async_wait<0>();   // requested rows land before the CTA exits
      if (threadIdx.x == 0) {
        // the last activation load (if any) lands too
        const unsigned long long t0 = globaltimer_ns();
        while (xuse > 0u && !mbar_try_wait(&s_xbar, (xuse - 1u) & 1u) && globaltimer_ns() - t0 < 10000000ull) {
        }
      }
      return;
    }
    prev_workers = w;
    if (P.rank >= w) {
      // an idle CTA: the next descriptor has landed, and every compute thread
      // is done with this one before its slot is refilled (a working CTA's
      // phase ended with that barrier)
      cp_async_wait<0>();
      csync();
    }
    slot = slot == 2 ? 0 : slot + 1;
  }
}

}  // namespace gdit
