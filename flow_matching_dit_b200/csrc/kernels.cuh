// Bandwidth-bound kernels of the action head: embodiment routing, backbone
// mask compaction, input gather / output scatter, LayerNorm + AdaLN
// modulation, and the per-K timestep tables.  All accesses are vectorised
// (16-byte) and coalesced; reductions use warp shuffles.
#pragma once

#include "ptx.cuh"

namespace gdit {

// Device copies of the caller's I/O pointers for one call.  A tiny kernel
// writes them before each graph replay, so a captured graph serves any buffers.
struct IoPtrs {
  const void* feats;
  const uint8_t* mask;
  const float* state;
  const int32_t* ids;
  const float* noise;
  float* out;
  const uint8_t* image_mask;   // [B, S] 1 = image token, or nullptr (none)
};

__global__ void set_io_kernel(IoPtrs* dst, IoPtrs src) { *dst = src; }

// ---------------------------------------------------------------- routing
//
// The embodiment id selects the encoders and the decoder (PhyAI "Single-GPU
// inference", Overview; CategorySpecificLinear, Isaac-GR00T architecture
// page).  Samples are stably sorted by id so that each category's rows are
// contiguous for the grouped GEMMs:
//   perm[i]  original index of the i-th sample in sorted order
//   seg[c]   first sorted position of category c (seg[C] = B)
//   vofs[b]  first packed valid backbone token of sample b (vofs[B] = total):
//            the tokens are packed in the caller's sample order, so that the
//            packing and the K/V projection of a range of samples can start
//            as soon as those samples' features have arrived
//   kspan[2i], kspan[2i + 1]  the packed tokens [begin, end) of sorted sample i
// An id outside [0, C) is routed to category 0 (never read out of bounds),
// flagged in bad[b], and reported through the status word.
constexpr int kRouteThreads = 1024;
constexpr int kMaxBatch = 4096;

__global__ void __launch_bounds__(kRouteThreads)
    route_kernel(const IoPtrs* io, int B, int S, int C, int* perm, int* seg, int* vofs, int* kspan, uint8_t* bad,
                 unsigned* status) {
  __shared__ int s_cnt[kMaxBatch];
  __shared__ int s_cat[kMaxBatch];
  __shared__ int s_pos[65];
  pdl_wait();
  pdl_launch_dependents();
  const int32_t* ids = io->ids;
  const uint8_t* mask = io->mask;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int b = warp; b < B; b += kRouteThreads / 32) {
    int c = 0;
    const uint8_t* mrow = mask + (long long)b * S;
    for (int j = lane; j < S; j += 32) c += mrow[j] != 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) s_cnt[b] = c;
  }
  for (int b = threadIdx.x; b < B; b += kRouteThreads) {
    int id = ids[b];
    const bool ok = id >= 0 && id < C;
    bad[b] = ok ? 0 : 1;
    if (!ok) {
      atomicOr(status, DEV_ERR_BAD_ID);
      id = 0;
    }
    s_cat[b] = id;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int c = 0; c <= C; ++c) s_pos[c] = 0;
    for (int b = 0; b < B; ++b) s_pos[s_cat[b] + 1]++;
    for (int c = 0; c < C; ++c) s_pos[c + 1] += s_pos[c];
    for (int c = 0; c <= C; ++c) seg[c] = s_pos[c];
    for (int b = 0; b < B; ++b) perm[s_pos[s_cat[b]]++] = b;   // stable: ties keep sample order
    int acc = 0;
    for (int b = 0; b < B; ++b) {
      vofs[b] = acc;
      acc += s_cnt[b];
    }
    vofs[B] = acc;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < B; i += kRouteThreads) {
    const int b = perm[i];
    kspan[2 * i] = vofs[b];
    kspan[2 * i + 1] = vofs[b] + s_cnt[b];
  }
}

// ---------------------------------------------------------------- packing
//
// Copies the valid backbone tokens (vl_mask == 1; Isaac-GR00T architecture
// page, backbone forward: attention_mask == 1) of samples b0, b0 + 1, ... in
// the caller's sample order to a dense bf16 matrix Xp [total_valid, Dvl].
// Only these rows enter the K/V projection, so padding costs nothing
// downstream.  grid = (sample - b0, chunk of 32 positions).
constexpr int kPackThreads = 256;

__global__ void __launch_bounds__(kPackThreads)
    pack_features_kernel(const IoPtrs* io, int bb_bf16, int S, int Dvl, int b0, const int* vofs, __nv_bfloat16* xp,
                         uint8_t* kflag, long long xp_rows, unsigned* status) {
  __shared__ int s_red[kPackThreads / 32];
  __shared__ int s_rows[32];
  __shared__ int s_n;
  __shared__ int s_before;
  pdl_wait();
  pdl_launch_dependents();
  const int b = b0 + blockIdx.x;
  const int j0 = blockIdx.y * 32;
  const uint8_t* mrow = io->mask + (long long)b * S;
  // valid tokens before this chunk
  int c = 0;
  for (int j = threadIdx.x; j < j0; j += kPackThreads) c += mrow[j] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x < 32) {
    int before = 0;
    for (int w = 0; w < kPackThreads / 32; ++w) before += s_red[w];
    const int j = j0 + threadIdx.x;
    const int valid = (j < S) ? (mrow[j] != 0) : 0;
    const unsigned bal = __ballot_sync(0xffffffffu, valid);
    const int rank = __popc(bal & ((1u << threadIdx.x) - 1u));
    if (valid) s_rows[rank] = j;
    if (threadIdx.x == 0) {
      s_n = __popc(bal);
      s_before = before;
    }
  }
  __syncthreads();
  const int n = s_n;
  const long long dst0 = (long long)vofs[b] + s_before;
  if (!checked_in_range(dst0, 0, xp_rows - n + 1, status)) return;   // rows dst0 .. dst0 + n - 1 inside xp
  // image flag of every packed token (the image/text split of the cross layers)
  if ((int)threadIdx.x < n)
    kflag[dst0 + threadIdx.x] =
        io->image_mask != nullptr ? (uint8_t)(io->image_mask[(long long)b * S + s_rows[threadIdx.x]] != 0) : 0;
  const int vec_per_row = Dvl / 8;            // 8 bf16 = 16 bytes
  for (int idx = threadIdx.x; idx < n * vec_per_row; idx += kPackThreads) {
    const int r = idx / vec_per_row;
    const int v = idx - r * vec_per_row;
    const long long src_row = (long long)b * S + s_rows[r];
    uint4 out;
    if (bb_bf16) {
      out = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(io->feats) + src_row * Dvl)[v];
    } else {
      const float4* f = reinterpret_cast<const float4*>(static_cast<const float*>(io->feats) + src_row * Dvl) + 2 * v;
      const float4 x0 = f[0], x1 = f[1];
      out.x = pack_bf16x2(x0.x, x0.y);
      out.y = pack_bf16x2(x0.z, x0.w);
      out.z = pack_bf16x2(x1.x, x1.y);
      out.w = pack_bf16x2(x1.z, x1.w);
    }
    reinterpret_cast<uint4*>(xp + (dst0 + r) * Dvl)[v] = out;
  }
}

// x (f32) and its bf16 copy from init_noise, bf16 state rows, all in sorted order.
__global__ void gather_inputs_kernel(const IoPtrs* io, int B, int HA, int Sd, const int* perm, float* x,
                                     __nv_bfloat16* xb, __nv_bfloat16* sb, unsigned* status) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x;
  const int b = perm[i];
  if (!checked_in_range(b, 0, B, status)) return;
  for (int e = threadIdx.x; e < HA; e += blockDim.x) {
    const float v = io->noise[(long long)b * HA + e];
    x[(long long)i * HA + e] = v;
    xb[(long long)i * HA + e] = __float2bfloat16_rn(v);
  }
  for (int e = threadIdx.x; e < Sd; e += blockDim.x)
    sb[(long long)i * Sd + e] = __float2bfloat16_rn(io->state[(long long)b * Sd + e]);
}

// out_actions[perm[i]] = x[i]; NaN for a sample whose embodiment id was invalid.
__global__ void scatter_out_kernel(const IoPtrs* io, int HA, const int* perm, const uint8_t* bad, const float* x,
                                   unsigned* status) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x;
  const int b = perm[i];
  if (!checked_in_range(b, 0, (long long)gridDim.x, status)) return;
  const bool nan_out = bad[b] != 0;
  for (int e = threadIdx.x; e < HA; e += blockDim.x)
    io->out[(long long)b * HA + e] = nan_out ? __int_as_float(0x7fc00000) : x[(long long)i * HA + e];
}

// ---------------------------------------------------------------- LayerNorm
//
// One warp per row of the f32 residual stream h [rows, D]; D = 128 * VEC.
//   mode 0 (AdaLN, "Transformer block structure": norm1(hidden_states, temb)):
//     u = LN(h) * (1 + p0) + p1      with p0 = scale, p1 = shift of this step/layer
//   mode 1 (affine norm3):  u = LN(h) * p0 + p1
// LN has no affine of its own, biased variance (two passes in registers).
// If restore != nullptr, rows r with r % period == 0 (the state token of each
// sample) are first reset from restore[r / period] and written back to h: the
// state features re-enter every Euler step.
// Vision-language layer norm of the packed backbone tokens, in place: one warp
// per packed row of Dvl = 256 * VEC bf16 features, f32 mean and (two-pass)
// variance in registers, y = (x - mean) * rstd * g + b rounded to bf16.  Rows
// past the call's valid-token count (vofs[B], on the device) are left alone.
template <int VEC>
__global__ void __launch_bounds__(256)
    vlln_kernel(__nv_bfloat16* xp, const int* total, const float* g, const float* b, float eps) {
  constexpr int Dvl = 256 * VEC;
  pdl_wait();
  pdl_launch_dependents();
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= *total) return;
  uint4* xr = reinterpret_cast<uint4*>(xp + row * Dvl);
  float v[8 * VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    const uint4 u = xr[lane + 32 * i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
      v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 8 * VEC; ++i) s += v[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s * (1.0f / Dvl);
  float q = 0.0f;
#pragma unroll
  for (int i = 0; i < 8 * VEC; ++i) q += (v[i] - mean) * (v[i] - mean);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q * (1.0f / Dvl) + eps);
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    const int c0 = (lane + 32 * i) * 8;
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(g + c0)), g1 = __ldg(reinterpret_cast<const float4*>(g + c0 + 4));
    const float4 b0 = __ldg(reinterpret_cast<const float4*>(b + c0)), b1 = __ldg(reinterpret_cast<const float4*>(b + c0 + 4));
    const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = pack_bf16x2((v[8 * i + 2 * j] - mean) * rstd * gg[2 * j] + bb[2 * j],
                         (v[8 * i + 2 * j + 1] - mean) * rstd * gg[2 * j + 1] + bb[2 * j + 1]);
    xr[lane + 32 * i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int VEC>
__global__ void __launch_bounds__(256)
    layernorm_kernel(float* h, int rows, const float* p0, const float* p1, int mode, float eps,
                     __nv_bfloat16* u, const float* restore, int period) {
  constexpr int D = 128 * VEC;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  // The modulation vectors are tables no earlier kernel writes: staged once
  // per CTA in shared memory before waiting for the previous kernel, so their
  // latency overlaps its tail (and they cost no registers: more CTAs per SM).
  __shared__ float4 sp[2][D / 4];
  for (int i = threadIdx.x; i < D / 4; i += blockDim.x) {
    sp[0][i] = __ldg(reinterpret_cast<const float4*>(p0) + i);
    sp[1][i] = __ldg(reinterpret_cast<const float4*>(p1) + i);
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  if (row >= rows) return;
  float4 x[VEC];
  float* hr = h + (long long)row * D;
  const bool from_restore = restore != nullptr && (row % period) == 0;
  const float* src = from_restore ? restore + (long long)(row / period) * D : hr;
#pragma unroll
  for (int i = 0; i < VEC; ++i) x[i] = reinterpret_cast<const float4*>(src)[lane + 32 * i];
  if (from_restore) {
#pragma unroll
    for (int i = 0; i < VEC; ++i) reinterpret_cast<float4*>(hr)[lane + 32 * i] = x[i];
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < VEC; ++i) s += (x[i].x + x[i].y) + (x[i].z + x[i].w);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s * (1.0f / D);
  float q = 0.0f;
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    const float a = x[i].x - mean, b = x[i].y - mean, c = x[i].z - mean, d = x[i].w - mean;
    q += (a * a + b * b) + (c * c + d * d);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q * (1.0f / D) + eps);
  __nv_bfloat16* ur = u + (long long)row * D;
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    const int c4 = lane + 32 * i;
    const float4 a = sp[0][c4], b = sp[1][c4];
    float4 y;
    y.x = (x[i].x - mean) * rstd;
    y.y = (x[i].y - mean) * rstd;
    y.z = (x[i].z - mean) * rstd;
    y.w = (x[i].w - mean) * rstd;
    if (mode == 0) {
      y.x = y.x * (1.0f + a.x) + b.x;
      y.y = y.y * (1.0f + a.y) + b.y;
      y.z = y.z * (1.0f + a.z) + b.z;
      y.w = y.w * (1.0f + a.w) + b.w;
    } else {
      y.x = y.x * a.x + b.x;
      y.y = y.y * a.y + b.y;
      y.z = y.z * a.z + b.z;
      y.w = y.w * a.w + b.w;
    }
    uint2 w;
    w.x = pack_bf16x2(y.x, y.y);
    w.y = pack_bf16x2(y.z, y.w);
    reinterpret_cast<uint2*>(ur)[c4] = w;
  }
}

// ---------------------------------------------------------------- timestep tables
//
// phi[k][j] = sinusoidal encoding of the discretised timestep td[k]
// (first half sin(td * w_i), second half cos(td * w_i), w_i = 10000^(-i/(n/2))),
// evaluated in double precision.
__global__ void sinusoid_kernel(const float* td, int K, int n, float* phi) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= K * n) return;
  const int k = idx / n, j = idx - k * n;
  const int half = n / 2;
  const int i = j < half ? j : j - half;
  const double w = exp(-(double)i / (double)half * log(10000.0));
  const double arg = (double)td[k] * w;
  phi[idx] = (float)(j < half ? sin(arg) : cos(arg));
}

// y[k][r] = act_out( W[r, :] . act_in(x[k, :]) + bias[r] ) for k < K, r < R.
// W bf16 [R, In] row-major; one warp per output row (the row is read once
// into registers in slices and applied to all K inputs).
__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

__global__ void __launch_bounds__(256)
    gemv_rows_kernel(const __nv_bfloat16* W, int R, int In, const float* x, int K, const float* bias, int in_silu,
                     int out_silu, float* y, long long y_ld) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const __nv_bfloat16* wr = W + (long long)r * In;
  for (int k = 0; k < K; ++k) {
    const float* xk = x + (long long)k * In;
    float acc = 0.0f;
    for (int j = lane; j < In; j += 32) {
      float xv = xk[j];
      if (in_silu) xv = silu_f(xv);
      acc += __bfloat162float(wr[j]) * xv;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      float v = acc + (bias ? bias[r] : 0.0f);
      if (out_silu) v = silu_f(v);
      y[(long long)k * y_ld + r] = v;
    }
  }
}

}  // namespace gdit
