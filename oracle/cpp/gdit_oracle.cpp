// Plain C++ CPU oracle of the GR00T N1.6 flow-matching action head, in float
// and in double (one template, two instantiations).
//
// TEST INFRASTRUCTURE ONLY.  It is called by the tests (through
// oracle/cpp_oracle.py) and by the benchmark's CPU-baseline leg.  It shares no
// code with the GPU library or with the numpy oracle: it is a second, separate
// restatement of the same pages, written as naive loops.
//
// Sources (page, then section):
//   ARCH  Isaac-GR00T "Model architecture": "Action head architecture",
//         "Diffusion transformer (DiT)" (Architecture details, Transformer block
//         structure, AlternateVLDiT variant), "Flow matching diffusion"
//         (Inference (denoising)), "Embodiment-specific projectors"
//         (CategorySpecificLinear, Multi-embodiment action encoder).
//   MODEL Isaac-GR00T "GR00T model class": num_timestep_buckets.
//
// Readings where the pages are silent (the same ones the numpy oracle takes):
// sinusoid = [sin | cos] halves with frequencies 10000^(-i/(n/2)) evaluated at
// the discretised timestep floor(1000 k / K); TimestepEncoder = Linear, SiLU,
// Linear; AdaLN = LayerNorm without affine, (scale, shift) = chunk of
// Linear(SiLU(temb)), out = LN(h) (1 + scale) + shift; norm3 = affine
// LayerNorm; exact (erf) GELU; ReLU inside CategorySpecificMLP; swish after the
// action encoder's W2; the state token first, its decoded row dropped; a
// query with no key gets a zero attention output.  Not covered here: the
// image/text split of the cross layers and the optional vision-language
// LayerNorm (the numpy oracle covers both).
//
// Layouts: plain linears [out, in] (y = x W^T + b); category linears
// [C, in, out] (y = x W[c] + b[c]); activations row-major.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

typedef struct {
  int num_layers, hidden, num_heads, head_dim, mlp_hidden, backbone_dim;
  int action_dim, state_dim, action_horizon, num_embodiments;
  int time_freq_dim, num_timestep_buckets;
  double ln_eps;
} oracle_geom;

}  // extern "C"

namespace {

template <typename T>
struct Weights {
  const T *t1w, *t1b, *t2w, *t2b;
  struct Block {
    const T *adaw, *adab, *qw, *qb, *kw, *kb, *vw, *vb, *ow, *ob, *g3, *b3, *f1w, *f1b, *f2w, *f2b;
  };
  std::vector<Block> blk;
  const T *oadaw, *oadab, *projw, *projb;
  const T *s1W, *s1b, *s2W, *s2b;       // state encoder
  const T *a1W, *a1b, *a2W, *a2b, *a3W, *a3b;   // action encoder
  const T *d1W, *d1b, *d2W, *d2b;       // action decoder
};

// The weight table in its canonical order (the order of the header comment of
// oracle/cpp_oracle.py): 4 timestep-encoder tensors, 16 per block, 4 of the
// output layer, then the 14 category tensors.
template <typename T>
bool bind(const oracle_geom& g, const T* const* w, int n, Weights<T>& W) {
  const int want = 4 + 16 * g.num_layers + 4 + 14;
  if (n != want) return false;
  int i = 0;
  W.t1w = w[i++]; W.t1b = w[i++]; W.t2w = w[i++]; W.t2b = w[i++];
  W.blk.resize(g.num_layers);
  for (auto& b : W.blk) {
    b.adaw = w[i++]; b.adab = w[i++]; b.qw = w[i++]; b.qb = w[i++]; b.kw = w[i++]; b.kb = w[i++];
    b.vw = w[i++]; b.vb = w[i++]; b.ow = w[i++]; b.ob = w[i++]; b.g3 = w[i++]; b.b3 = w[i++];
    b.f1w = w[i++]; b.f1b = w[i++]; b.f2w = w[i++]; b.f2b = w[i++];
  }
  W.oadaw = w[i++]; W.oadab = w[i++]; W.projw = w[i++]; W.projb = w[i++];
  W.s1W = w[i++]; W.s1b = w[i++]; W.s2W = w[i++]; W.s2b = w[i++];
  W.a1W = w[i++]; W.a1b = w[i++]; W.a2W = w[i++]; W.a2b = w[i++]; W.a3W = w[i++]; W.a3b = w[i++];
  W.d1W = w[i++]; W.d1b = w[i++]; W.d2W = w[i++]; W.d2b = w[i++];
  return i == want;
}

template <typename T>
using Mat = std::vector<T>;   // row-major [rows, cols]

// nn.Linear: y[r, o] = b[o] + sum_i x[r, i] W[o, i]   (W stored [out, in])
template <typename T>
Mat<T> linear(const Mat<T>& x, int rows, int in, const T* W, const T* b, int out) {
  Mat<T> y((size_t)rows * out);
#pragma omp parallel for if (!omp_in_parallel() && (long long)rows * out * in > (1 << 18)) schedule(static)
  for (int o = 0; o < out; ++o)
    for (int r = 0; r < rows; ++r) {
      T acc = b[o];
      const T* xr = &x[(size_t)r * in];
      const T* wo = W + (size_t)o * in;
      for (int i = 0; i < in; ++i) acc += xr[i] * wo[i];
      y[(size_t)r * out + o] = acc;
    }
  return y;
}

// CategorySpecificLinear (ARCH "CategorySpecificLinear"): y = x W[c] + b[c]
// with W [C, in, out], b [C, out].
template <typename T>
Mat<T> cat_linear(const Mat<T>& x, int rows, int in, const T* W, const T* b, int out, int c) {
  const T* Wc = W + (size_t)c * in * out;
  const T* bc = b + (size_t)c * out;
  Mat<T> y((size_t)rows * out);
#pragma omp parallel for if (!omp_in_parallel() && (long long)rows * out * in > (1 << 18)) schedule(static)
  for (int r = 0; r < rows; ++r) {
    T* yr = &y[(size_t)r * out];
    for (int o = 0; o < out; ++o) yr[o] = bc[o];
    for (int i = 0; i < in; ++i) {
      const T xi = x[(size_t)r * in + i];
      const T* wi = Wc + (size_t)i * out;
      for (int o = 0; o < out; ++o) yr[o] += xi * wi[o];
    }
  }
  return y;
}

// LayerNorm over each row, biased variance (two passes); optional affine.
template <typename T>
Mat<T> layer_norm(const Mat<T>& x, int rows, int n, T eps, const T* gamma, const T* beta) {
  Mat<T> y(x.size());
  for (int r = 0; r < rows; ++r) {
    const T* xr = &x[(size_t)r * n];
    T mean = 0;
    for (int i = 0; i < n; ++i) mean += xr[i];
    mean /= (T)n;
    T var = 0;
    for (int i = 0; i < n; ++i) var += (xr[i] - mean) * (xr[i] - mean);
    var /= (T)n;
    const T inv = (T)1 / std::sqrt(var + eps);
    for (int i = 0; i < n; ++i) {
      T v = (xr[i] - mean) * inv;
      if (gamma != nullptr) v = v * gamma[i] + beta[i];
      y[(size_t)r * n + i] = v;
    }
  }
  return y;
}

template <typename T>
T silu(T x) { return x / ((T)1 + std::exp(-x)); }

template <typename T>
T gelu(T x) { return (T)0.5 * x * ((T)1 + std::erf(x / std::sqrt((T)2))); }

// phi_n(p): [sin(p w_0) .. sin(p w_{n/2-1}) | cos(p w_0) .. cos(p w_{n/2-1})],
// w_i = 10000^(-i / (n/2)); computed in double.
template <typename T>
std::vector<T> sinusoid(double p, int n) {
  const int half = n / 2;
  std::vector<T> e(n);
  for (int i = 0; i < half; ++i) {
    const double w = std::pow(10000.0, -(double)i / (double)half);
    e[i] = (T)std::sin(p * w);
    e[half + i] = (T)std::cos(p * w);
  }
  return e;
}

// AdaLayerNorm: (scale, shift) = chunk(Linear(SiLU(temb)), 2), scale first;
// out = LN(h) (1 + scale) + shift.
template <typename T>
Mat<T> ada_ln(const Mat<T>& h, int rows, int D, const std::vector<T>& temb, const T* w, const T* b, T eps) {
  Mat<T> s(D);
  for (int i = 0; i < D; ++i) s[i] = silu(temb[i]);
  const Mat<T> emb = linear(s, 1, D, w, b, 2 * D);
  Mat<T> y = layer_norm(h, rows, D, eps, (const T*)nullptr, (const T*)nullptr);
  for (int r = 0; r < rows; ++r)
    for (int i = 0; i < D; ++i) y[(size_t)r * D + i] = y[(size_t)r * D + i] * ((T)1 + emb[i]) + emb[D + i];
  return y;
}

// Multi-head attention of one sample: q [nq, D], k and v [nk, D] (only the
// keys the sample attends to); per head softmax(q_h k_h^T / sqrt(dh)) v_h.
template <typename T>
Mat<T> attention(const Mat<T>& q, int nq, const Mat<T>& k, const Mat<T>& v, int nk, int nh, int dh) {
  const int D = nh * dh;
  Mat<T> out((size_t)nq * D, (T)0);
  if (nk == 0) return out;
  std::vector<T> s(nk);
  const T scale = (T)1 / std::sqrt((T)dh);
  for (int h = 0; h < nh; ++h)
    for (int i = 0; i < nq; ++i) {
      T m = -INFINITY;
      for (int j = 0; j < nk; ++j) {
        T acc = 0;
        for (int d = 0; d < dh; ++d) acc += q[(size_t)i * D + h * dh + d] * k[(size_t)j * D + h * dh + d];
        s[j] = acc * scale;
        if (s[j] > m) m = s[j];
      }
      T sum = 0;
      for (int j = 0; j < nk; ++j) {
        s[j] = std::exp(s[j] - m);
        sum += s[j];
      }
      for (int d = 0; d < dh; ++d) {
        T acc = 0;
        for (int j = 0; j < nk; ++j) acc += s[j] * v[(size_t)j * D + h * dh + d];
        out[(size_t)i * D + h * dh + d] = acc / sum;
      }
    }
  return out;
}

// One sample: K Euler steps of x <- x + (1/K) v(x, t_k) (ARCH "Inference
// (denoising)").
template <typename T>
void one_sample(const oracle_geom& g, const Weights<T>& W, const T* feats, const uint8_t* mask, const T* state,
                int c, const T* noise, int S, int K, T* out) {
  const int D = g.hidden, F = g.mlp_hidden, A = g.action_dim, H = g.action_horizon, N = H + 1;
  const int Dvl = g.backbone_dim, Sd = g.state_dim, L = g.num_layers, nh = g.num_heads, dh = g.head_dim;
  const T eps = (T)g.ln_eps;
  // valid backbone tokens (mask == 1) and every cross layer's K/V over them
  std::vector<int> valid;
  for (int j = 0; j < S; ++j)
    if (mask[j]) valid.push_back(j);
  const int nv = (int)valid.size();
  Mat<T> X((size_t)nv * Dvl);
  for (int r = 0; r < nv; ++r)
    std::memcpy(&X[(size_t)r * Dvl], feats + (size_t)valid[r] * Dvl, sizeof(T) * Dvl);
  std::vector<Mat<T>> Kc(L), Vc(L);
  for (int l = 0; l < L; l += 2) {
    Kc[l] = linear(X, nv, Dvl, W.blk[l].kw, W.blk[l].kb, D);
    Vc[l] = linear(X, nv, Dvl, W.blk[l].vw, W.blk[l].vb, D);
  }
  // state encoder: ReLU(state W1[c] + b1[c]) W2[c] + b2[c]
  Mat<T> st(state, state + Sd);
  Mat<T> s1 = cat_linear(st, 1, Sd, W.s1W, W.s1b, D, c);
  for (auto& v : s1) v = v > (T)0 ? v : (T)0;
  const Mat<T> sfeat = cat_linear(s1, 1, D, W.s2W, W.s2b, D, c);

  Mat<T> x(noise, noise + (size_t)H * A);
  const T dt = (T)1 / (T)K;
  for (int k = 0; k < K; ++k) {
    const double td = std::floor((double)k / (double)K * (double)g.num_timestep_buckets);
    // TimestepEncoder: L2(SiLU(L1(phi_256(td))))
    const std::vector<T> ph = sinusoid<T>(td, g.time_freq_dim);
    Mat<T> t1 = linear(Mat<T>(ph.begin(), ph.end()), 1, g.time_freq_dim, W.t1w, W.t1b, D);
    for (auto& v : t1) v = silu(v);
    const Mat<T> temb = linear(t1, 1, D, W.t2w, W.t2b, D);
    // action encoder: a = x W1[c] + b1; z = swish([a, tau] W2[c] + b2); e = z W3[c] + b3
    const Mat<T> a = cat_linear(x, H, A, W.a1W, W.a1b, D, c);
    const std::vector<T> tau = sinusoid<T>(td, D);
    Mat<T> at((size_t)H * 2 * D);
    for (int r = 0; r < H; ++r)
      for (int i = 0; i < D; ++i) {
        at[(size_t)r * 2 * D + i] = a[(size_t)r * D + i];
        at[(size_t)r * 2 * D + D + i] = tau[i];
      }
    Mat<T> z = cat_linear(at, H, 2 * D, W.a2W, W.a2b, D, c);
    for (auto& v : z) v = silu(v);
    const Mat<T> e = cat_linear(z, H, D, W.a3W, W.a3b, D, c);
    // h = [state features ; action features]
    Mat<T> h((size_t)N * D);
    for (int i = 0; i < D; ++i) h[i] = sfeat[i];
    for (int r = 0; r < H; ++r)
      for (int i = 0; i < D; ++i) h[(size_t)(r + 1) * D + i] = e[(size_t)r * D + i];
    // 32 blocks: even layers cross-attend to the backbone, odd layers self-attend
    for (int l = 0; l < L; ++l) {
      const auto& B = W.blk[l];
      const Mat<T> u = ada_ln(h, N, D, temb, B.adaw, B.adab, eps);
      const Mat<T> q = linear(u, N, D, B.qw, B.qb, D);
      Mat<T> att;
      if (l % 2 == 1) {
        const Mat<T> ks = linear(u, N, D, B.kw, B.kb, D);
        const Mat<T> vs = linear(u, N, D, B.vw, B.vb, D);
        att = attention(q, N, ks, vs, N, nh, dh);
      } else {
        att = attention(q, N, Kc[l], Vc[l], nv, nh, dh);
      }
      const Mat<T> o = linear(att, N, D, B.ow, B.ob, D);
      for (size_t i = 0; i < h.size(); ++i) h[i] += o[i];
      const Mat<T> n3 = layer_norm(h, N, D, eps, B.g3, B.b3);
      Mat<T> f = linear(n3, N, D, B.f1w, B.f1b, F);
      for (auto& v : f) v = gelu(v);
      const Mat<T> f2 = linear(f, N, F, B.f2w, B.f2b, D);
      for (size_t i = 0; i < h.size(); ++i) h[i] += f2[i];
    }
    // output AdaLN + proj_out, then the decoder on the action rows (row 0 dropped)
    const Mat<T> y = linear(ada_ln(h, N, D, temb, W.oadaw, W.oadab, eps), N, D, W.projw, W.projb, D);
    const Mat<T> ya(y.begin() + D, y.end());
    Mat<T> r1 = cat_linear(ya, H, D, W.d1W, W.d1b, D, c);
    for (auto& v : r1) v = v > (T)0 ? v : (T)0;
    const Mat<T> vel = cat_linear(r1, H, D, W.d2W, W.d2b, A, c);
    for (size_t i = 0; i < x.size(); ++i) x[i] += dt * vel[i];
  }
  std::memcpy(out, x.data(), sizeof(T) * x.size());
}

template <typename T>
int get_action(const oracle_geom* g, const T* const* w, int n_w, const T* feats, const uint8_t* mask,
               const T* state, const int32_t* ids, const T* noise, int B, int S, int K, int threads, T* out) {
  if (g == nullptr || w == nullptr || K < 1 || B < 1 || S < 0) return -1;
  if (g->hidden != g->num_heads * g->head_dim || g->num_layers % 2 != 0) return -1;
  Weights<T> W;
  if (!bind(*g, w, n_w, W)) return -1;
  for (int b = 0; b < B; ++b)
    if (ids[b] < 0 || ids[b] >= g->num_embodiments) return -2;
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#else
  (void)threads;
#endif
  const size_t fs = (size_t)S * g->backbone_dim, xs = (size_t)g->action_horizon * g->action_dim;
  // samples are independent: one thread per sample when there are at least
  // as many samples as threads; otherwise the samples run one after the other
  // and each linear parallelises over its outputs
#ifdef _OPENMP
  const bool by_sample = B > 1 && B >= omp_get_max_threads();
#else
  const bool by_sample = false;
#endif
#pragma omp parallel for schedule(dynamic, 1) if (by_sample)
  for (int b = 0; b < B; ++b)
    one_sample(*g, W, feats + b * fs, mask + (size_t)b * S, state + (size_t)b * g->state_dim, ids[b],
               noise + b * xs, S, K, out + b * xs);
  return 0;
}

}  // namespace

extern "C" {

int oracle_get_action_f64(const oracle_geom* g, const double* const* w, int n_w, const double* feats,
                          const uint8_t* mask, const double* state, const int32_t* ids, const double* noise, int B,
                          int S, int K, int threads, double* out) {
  return get_action<double>(g, w, n_w, feats, mask, state, ids, noise, B, S, K, threads, out);
}

int oracle_get_action_f32(const oracle_geom* g, const float* const* w, int n_w, const float* feats,
                          const uint8_t* mask, const float* state, const int32_t* ids, const float* noise, int B,
                          int S, int K, int threads, float* out) {
  return get_action<float>(g, w, n_w, feats, mask, state, ids, noise, B, S, K, threads, out);
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
