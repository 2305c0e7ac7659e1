"""Plain fp64 CPU oracle of the GR00T N1.6 flow-matching action head.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The GPU library never
calls it and shares no code with it; the two meet only in the seeded inputs of
``synth``.

It is written for a reader who checks it against the pages by eye: each step is
one numpy expression in float64, every sample is run on its own, and no step is
fused, blocked or reordered.  Matrix products use numpy's matmul (a library
primitive); everything else is written out.

Sources (page, then section):
  [ARCH]   nvidia-isaac-gr00t.mintlify.app/architecture.md (Isaac-GR00T "Model
           architecture"): "Action head architecture", "Diffusion transformer
           (DiT)" (Architecture details, Transformer block structure,
           AlternateVLDiT variant), "Flow matching diffusion" (Inference
           (denoising)), "Embodiment-specific projectors" (CategorySpecificLinear,
           Multi-embodiment action encoder).
  [MODEL]  nvidia-isaac-gr00t.mintlify.app/api/model/gr00t-model.md ("GR00T model
           class"): get_action, "Flow matching diffusion" config
           (num_inference_timesteps, num_timestep_buckets).
  [WS1]    phyai.mintlify.app/models/gr00t/ws1.md ("Single-GPU inference for
           GR00T-N1.7"): Overview (embodiment id routes the encoders/decoder) and
           the request path.

Where the pages are silent the plainest reading is taken; each such reading is
marked READING below.

Parity pins: every function here is pinned by ``tests/test_oracle_*.py`` to
closed forms, invariants, library routines (torch LayerNorm / GELU / SDPA /
linear / bmm) or brute force.  One thing is "parity unpinned": agreement with
real GR00T checkpoints, since no weights or example outputs are available.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
from scipy.special import erf as _erf


# --------------------------------------------------------------------------
# input decoding
# --------------------------------------------------------------------------

def to_f64(a) -> np.ndarray:
    """float64 copy of an input array; uint16 arrays hold bf16 bit patterns."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# --------------------------------------------------------------------------
# elementary functions
# --------------------------------------------------------------------------

def sinusoidal_embedding(p, n: int) -> np.ndarray:
    """phi_n(p): sinusoidal encoding of a (discretised) timestep p.

    [ARCH] "Action head architecture" (action encoder uses sinusoidal encoding of
    diffusion timesteps) and "Architecture details" (TimestepEncoder "using
    sinusoidal embeddings").  READING: first half sin(p*w_i), second half
    cos(p*w_i), w_i = 10000^(-i/(n/2)), i = 0..n/2-1, evaluated at the
    discretised timestep (0..999), not at t in [0, 1].
    """
    half = n // 2
    i = np.arange(half, dtype=np.float64)
    w = np.power(10000.0, -i / half)
    arg = np.asarray(p, dtype=np.float64)[..., None] * w
    return np.concatenate([np.sin(arg), np.cos(arg)], axis=-1)


def euler_schedule(num_steps: int, buckets: int = 1000) -> Tuple[List[float], List[float], float]:
    """(t_k, t_discretized_k, dt) of the K-step Euler loop.

    [ARCH] "Inference (denoising)": dt = 1/K, t_cont = k/K for k = 0..K-1.
    [MODEL] "Flow matching diffusion": num_timestep_buckets = 1000.  READING:
    t_discretized = floor(t_cont * buckets), computed in IEEE double.
    """
    t = [k / num_steps for k in range(num_steps)]
    td = [float(math.floor(tk * buckets)) for tk in t]
    return t, td, 1.0 / num_steps


def linear(x: np.ndarray, w: np.ndarray, b: np.ndarray) -> np.ndarray:
    """PyTorch nn.Linear: y = x W^T + b with W stored [out, in]."""
    return x @ w.T + b


def category_linear(x: np.ndarray, W: np.ndarray, b: np.ndarray, c: int) -> np.ndarray:
    """CategorySpecificLinear for one sample of category c.

    [ARCH] "CategorySpecificLinear": W is [num_categories, in, out], b is
    [num_categories, out]; the forward selects W[c], b[c] and computes
    x @ W[c] + b[c] (a batched matmul over samples, one category each).
    """
    return x @ W[c] + b[c]


def layer_norm(x: np.ndarray, eps: float, gamma=None, beta=None) -> np.ndarray:
    """LayerNorm over the last axis with biased variance; optional affine."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * gamma + beta
    return y


def silu(x: np.ndarray) -> np.ndarray:
    """x * sigmoid(x) (also called swish, [ARCH] action encoder)."""
    return x / (1.0 + np.exp(-x))


swish = silu


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU x * Phi(x) ([ARCH] "Transformer block structure": MLP with GELU).
    READING: the erf form, not the tanh approximation."""
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def relu(x: np.ndarray) -> np.ndarray:
    return np.maximum(x, 0.0)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, num_heads: int,
              return_probs: bool = False):
    """Multi-head scaled dot-product attention of one sample.

    q [Nq, nh*dh]; k, v [Nk, nh*dh] hold only the keys the sample may attend to.
    Per head: P = softmax(q_h k_h^T / sqrt(dh)) over keys, out_h = P v_h; heads
    are concatenated.  READING: a query with no key to attend to gets a zero
    output (before the output projection).
    """
    nq, width = q.shape
    dh = width // num_heads
    out = np.zeros((nq, width), dtype=np.float64)
    probs = []
    if k.shape[0] == 0:
        return (out, probs) if return_probs else out
    for h in range(num_heads):
        cols = slice(h * dh, (h + 1) * dh)
        s = (q[:, cols] @ k[:, cols].T) / math.sqrt(dh)
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        p = e / e.sum(axis=1, keepdims=True)
        out[:, cols] = p @ v[:, cols]
        probs.append(p)
    return (out, probs) if return_probs else out


# --------------------------------------------------------------------------
# model pieces
# --------------------------------------------------------------------------

class Model:
    """float64 view of a weight table (see ``synth.weight_shapes`` for names).

    Converted tensors are cached; category-specific tensors are converted one
    category at a time.
    """

    def __init__(self, weights: Dict[str, np.ndarray], geom):
        self.w = weights
        self.g = geom
        self._cache: Dict[str, np.ndarray] = {}
        self._cat_cache: Dict[Tuple[str, int], np.ndarray] = {}

    def __getitem__(self, name: str) -> np.ndarray:
        a = self._cache.get(name)
        if a is None:
            a = to_f64(self.w[name])
            self._cache[name] = a
        return a

    def cat(self, name: str, c: int) -> np.ndarray:
        key = (name, c)
        a = self._cat_cache.get(key)
        if a is None:
            a = to_f64(np.asarray(self.w[name])[c])
            self._cat_cache[key] = a
        return a


def category_mlp(m: Model, prefix: str, x: np.ndarray, c: int) -> np.ndarray:
    """CategorySpecificMLP: layer2(ReLU(layer1(x))), both category-specific.

    [ARCH] "Action head architecture" (state_encoder / action_decoder are
    CategorySpecificMLP).  READING: ReLU between the two layers.
    """
    h = relu(x @ m.cat(prefix + ".l1.W", c) + m.cat(prefix + ".l1.b", c))
    return h @ m.cat(prefix + ".l2.W", c) + m.cat(prefix + ".l2.b", c)


def state_encoder(m: Model, state: np.ndarray, c: int) -> np.ndarray:
    """state [T_s, Sd] -> state features [T_s, D] ([ARCH] state_encoder)."""
    return category_mlp(m, "state_enc", state, c)


def action_encoder(m: Model, actions: np.ndarray, td: float, c: int) -> np.ndarray:
    """MultiEmbodimentActionEncoder for one sample.

    [ARCH] "Multi-embodiment action encoder": a = W1(actions); tau = sinusoidal
    encoding of the timestep, the same for every action token; x = [a, tau]
    (concatenated along features, a first); x = swish(W2(x)); return W3(x).
    """
    D = m.g.hidden
    a = actions @ m.cat("act_enc.W1.W", c) + m.cat("act_enc.W1.b", c)
    tau = np.broadcast_to(sinusoidal_embedding(td, D), a.shape)
    x = np.concatenate([a, tau], axis=-1)
    x = swish(x @ m.cat("act_enc.W2.W", c) + m.cat("act_enc.W2.b", c))
    return x @ m.cat("act_enc.W3.W", c) + m.cat("act_enc.W3.b", c)


def action_decoder(m: Model, y: np.ndarray, c: int) -> np.ndarray:
    """[ARCH] action_decoder: CategorySpecificMLP hidden -> hidden -> action_dim."""
    return category_mlp(m, "act_dec", y, c)


def timestep_embedding(m: Model, td: float) -> np.ndarray:
    """DiT TimestepEncoder: temb = L2(SiLU(L1(phi_256(td)))) ([ARCH] "Architecture
    details").  READING: Linear -> SiLU -> Linear, width time_freq_dim -> D -> D."""
    e = sinusoidal_embedding(td, m.g.time_freq_dim)
    return linear(silu(linear(e, m["t_enc.l1.w"], m["t_enc.l1.b"])), m["t_enc.l2.w"], m["t_enc.l2.b"])


def ada_layer_norm(h: np.ndarray, temb: np.ndarray, w: np.ndarray, b: np.ndarray,
                   eps: float) -> np.ndarray:
    """AdaLayerNorm (norm_type="ada_norm", [ARCH] "Transformer block structure":
    norm1(hidden_states, temb)).

    READING: (scale, shift) = chunk(Linear(SiLU(temb)), 2), scale first;
    out = LN(h) * (1 + scale) + shift with a LayerNorm without affine.
    """
    emb = linear(silu(temb), w, b)
    D = h.shape[-1]
    scale, shift = emb[:D], emb[D:]
    return layer_norm(h, eps) * (1.0 + scale) + shift


def cross_kv(m: Model, layer: int, feats_valid: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Keys and values of a cross-attention layer over the valid backbone tokens.

    [ARCH] "Transformer block structure" (attn1 with encoder_hidden_states) and
    "AlternateVLDiT variant" (the backbone attention mask selects the tokens).
    They depend only on the backbone features, so they are the same in every
    Euler step.
    """
    p = f"blk{layer}."
    return (linear(feats_valid, m[p + "k.w"], m[p + "k.b"]),
            linear(feats_valid, m[p + "v.w"], m[p + "v.b"]))


def dit_block(m: Model, layer: int, h: np.ndarray, temb: np.ndarray,
              kv: Optional[Tuple[np.ndarray, np.ndarray]]) -> np.ndarray:
    """One BasicTransformerBlock ([ARCH] "Transformer block structure").

    norm = AdaLN(h, temb); a = attention (self for odd layers: kv is None;
    cross to the backbone for even layers, per "AlternateVLDiT variant");
    h = h + O(a); h = h + FF(LN3(h)) with FF = Linear -> GELU -> Linear.
    READING: norm3 is an affine LayerNorm; the residual adds carry no gate.
    """
    g = m.g
    p = f"blk{layer}."
    u = ada_layer_norm(h, temb, m[p + "ada.w"], m[p + "ada.b"], g.ln_eps)
    q = linear(u, m[p + "q.w"], m[p + "q.b"])
    if kv is None:
        k = linear(u, m[p + "k.w"], m[p + "k.b"])
        v = linear(u, m[p + "v.w"], m[p + "v.b"])
    else:
        k, v = kv
    a = attention(q, k, v, g.num_heads)
    h = h + linear(a, m[p + "o.w"], m[p + "o.b"])
    f = gelu(linear(layer_norm(h, g.ln_eps, m[p + "ln3.g"], m[p + "ln3.b"]),
                    m[p + "ff1.w"], m[p + "ff1.b"]))
    return h + linear(f, m[p + "ff2.w"], m[p + "ff2.b"])


def dit(m: Model, h: np.ndarray, temb: np.ndarray, kvs: Dict[int, Tuple[np.ndarray, np.ndarray]]) -> np.ndarray:
    """AlternateVLDiT forward for one sample: layers 0..L-1, odd layers
    self-attention, even layers cross-attention ([ARCH] "AlternateVLDiT
    variant"), then the output AdaLN and proj_out (READING: the DiT's final
    layer maps hidden -> output_dim = hidden through an AdaLN modulated by temb
    and a Linear; [ARCH] "Architecture details" names output_dim)."""
    g = m.g
    for layer in range(g.num_layers):
        h = dit_block(m, layer, h, temb, None if layer % 2 == 1 else kvs[layer])
    y = ada_layer_norm(h, temb, m["out.ada.w"], m["out.ada.b"], g.ln_eps)
    return linear(y, m["out.proj.w"], m["out.proj.b"])


def velocity(m: Model, x: np.ndarray, td: float, state_feat: np.ndarray,
             kvs: Dict[int, Tuple[np.ndarray, np.ndarray]], c: int) -> np.ndarray:
    """One evaluation of the velocity field v(x, t) for one sample.

    [ARCH] "Inference (denoising)": encode the actions, concatenate state
    features first ("sa_embs = cat(state_features, action_features)"), run the
    DiT, decode.  READING: the decoder output of the state token is dropped; the
    H action tokens give the velocity [H, A].
    """
    temb = timestep_embedding(m, td)
    e = action_encoder(m, x, td, c)
    h = np.concatenate([state_feat, e], axis=0)
    y = dit(m, h, temb, kvs)
    v = action_decoder(m, y, c)
    return v[state_feat.shape[0]:]


def cross_key_mask(layer: int, mask: np.ndarray, image_mask, n: int) -> np.ndarray:
    """The backbone tokens cross layer `layer` attends to ([ARCH] "AlternateVLDiT
    variant").  Without the image/text split (n == 0, the task's workloads) it
    is every valid token (mask == 1).  With it, the page builds
    image = image_mask & mask and text = ~image_mask & mask once, and a cross
    block with index idx uses text when idx % (2 n) == 0, else image.
    READING: image_mask None means no token is an image token."""
    valid = np.asarray(mask).astype(bool)
    if n == 0:
        return valid
    img = np.zeros_like(valid) if image_mask is None else np.asarray(image_mask).astype(bool)
    if layer % (2 * n) == 0:
        return (~img) & valid
    return img & valid


def prepare_sample(m: Model, feats: np.ndarray, mask: np.ndarray, state: np.ndarray, c: int,
                   image_mask=None, n: int = 0):
    """Per-sample quantities that do not change across Euler steps: the state
    features and every cross layer's K/V over the tokens it attends to
    (``cross_key_mask``; [ARCH] backbone forward: attention_mask == 1)."""
    f = to_f64(feats)
    if "vlln.g" in m.w:
        # READING: the vision-language layer norm ([ARCH] config "tune_vlln":
        # a trainable LayerNorm of the action head) normalises every backbone
        # token's features, with its gain and bias, before the cross layers
        f = layer_norm(f, m.g.ln_eps, m["vlln.g"], m["vlln.b"])
    kvs = {layer: cross_kv(m, layer, f[cross_key_mask(layer, mask, image_mask, n)])
           for layer in range(0, m.g.num_layers, 2)}
    s = state_encoder(m, to_f64(state).reshape(-1, m.g.state_dim), c)
    return s, kvs


def get_action(weights: Dict[str, np.ndarray], geom, backbone_features, vl_mask, state,
               embodiment_id, init_noise, num_steps: int,
               samples: Optional[Sequence[int]] = None,
               model: Optional[Model] = None, image_mask=None) -> np.ndarray:
    """Flow-matching Euler inference ([ARCH] "Inference (denoising)").

    x = init_noise; for k = 0..K-1: x = x + dt * v(x, t_k); returns x [B, H, A]
    (float64).  ``samples`` restricts the run to those batch rows (samples are
    independent), returned in that order.  ``init_noise`` is an input, as in the
    request's optional noise field ([WS1] "Prepare a request": a fixed tensor
    gives deterministic regression checks).  ``image_mask`` [B, S] marks image
    tokens for the image/text split of the cross layers, which is on when
    ``geom.attend_text_every_n_blocks`` > 0 (``cross_key_mask``).
    """
    m = model if model is not None else Model(weights, geom)
    ids = np.asarray(embodiment_id).reshape(-1)
    rows = range(len(ids)) if samples is None else samples
    _, tds, dt = euler_schedule(num_steps, geom.num_timestep_buckets)
    outs = []
    for b in rows:
        c = int(ids[b])
        if not 0 <= c < geom.num_embodiments:
            raise ValueError(f"embodiment_id {c} out of range")
        n = int(getattr(geom, "attend_text_every_n_blocks", 0))
        s, kvs = prepare_sample(m, backbone_features[b], vl_mask[b], state[b], c,
                                None if image_mask is None else image_mask[b], n)
        x = to_f64(init_noise[b]).copy()
        for td in tds:
            x = x + dt * velocity(m, x, td, s, kvs, c)
        outs.append(x)
    return np.stack(outs)


def training_loss(weights: Dict[str, np.ndarray], geom, backbone_features, vl_mask, state, embodiment_id,
                  actions, noise, t, action_mask, model: Optional[Model] = None, image_mask=None):
    """Flow-matching training objective of the action head, forward only
    ([ARCH] "Flow matching diffusion", "Training objective").

    Per sample b with time t_b: x_t = (1 - t_b) noise_b + t_b actions_b; the
    target velocity is actions_b - noise_b; the prediction is the velocity
    field at x_t with t_discretized = floor(t_b * buckets) (as in inference).
    READING: t is an input (the page samples it from Beta(1.5, 1); the random
    draw is passed in).  READING: the loss is the masked mean of the
    element-wise squared error, sum(mask * (pred - v)^2) / (sum(mask) + 1e-6)
    (the printed code multiplies a mean-reduced mse_loss by the mask; the mask
    and the denominator only make sense element-wise).
    Returns (loss, pred [B, H, A]) in float64.
    """
    m = model if model is not None else Model(weights, geom)
    ids = np.asarray(embodiment_id).reshape(-1)
    n = int(getattr(geom, "attend_text_every_n_blocks", 0))
    a = to_f64(actions)
    e = to_f64(noise)
    tt = to_f64(t).reshape(-1)
    preds = []
    for b in range(len(ids)):
        c = int(ids[b])
        if not 0 <= c < geom.num_embodiments:
            raise ValueError(f"embodiment_id {c} out of range")
        s, kvs = prepare_sample(m, backbone_features[b], vl_mask[b], state[b], c,
                                None if image_mask is None else image_mask[b], n)
        xt = (1.0 - tt[b]) * e[b] + tt[b] * a[b]
        td = math.floor(tt[b] * geom.num_timestep_buckets)
        preds.append(velocity(m, xt, float(td), s, kvs, c))
    pred = np.stack(preds)
    mask = to_f64(action_mask)
    loss = float((mask * (pred - (a - e)) ** 2).sum() / (mask.sum() + 1e-6))
    return loss, pred
