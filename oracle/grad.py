"""Gradients of the flow-matching training loss, fp64 on the CPU.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests may
import it.

``training_loss_and_grads`` takes the same arguments as
``oracle.training_loss`` and also returns d loss / d parameter for every
weight of the table.  The forward is the action head's training objective
([ARCH] "Flow matching diffusion", "Training objective"; readings as in
``oracle.training_loss``), restated step for step in torch float64 ops so that
torch's autograd (a library primitive) differentiates it exactly up to
rounding.  Index work (which backbone tokens a cross layer sees) comes from
``oracle.cross_key_mask``; the sinusoid of the integer timestep carries no
parameter and is taken from ``oracle.sinusoidal_embedding``.

Pins (tests/test_oracle_grad.py), none of which goes through torch on the
expected side: the loss equals the numpy oracle's; central finite differences
of the numpy oracle's loss along random directions equal the directional
derivative; the decoder's last bias has the closed-form gradient
2 sum(mask (pred - target)) / (sum(mask) + 1e-6) per category; parameters off
the path (unused categories, an all-zero mask) get zero gradient.
"""

from __future__ import annotations

import math
from typing import Dict

import numpy as np
import torch

from .dit import cross_key_mask, sinusoidal_embedding, to_f64


def _layer_norm(x, eps, g=None, b=None):
    mu = x.mean(dim=-1, keepdim=True)
    var = ((x - mu) ** 2).mean(dim=-1, keepdim=True)
    y = (x - mu) / torch.sqrt(var + eps)
    return y if g is None else y * g + b


def _silu(x):
    return x / (1.0 + torch.exp(-x))


def _gelu(x):
    return 0.5 * x * (1.0 + torch.erf(x / math.sqrt(2.0)))


def _linear(x, w, b):
    return x @ w.T + b


def _attention(q, k, v, num_heads):
    nq, width = q.shape
    if k.shape[0] == 0:
        return torch.zeros((nq, width), dtype=q.dtype)
    dh = width // num_heads
    outs = []
    for h in range(num_heads):
        cols = slice(h * dh, (h + 1) * dh)
        s = (q[:, cols] @ k[:, cols].T) / math.sqrt(dh)
        p = torch.softmax(s, dim=1)
        outs.append(p @ v[:, cols])
    return torch.cat(outs, dim=1)


def _cat_mlp(P, prefix, x, c):
    h = torch.relu(x @ P[prefix + ".l1.W"][c] + P[prefix + ".l1.b"][c])
    return h @ P[prefix + ".l2.W"][c] + P[prefix + ".l2.b"][c]


def _velocity(P, g, x, td, state_feat, kvs, c):
    D = g.hidden
    phi = torch.from_numpy(sinusoidal_embedding(td, g.time_freq_dim))
    temb = _linear(_silu(_linear(phi, P["t_enc.l1.w"], P["t_enc.l1.b"])), P["t_enc.l2.w"], P["t_enc.l2.b"])
    a = x @ P["act_enc.W1.W"][c] + P["act_enc.W1.b"][c]
    tau = torch.from_numpy(sinusoidal_embedding(td, D)).expand(a.shape[0], D)
    z = _silu(torch.cat([a, tau], dim=-1) @ P["act_enc.W2.W"][c] + P["act_enc.W2.b"][c])
    e = z @ P["act_enc.W3.W"][c] + P["act_enc.W3.b"][c]
    h = torch.cat([state_feat, e], dim=0)

    def ada(hh, w, b):
        emb = _linear(_silu(temb), w, b)
        return _layer_norm(hh, g.ln_eps) * (1.0 + emb[:D]) + emb[D:]

    for layer in range(g.num_layers):
        p = f"blk{layer}."
        u = ada(h, P[p + "ada.w"], P[p + "ada.b"])
        q = _linear(u, P[p + "q.w"], P[p + "q.b"])
        if layer % 2 == 1:
            k = _linear(u, P[p + "k.w"], P[p + "k.b"])
            v = _linear(u, P[p + "v.w"], P[p + "v.b"])
        else:
            k, v = kvs[layer]
        h = h + _linear(_attention(q, k, v, g.num_heads), P[p + "o.w"], P[p + "o.b"])
        f = _gelu(_linear(_layer_norm(h, g.ln_eps, P[p + "ln3.g"], P[p + "ln3.b"]), P[p + "ff1.w"], P[p + "ff1.b"]))
        h = h + _linear(f, P[p + "ff2.w"], P[p + "ff2.b"])
    y = _linear(ada(h, P["out.ada.w"], P["out.ada.b"]), P["out.proj.w"], P["out.proj.b"])
    return _cat_mlp(P, "act_dec", y, c)[state_feat.shape[0]:]


def training_loss_and_grads(weights: Dict[str, np.ndarray], geom, backbone_features, vl_mask, state,
                            embodiment_id, actions, noise, t, action_mask, image_mask=None):
    """(loss, {name: d loss / d weight}) of the training objective, float64.

    Same inputs and readings as ``oracle.training_loss``: x_t = (1 - t) noise +
    t actions, target actions - noise, prediction at floor(t * buckets),
    loss = sum(mask (pred - target)^2) / (sum(mask) + 1e-6).  Gradients are
    float64 arrays of each weight's shape (zeros where the loss does not
    depend on the entry)."""
    P = {k: torch.tensor(to_f64(v), requires_grad=True) for k, v in weights.items()}
    g = geom
    n = int(getattr(g, "attend_text_every_n_blocks", 0))
    ids = np.asarray(embodiment_id).reshape(-1)
    a_all = torch.from_numpy(to_f64(actions))
    e_all = torch.from_numpy(to_f64(noise))
    tt = to_f64(t).reshape(-1)
    mask = torch.from_numpy(to_f64(action_mask))
    total = torch.zeros((), dtype=torch.float64)
    for b in range(len(ids)):
        c = int(ids[b])
        if not 0 <= c < g.num_embodiments:
            raise ValueError(f"embodiment_id {c} out of range")
        f = torch.from_numpy(to_f64(backbone_features[b]))
        if "vlln.g" in P:
            f = _layer_norm(f, g.ln_eps, P["vlln.g"], P["vlln.b"])
        img = None if image_mask is None else image_mask[b]
        kvs = {}
        for layer in range(0, g.num_layers, 2):
            sel = torch.from_numpy(np.nonzero(cross_key_mask(layer, vl_mask[b], img, n))[0])
            fv = f[sel]
            p = f"blk{layer}."
            kvs[layer] = (_linear(fv, P[p + "k.w"], P[p + "k.b"]), _linear(fv, P[p + "v.w"], P[p + "v.b"]))
        s = torch.from_numpy(to_f64(state[b]).reshape(-1, g.state_dim))
        s = _cat_mlp(P, "state_enc", s, c)
        xt = (1.0 - tt[b]) * e_all[b] + tt[b] * a_all[b]
        td = float(math.floor(tt[b] * g.num_timestep_buckets))
        pred = _velocity(P, g, xt, td, s, kvs, c)
        total = total + (mask[b] * (pred - (a_all[b] - e_all[b])) ** 2).sum()
    loss = total / (mask.sum() + 1e-6)
    loss.backward()
    grads = {k: (p.grad.numpy().copy() if p.grad is not None else np.zeros(p.shape)) for k, p in P.items()}
    return float(loss.detach()), grads
