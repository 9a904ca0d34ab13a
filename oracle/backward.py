"""Gradients of the OneTrans block stack: the oracle of the backward pass
(TEST INFRASTRUCTURE ONLY; only tests/ and bench.py's CPU legs may use it).

The forward is restated here in plain fp64 PyTorch ops, step by step as in
onetrans_oracle.c (summary page, block / pyramid / KV-cache paragraphs):
per user the S side layer by layer (RMSNorm, shared QKV, causal attention of
the query tail over the layer's S keys, output projection, RMSNorm, GELU
FFN, residuals; the next layer's S rows are the tail), and per candidate the
NS side (private weights per NS position, attention over every S key of the
layer and the candidate's NS keys m <= n).  The gradients are torch
autograd's of the scalar loss
    sum(s_out * G_s) + sum(ns_out * G_ns)
for given upstream gradients G_s [U, q_last, d] and G_ns [U, C, N, d]:
autograd is the library step; the restated forward is pinned to the C
oracle and the gradients to central finite differences of the C oracle.

The S-side FFN dense or a sparse mixture of experts (cfg.moe_experts = E,
top cfg.moe_topk: the router reads the FFN's normalised input, the k largest
logits (ties to the lower expert index) are softmax-ed into gates, y = h +
sum_j g_j FFN_e(j)(z); the selection itself carries no gradient); the
OneTrans causal mask, or full (non-causal) attention
(cfg.full_attn, one candidate per user: summary page, limitations paragraph
— every token of a candidate's sequence sees every other, so the S rows
depend on the candidate and the two sides run jointly per layer).
"""

from __future__ import annotations

import math

import torch

W_NAMES = ("Wqkv_s", "Wo_s", "W1_s", "W2_s", "g1_s", "g2_s",
           "Wqkv_ns", "Wo_ns", "W1_ns", "W2_ns", "g1_ns", "g2_ns")
MOE_NAMES = ("W_router", "W1_moe", "W2_moe")


def names(cfg):
    """The tensors a config differentiates (a mixture adds its router and
    experts; the dense S-side W1_s / W2_s then get zero gradients)."""
    return W_NAMES + (MOE_NAMES if getattr(cfg, "moe_experts", 0) else ())


def _rms(x, g, eps):
    return x * torch.rsqrt((x * x).mean(-1, keepdim=True) + eps) * g


def _gelu(z):
    return 0.5 * z * (1.0 + torch.erf(z / math.sqrt(2.0)))


def _attend(q, k, v, mask, heads):
    """q [Tq, d], k / v [Tk, d], mask [Tq, Tk] (True = visible) -> [Tq, d]."""
    Tq, d = q.shape
    hd = d // heads
    qh = q.view(Tq, heads, hd).transpose(0, 1)
    kh = k.view(-1, heads, hd).transpose(0, 1)
    vh = v.view(-1, heads, hd).transpose(0, 1)
    s = qh @ kh.transpose(1, 2) / math.sqrt(hd)
    s = s.masked_fill(~mask, float("-inf"))
    p = torch.softmax(s, dim=-1)
    return (p @ vh).transpose(0, 1).reshape(Tq, d)


def _s_ffn(cfg, w, l, h):
    """The S-side FFN of layer l on rows h [q, d], residual included."""
    z = _rms(h, w["g2_s"][l], cfg.eps)
    E = getattr(cfg, "moe_experts", 0)
    if not E:
        return h + _gelu(z @ w["W1_s"][l].T) @ w["W2_s"][l].T
    k = cfg.moe_topk
    logits = z @ w["W_router"][l].T                                   # [q, E]
    # top-k by a stable sort of the negated logits: equal logits keep the
    # lower expert index first
    sel = torch.sort(-logits.detach(), dim=-1, stable=True).indices[:, :k]
    gates = torch.softmax(torch.gather(logits, 1, sel), dim=-1)       # [q, k]
    ys = torch.stack([_gelu(z @ w["W1_moe"][l, e].T) @ w["W2_moe"][l, e].T for e in range(E)])  # [E, q, d]
    rows = torch.arange(h.shape[0])
    out = h
    for j in range(k):
        out = out + gates[:, j:j + 1] * ys[sel[:, j], rows]
    return out


def _forward_full(cfg, w, S, ns):
    """Full attention, one candidate per user: per layer the joint sequence
    [S rows; NS rows], queries = the S tail and every NS row, keys = every
    row, all visible."""
    d, H, N, eps = cfg.d, cfg.heads, cfg.n_ns, cfg.eps
    assert ns.shape[1] == 1, "full attention runs one candidate per user"
    s_outs, ns_outs = [], []
    for u in range(S.shape[0]):
        x, y = S[u], ns[u, 0]
        for l in range(cfg.layers):
            L, q = x.shape[0], cfg.q[l]
            qkv_s = _rms(x, w["g1_s"][l], eps) @ w["Wqkv_s"][l].T
            qkv_n = torch.stack([_rms(y[n], w["g1_ns"][l, n], eps) @ w["Wqkv_ns"][l, n].T for n in range(N)])
            Q = torch.cat([qkv_s[L - q:, :d], qkv_n[:, :d]])
            K = torch.cat([qkv_s[:, d:2 * d], qkv_n[:, d:2 * d]])
            V = torch.cat([qkv_s[:, 2 * d:], qkv_n[:, 2 * d:]])
            a = _attend(Q, K, V, torch.ones(q + N, L + N, dtype=torch.bool), H)
            h = x[L - q:] + a[:q] @ w["Wo_s"][l].T
            x = _s_ffn(cfg, w, l, h)
            rows = []
            for n in range(N):
                hn = y[n] + a[q + n] @ w["Wo_ns"][l, n].T
                rows.append(hn + _gelu(_rms(hn, w["g2_ns"][l, n], eps) @ w["W1_ns"][l, n].T) @ w["W2_ns"][l, n].T)
            y = torch.stack(rows)
        s_outs.append(x)
        ns_outs.append(y[None])
    return torch.stack(s_outs), torch.stack(ns_outs)


def forward(cfg, w, S, ns):
    """S [U, L0, d], ns [U, C, N, d] (fp64 tensors) -> (s_out [U, q_last, d],
    ns_out [U, C, N, d]) with the weights of dict w (fp64 tensors)."""
    if getattr(cfg, "full_attn", False):
        return _forward_full(cfg, w, S, ns)
    d, H, N, eps = cfg.d, cfg.heads, cfg.n_ns, cfg.eps
    s_outs, ns_outs = [], []
    for u in range(S.shape[0]):
        x = S[u]
        kvs = []
        for l in range(cfg.layers):
            L, q = x.shape[0], cfg.q[l]
            z = _rms(x, w["g1_s"][l], eps)
            qkv = z @ w["Wqkv_s"][l].T
            Q, K, V = qkv[L - q:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
            kvs.append((K, V))
            t = torch.arange(L - q, L).unsqueeze(1)
            mask = torch.arange(L).unsqueeze(0) <= t            # S row t sees S keys 0..t
            a = _attend(Q, K, V, mask, H)
            h = x[L - q:] + a @ w["Wo_s"][l].T
            x = _s_ffn(cfg, w, l, h)
        s_outs.append(x)
        cand = []
        for c in range(ns.shape[1]):
            y = ns[u, c]
            for l in range(cfg.layers):
                K_s, V_s = kvs[l]
                L = K_s.shape[0]
                rows = []
                qkv = torch.stack([_rms(y[n], w["g1_ns"][l, n], eps) @ w["Wqkv_ns"][l, n].T
                                   for n in range(N)])
                Qn, Kn, Vn = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
                K = torch.cat([K_s, Kn])
                V = torch.cat([V_s, Vn])
                mask = torch.cat([torch.ones(N, L, dtype=torch.bool),
                                  torch.arange(N).unsqueeze(0) <= torch.arange(N).unsqueeze(1)], dim=1)
                a = _attend(Qn, K, V, mask, H)
                for n in range(N):
                    h = y[n] + a[n] @ w["Wo_ns"][l, n].T
                    f = _gelu(_rms(h, w["g2_ns"][l, n], eps) @ w["W1_ns"][l, n].T) @ w["W2_ns"][l, n].T
                    rows.append(h + f)
                y = torch.stack(rows)
            cand.append(y)
        ns_outs.append(torch.stack(cand))
    return torch.stack(s_outs), torch.stack(ns_outs)


def gradients(cfg, w, S, ns, G_s, G_ns):
    """(loss, grads): grads maps "S", "ns" and every weight name to the
    gradient of sum(s_out * G_s) + sum(ns_out * G_ns), fp64 CPU tensors."""
    wt = {k: torch.as_tensor(w[k]).detach().double().clone().requires_grad_(True) for k in names(cfg)}
    St = torch.as_tensor(S).detach().double().clone().requires_grad_(True)
    nst = torch.as_tensor(ns).detach().double().clone().requires_grad_(True)
    s_out, ns_out = forward(cfg, wt, St, nst)
    loss = (s_out * torch.as_tensor(G_s).double()).sum() + (ns_out * torch.as_tensor(G_ns).double()).sum()
    loss.backward()
    grads = {"S": St.grad, "ns": nst.grad}
    grads.update({k: wt[k].grad if wt[k].grad is not None else torch.zeros_like(wt[k]) for k in names(cfg)})
    return float(loss.detach()), grads
