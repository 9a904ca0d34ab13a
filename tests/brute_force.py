"""Brute-force OneTrans block stack in pure Python (test-only second implementation).

An independent restatement used to pin the C oracle on tiny inputs: every
candidate's tokens are one Python list of Token records, each token looks up
its own parameter set (S shared / NS private by position), and visibility is
decided token pair by token pair from the mask rule of the OneTrans summary
page (an S-token sees earlier S-tokens and itself; an NS-token sees every
S-token and the preceding NS-tokens of its candidate, and itself).  Plain
floats and the math module only; no numpy arithmetic, no shared code with the
C oracle.

FP8 rules (optional): every projection input is rounded to e4m3 by torch's
float8_e4m3fn cast (saturated at +-448 first), with one scale per input row
(amax / 448) or one given scale per input tensor; each weight matrix with one
scale amax / 448.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass
class Token:
    kind: str        # "S" or "NS"
    index: int       # S: position in the S stream; NS: position n
    x: list


def _rms(x, g, eps):
    ms = sum(v * v for v in x) / len(x)
    inv = 1.0 / math.sqrt(ms + eps)
    return [v * inv * gg for v, gg in zip(x, g)]


def _mv(W, x):
    """W given as list of output rows (out x in)."""
    return [sum(wk * xk for wk, xk in zip(row, x)) for row in W]


def _e4m3(vals):
    """Round to e4m3 (nearest even, saturating) with torch's float8 cast."""
    t = torch.tensor(vals, dtype=torch.float64).clamp(-448.0, 448.0)
    return t.to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).tolist()


class Fp8:
    """Quantisation state of one run: rule 1 (scale per input row) or 2 (one
    given scale per input tensor, act_scale[l][set][t]); amax[l][set][t]
    collects max |x| of every input seen."""

    def __init__(self, rule, act_scale=None, amax=None):
        self.rule, self.act_scale, self.amax = rule, act_scale, amax
        self._wq = {}

    def weights(self, W):
        key = id(W)
        if key not in self._wq:
            flat = [v for row in W for v in row]
            a = max(abs(v) for v in flat)
            s = a / 448.0 if a > 0 else 1.0
            q = _e4m3([v / s for v in flat])
            n = len(W[0])
            self._wq[key] = ([q[i * n:(i + 1) * n] for i in range(len(W))], s, W)
        return self._wq[key][0], self._wq[key][1]


def _proj(W, x, fp8, slot):
    """x W^T; under an FP8 rule both operands are quantised first.  slot =
    (layer, parameter set, input index) of the input tensor."""
    l, st, t = slot
    if fp8 is not None and fp8.amax is not None:
        a = max(abs(v) for v in x)
        fp8.amax[l][st][t] = max(fp8.amax[l][st][t], a)
    if fp8 is None or fp8.rule == 0:
        return _mv(W, x)
    if fp8.rule == 1:
        a = max(abs(v) for v in x)
        sx = a / 448.0 if a > 0 else 1.0
    else:
        sx = fp8.act_scale[l][st][t]
    xq = _e4m3([v / sx for v in x])
    Wq, sw = fp8.weights(W)
    return [v * sx * sw for v in _mv(Wq, xq)]


def _gelu(z):
    return 0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0)))


def _visible(qt: Token, kt: Token, full: bool = False) -> bool:
    if full:            # full attention: every token of the sequence
        return True
    if qt.kind == "S":
        return kt.kind == "S" and kt.index <= qt.index
    return kt.kind == "S" or kt.index <= qt.index


def _set(tok: Token) -> int:
    """Parameter set index: 0 for S tokens, 1 + n for NS position n."""
    return 0 if tok.kind == "S" else 1 + tok.index


def _params(w, l, tok: Token):
    """Nested lists for the token's parameter set at layer l."""
    if tok.kind == "S":
        return (w["Wqkv_s"][l], w["Wo_s"][l], w["W1_s"][l], w["W2_s"][l], w["g1_s"][l],
                w["g2_s"][l])
    n = tok.index
    return (w["Wqkv_ns"][l][n], w["Wo_ns"][l][n], w["W1_ns"][l][n], w["W2_ns"][l][n],
            w["g1_ns"][l][n], w["g2_ns"][l][n])


def _moe_ffn(w, l, z, topk):
    """Sparse mixture of experts on the S side: top-k router logits (ties to
    the lower index), softmax over them, gated sum of the experts' FFNs."""
    logits = _mv(w["W_router"][l], z)
    order = sorted(range(len(logits)), key=lambda e: (-logits[e], e))[:topk]
    mx = logits[order[0]]
    ex = [math.exp(logits[e] - mx) for e in order]
    out = [0.0] * len(z)
    for e, x in zip(order, ex):
        f = [_gelu(v) for v in _mv(w["W1_moe"][l][e], z)]
        out = [o + x / sum(ex) * v for o, v in zip(out, _mv(w["W2_moe"][l][e], f))]
    return out


def run_candidate(w, S_rows, ns_rows, q_sched, heads, eps, fp8=None, full=False, moe_topk=0):
    """One candidate: S_rows [L0][d], ns_rows [N][d] (lists).

    Returns (S tail rows after the last layer, NS rows, per-layer (K, V) of
    the S tokens).  ``w`` holds nested Python lists; ``fp8`` an Fp8 state or
    None; ``full``: full (non-causal) attention over the candidate's sequence;
    ``moe_topk`` > 0: the S tokens' FFN is the mixture of experts in ``w``.
    """
    d = len(S_rows[0])
    hd = d // heads
    seq = [Token("S", i, list(r)) for i, r in enumerate(S_rows)]
    seq += [Token("NS", n, list(r)) for n, r in enumerate(ns_rows)]
    kv_layers = []
    for l, q in enumerate(q_sched):
        n_s = sum(1 for t in seq if t.kind == "S")
        proj = []
        for t in seq:
            Wqkv, _, _, _, g1, _ = _params(w, l, t)
            qkv = _proj(Wqkv, _rms(t.x, g1, eps), fp8, (l, _set(t), 0))
            proj.append((qkv[:d], qkv[d:2 * d], qkv[2 * d:]))
        kv_layers.append(([p[1] for t, p in zip(seq, proj) if t.kind == "S"],
                          [p[2] for t, p in zip(seq, proj) if t.kind == "S"]))
        new_seq = []
        for i, t in enumerate(seq):
            if t.kind == "S" and t.index < n_s - q:
                continue  # not in this layer's query tail
            a = []
            for h in range(heads):
                qv = proj[i][0][h * hd:(h + 1) * hd]
                scores, vals = [], []
                for j, kt in enumerate(seq):
                    if not _visible(t, kt, full):
                        continue
                    kvec = proj[j][1][h * hd:(h + 1) * hd]
                    scores.append(sum(a_ * b_ for a_, b_ in zip(qv, kvec)) / math.sqrt(hd))
                    vals.append(proj[j][2][h * hd:(h + 1) * hd])
                m = max(scores)
                e = [math.exp(s - m) for s in scores]
                z = sum(e)
                a += [sum(e[k] / z * vals[k][c] for k in range(len(e))) for c in range(hd)]
            _, Wo, W1, W2, _, g2 = _params(w, l, t)
            st = _set(t)
            hrow = [xv + ov for xv, ov in zip(t.x, _proj(Wo, a, fp8, (l, st, 1)))]
            if moe_topk and t.kind == "S":
                y = [hv + fv for hv, fv in zip(hrow, _moe_ffn(w, l, _rms(hrow, g2, eps), moe_topk))]
            else:
                f = [_gelu(v) for v in _proj(W1, _rms(hrow, g2, eps), fp8, (l, st, 2))]
                y = [hv + fv for hv, fv in zip(hrow, _proj(W2, f, fp8, (l, st, 3)))]
            new_seq.append(Token(t.kind, t.index, y))
        # re-index the S tail 0..q-1 so the next layer's S stream starts at 0
        s_tail = [t for t in new_seq if t.kind == "S"]
        for k, t in enumerate(s_tail):
            t.index = k
        seq = new_seq
    return ([t.x for t in seq if t.kind == "S"], [t.x for t in seq if t.kind == "NS"],
            kv_layers)
