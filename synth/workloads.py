"""Workload shapes and seeded generators.

Each workload follows one of the five synthetic configurations that stand in
for the pages' private ByteDance logs (the OneTrans summary page, "Offline
logs" paragraph, says there is no public table).  Model shapes follow the
OneTransS / OneTransL sentence of that page; every value is drawn here from a
``torch.Generator`` on the CPU and rounded to the run's storage dtype.

Every random tensor has its own generator, seeded from ``(workload seed,
tag, index)``, so that the rows of user ``u`` (or candidate ``c`` of user
``u``) are the same whether one user or the whole batch is generated.  That is
what lets the oracle run on a subset of users and candidates of a large batch.

Nothing in this module computes any part of the block.
"""

from __future__ import annotations

import hashlib
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    d: int
    heads: int
    ffn: int
    n_ns: int            # N: NS tokens per candidate
    L0: int              # S tokens per user entering layer 0
    q_end: int | None    # pyramid end length; None = no pyramid
    F: int               # Auto-Split input width
    users: int
    cands: int
    dtype: str           # "f32" | "bf16" | "fp8" (fp8: bf16 storage, e4m3 GEMMs)
    seed: int
    eps: float = 1e-6
    seq_lens: tuple = ()         # behaviour sequences joined into the S stream
    interleave: bool = False     # merge sequences by timestamp instead of concatenating
    zipf_s: float | None = None  # S rows are gathered Zipf item ids (long-sequence case)
    table_rows: int = 0
    table_std: float = 0.02
    description: str = ""

    @property
    def hd(self) -> int:
        return self.d // self.heads

    @property
    def storage(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    # Tiny block check, fp32: one block, no pyramid, 1 user x 4 candidates.
    "tiny_fp32": Workload(
        "tiny_fp32", layers=1, d=64, heads=2, ffn=256, n_ns=8, L0=32, q_end=None,
        F=256, users=1, cands=4, dtype="f32", seed=0, seq_lens=(32,),
        description="1 block, d=64, 2 heads, FFN 256, 32 S + 8 NS tokens, fp32"),
    # OneTransS-shaped full forward: 3 sequences joined by 2 learned [SEP].
    "onetrans_s_full": Workload(
        "onetrans_s_full", layers=6, d=256, heads=4, ffn=1024, n_ns=16, L0=1190,
        q_end=12, F=1024, users=64, cands=1, dtype="bf16", seed=1,
        seq_lens=(600, 400, 188),
        description="OneTransS full forward, 6 layers d=256, 1190->12, B=64"),
    # OneTransS serving: encode 16 users, score 512 candidates each.
    "onetrans_s_serve": Workload(
        "onetrans_s_serve", layers=6, d=256, heads=4, ffn=1024, n_ns=16, L0=1190,
        q_end=12, F=1024, users=16, cands=512, dtype="bf16", seed=2,
        seq_lens=(600, 400, 188),
        description="OneTransS serving, encode U=16, score 16x512 candidates"),
    # OneTransL-shaped full forward: 4 time-interleaved sequences + 3 [SEP].
    "onetrans_l_full": Workload(
        "onetrans_l_full", layers=8, d=384, heads=6, ffn=1536, n_ns=24, L0=1500,
        q_end=16, F=1024, users=32, cands=1, dtype="bf16", seed=3,
        seq_lens=(600, 400, 300, 197), interleave=True,
        description="OneTransL full forward, 8 layers d=384, 1500->16, B=32"),
    # Long-sequence FP8 serving: Zipf item ids gathered from a 2^20-row table.
    "long_fp8": Workload(
        "long_fp8", layers=8, d=384, heads=6, ffn=1536, n_ns=32, L0=8192, q_end=16,
        F=1024, users=8, cands=256, dtype="fp8", seed=4, zipf_s=1.1,
        table_rows=1 << 20,
        description="8192-token FP8 serving, U=8 x 256 candidates"),
}


def _seed_of(seed: int, *tags) -> int:
    h = hashlib.sha256(repr((seed,) + tags).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed: int, *tags) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(_seed_of(seed, *tags))
    return g


def storage_round(t: torch.Tensor, wl: Workload) -> torch.Tensor:
    """Round a float tensor to the workload's storage dtype (RNE)."""
    return t.to(wl.storage)


def _randn(gen, shape, std=1.0):
    return torch.randn(shape, generator=gen, dtype=torch.float32) * std


def gen_weights(wl: Workload) -> dict[str, torch.Tensor]:
    """Random-init weights of the workload's architecture, in storage dtype.

    Layouts (row-major, "out x in" like a linear layer's weight):
      Wqkv_s [layers, 3d, d]  rows 0..d-1 = Q, d..2d-1 = K, 2d..3d-1 = V
      Wo_s   [layers, d, d]
      W1_s   [layers, ffn, d]
      W2_s   [layers, d, ffn]
      g1_s, g2_s [layers, d]
      Wqkv_ns [layers, N, 3d, d], Wo_ns [layers, N, d, d],
      W1_ns [layers, N, ffn, d], W2_ns [layers, N, d, ffn],
      g1_ns, g2_ns [layers, N, d]
      W_split [N*d, F]
      sep [n_seq-1, d]   learned [SEP] rows (S-side input data, not block weights)
    Matrices ~ N(0, 1/fan_in); RMSNorm gains ~ 1 + 0.1 N(0,1).
    """
    L, d, f, N = wl.layers, wl.d, wl.ffn, wl.n_ns
    s = wl.seed
    out: dict[str, torch.Tensor] = {}

    def mat(tag, shape, fan_in):
        return storage_round(_randn(_gen(s, "w", tag), shape, fan_in ** -0.5), wl)

    def gain(tag, shape):
        return storage_round(1.0 + 0.1 * _randn(_gen(s, "w", tag), shape), wl)

    out["Wqkv_s"] = mat("Wqkv_s", (L, 3 * d, d), d)
    out["Wo_s"] = mat("Wo_s", (L, d, d), d)
    out["W1_s"] = mat("W1_s", (L, f, d), d)
    out["W2_s"] = mat("W2_s", (L, d, f), f)
    out["g1_s"] = gain("g1_s", (L, d))
    out["g2_s"] = gain("g2_s", (L, d))
    # NS weights are the bulk of the parameters: draw them one layer at a time.
    for name, shape, fan in (("Wqkv_ns", (N, 3 * d, d), d), ("Wo_ns", (N, d, d), d),
                             ("W1_ns", (N, f, d), d), ("W2_ns", (N, d, f), f)):
        out[name] = torch.stack([mat((name, l), shape, fan) for l in range(L)])
    out["g1_ns"] = gain("g1_ns", (L, N, d))
    out["g2_ns"] = gain("g2_ns", (L, N, d))
    out["W_split"] = mat("W_split", (N * d, wl.F), wl.F)
    nsep = max(len(wl.seq_lens) - 1, 0)
    out["sep"] = storage_round(_randn(_gen(s, "sep"), (nsep, d)), wl)
    return out


def _interleave_order(wl: Workload, gen: torch.Generator):
    """Row order of one user's S stream: list of (seq k, index i) or ('sep', k).

    Concatenation: seq0 | SEP0 | seq1 | SEP1 | ... | seq_last.
    Time interleave: every event gets a U(0,1) timestamp (sorted within its
    sequence), events merge by (timestamp, sequence id, index), and SEP_k goes
    right after the last event of sequence k unless that event ends the stream.
    """
    lens = wl.seq_lens
    if not wl.interleave:
        order = []
        for k, n in enumerate(lens):
            order += [(k, i) for i in range(n)]
            if k + 1 < len(lens):
                order.append(("sep", k))
        return order
    events = []
    for k, n in enumerate(lens):
        ts = torch.sort(torch.rand(n, generator=gen, dtype=torch.float64)).values
        events += [(float(ts[i]), k, i) for i in range(n)]
    events.sort()
    last = {k: max(j for j, e in enumerate(events) if e[1] == k) for k in range(len(lens))}
    order = []
    sep_ids = [k for k in range(len(lens)) if last[k] != len(events) - 1]
    sep_of = {k: j for j, k in enumerate(sep_ids)}
    for j, (_, k, i) in enumerate(events):
        order.append((k, i))
        if k in sep_of and last[k] == j:
            order.append(("sep", sep_of[k]))
    return order


def gen_s_tokens(wl: Workload, users=None, weights=None) -> torch.Tensor:
    """S-token rows [len(users), L0, d] in storage dtype.

    Behaviour events ~ N(0,1); learned [SEP] rows come from ``weights['sep']``.
    For the Zipf workload use :func:`gen_zipf_ids` + :func:`gen_embedding_table`.
    """
    if wl.zipf_s is not None:
        raise ValueError("the Zipf workload gathers S rows from an embedding table")
    users = range(wl.users) if users is None else users
    if weights is None:
        weights = gen_weights(wl)
    sep = weights["sep"].float()
    rows = []
    for u in users:
        g = _gen(wl.seed, "S", u)
        seqs = [_randn(g, (n, wl.d)) for n in wl.seq_lens]
        order = _interleave_order(wl, _gen(wl.seed, "ts", u))
        x = torch.stack([sep[k] if a == "sep" else seqs[a][k] for a, k in order])
        assert x.shape[0] == wl.L0, (x.shape, wl.L0)
        rows.append(x)
    return storage_round(torch.stack(rows), wl)


def gen_auto_split_features(wl: Workload, users=None, cands=None) -> torch.Tensor:
    """Static feature vectors x [len(users), len(cands), F] ~ N(0,1)."""
    users = range(wl.users) if users is None else users
    cands = range(wl.cands) if cands is None else list(cands)
    out = []
    for u in users:
        allc = _randn(_gen(wl.seed, "x", u), (wl.cands, wl.F))
        out.append(allc[list(cands)])
    return storage_round(torch.stack(out), wl)


def gen_embedding_table(wl: Workload, rows: int | None = None) -> torch.Tensor:
    """Item embedding table [table_rows, d] ~ N(0, table_std^2), bf16."""
    rows = wl.table_rows if rows is None else rows
    g = _gen(wl.seed, "table")
    chunks, left = [], rows
    while left:
        n = min(left, 1 << 18)
        chunks.append((_randn(g, (n, wl.d)) * wl.table_std).to(torch.bfloat16))
        left -= n
    return torch.cat(chunks)


def gen_zipf_ids(wl: Workload, users=None, rows: int | None = None) -> torch.Tensor:
    """Item ids [len(users), L0] int64: rank k in [1, rows] with P(k) ~ k^-s,
    mapped to table row perm[k-1] of a seeded permutation (hot ids scattered)."""
    rows = wl.table_rows if rows is None else rows
    users = range(wl.users) if users is None else users
    k = torch.arange(1, rows + 1, dtype=torch.float64)
    cdf = torch.cumsum(k ** (-wl.zipf_s), 0)
    cdf /= cdf[-1].clone()
    perm = torch.randperm(rows, generator=_gen(wl.seed, "perm"))
    out = []
    for u in users:
        r = torch.rand(wl.L0, generator=_gen(wl.seed, "ids", u), dtype=torch.float64)
        rank0 = torch.searchsorted(cdf, r).clamp_(max=rows - 1)
        out.append(perm[rank0])
    return torch.stack(out).to(torch.int64)
