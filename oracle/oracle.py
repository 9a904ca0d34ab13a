"""Python face of the CPU fp64 oracle (TEST INFRASTRUCTURE ONLY).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this module.  It loads the C oracle through ctypes and never
touches a GPU or the CUDA product library.

Inputs are float32 arrays (exact for every bf16 / fp32 value the runs use);
outputs are float64.  See onetrans_oracle.c for what is computed and where on
the pages each step comes from.
"""

from __future__ import annotations

import ctypes as C
from dataclasses import dataclass, field
from fractions import Fraction

import numpy as np

from . import build as _build

MAX_LAYERS = 64


class _Cfg(C.Structure):
    _fields_ = [("layers", C.c_int), ("d", C.c_int), ("heads", C.c_int), ("ffn", C.c_int),
                ("n_ns", C.c_int), ("L0", C.c_int), ("q", C.c_int * MAX_LAYERS),
                ("eps", C.c_double), ("fp8", C.c_int), ("act_scale", C.POINTER(C.c_double)),
                ("act_amax", C.POINTER(C.c_double)), ("full_attn", C.c_int),
                ("moe_experts", C.c_int), ("moe_topk", C.c_int)]


# FP8 rules of the projection inputs (see onetrans_oracle.c): off, one scale
# per input row (the calibration pass), one fixed scale per input tensor.
FP8_OFF, FP8_ROW, FP8_TENSOR = 0, 1, 2
# the four projection inputs of a parameter set, in the act_scale layout
INPUTS = ("qkv", "o", "w1", "w2")


_WNAMES = ("Wqkv_s", "Wo_s", "W1_s", "W2_s", "g1_s", "g2_s",
           "Wqkv_ns", "Wo_ns", "W1_ns", "W2_ns", "g1_ns", "g2_ns")
# sparse-MoE S-side FFN (optional): router [layers][E][d], experts
# W1 [layers][E][ffn][d], W2 [layers][E][d][ffn]
_MOE_NAMES = ("W_router", "W1_moe", "W2_moe")


class _W(C.Structure):
    _fields_ = [(n, C.POINTER(C.c_float)) for n in _WNAMES + _MOE_NAMES]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(_build.build())
        dp, fp = C.POINTER(C.c_double), C.POINTER(C.c_float)
        L.orc_encode_user.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), fp, C.c_int, dp, dp]
        L.orc_score_candidates.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), dp, C.c_int, dp,
                                           C.c_int, dp]
        L.orc_encode_append.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), dp, fp, C.c_int, C.c_int,
                                        dp, dp]
        L.orc_full_forward_joint.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), fp, C.c_int, dp,
                                             C.c_int, dp, dp, dp]
        L.orc_auto_split.argtypes = [fp, C.c_long, C.c_int, fp, C.c_int, dp]
        L.orc_embed_gather.argtypes = [fp, C.c_long, C.c_int, C.POINTER(C.c_longlong), C.c_long,
                                       dp]
        L.orc_kv_user_elems.argtypes = [C.POINTER(_Cfg)]
        L.orc_kv_user_elems.restype = C.c_long
        L.orc_kv_layer_offset.argtypes = [C.POINTER(_Cfg), C.c_int]
        L.orc_kv_layer_offset.restype = C.c_long
        L.orc_project_rows.argtypes = [dp, C.c_long, C.c_int, fp, C.c_int, C.c_int, C.c_double,
                                       dp, dp]
        L.orc_e4m3_round.argtypes = [C.c_double]
        L.orc_e4m3_round.restype = C.c_double
        L.orc_set_threads.argtypes = [C.c_int]
        L.orc_set_threads.restype = C.c_int
        _lib = L
    return _lib


def set_threads(n: int = 0) -> int:
    """Set (n > 0) and return the OpenMP thread count the oracle uses."""
    return lib().orc_set_threads(n)


def pyramid_schedule(L0: int, q_end: int | None, layers: int) -> list[int]:
    """Query tail per layer: q_l = round(L0 - (L0 - q_end) * l / (layers - 1)).

    Linear from L0 (layer 0 keeps every row) to q_end at the last layer, ties
    to even; no pyramid (q_end None, or a single layer) keeps L0 everywhere.
    Follows the pyramid sentence of the OneTrans summary page and the
    workloads' stated formula.
    """
    if q_end is None or layers == 1:
        return [L0] * layers
    out = []
    for l in range(layers):
        v = Fraction(L0) - Fraction(L0 - q_end) * Fraction(l, layers - 1)
        out.append(round(v))  # Fraction.__round__ rounds half to even
    return out


@dataclass
class Config:
    """Block-stack shape.  ``fp8``: FP8_OFF (also False), FP8_ROW (also True)
    or FP8_TENSOR, which needs ``act_scale`` [layers][1 + n_ns][4] (set 0 =
    S, 1 + n = NS position n; inputs of QKV, O, W1, W2)."""
    layers: int
    d: int
    heads: int
    ffn: int
    n_ns: int
    L0: int
    q: list = field(default_factory=list)
    eps: float = 1e-6
    fp8: int = FP8_OFF
    act_scale: object = None
    full_attn: bool = False     # full (non-causal) attention: joint form only
    moe_experts: int = 0        # E > 0: sparse mixture of E experts as the S-side FFN
    moe_topk: int = 1           # experts per S row (1 or 2)

    @staticmethod
    def of(wl, q=None, fp8=None, act_scale=None) -> "Config":
        q = pyramid_schedule(wl.L0, wl.q_end, wl.layers) if q is None else list(q)
        if fp8 is None:
            fp8 = FP8_TENSOR if act_scale is not None else (
                FP8_ROW if wl.dtype == "fp8" else FP8_OFF)
        return Config(wl.layers, wl.d, wl.heads, wl.ffn, wl.n_ns, wl.L0, q, wl.eps, fp8,
                      act_scale)

    def scale_shape(self) -> tuple:
        return (self.layers, 1 + self.n_ns, 4)

    def rows_at(self, l: int) -> int:
        return self.L0 if l == 0 else self.q[l - 1]

    def _c(self, amax=None) -> _Cfg:
        """The C struct; ``amax`` (float64 [layers][1 + n_ns][4], C order) is
        max-accumulated by the call it is passed to."""
        c = _Cfg()
        c.layers, c.d, c.heads, c.ffn, c.n_ns, c.L0 = (self.layers, self.d, self.heads, self.ffn,
                                                      self.n_ns, self.L0)
        for i, v in enumerate(self.q):
            c.q[i] = int(v)
        c.eps = float(self.eps)
        c.fp8 = int(self.fp8)
        c.full_attn = int(bool(self.full_attn))
        c.moe_experts = int(self.moe_experts)
        c.moe_topk = int(self.moe_topk)
        if self.fp8 == FP8_TENSOR:
            if self.act_scale is None:
                raise ValueError("per-tensor FP8 needs act_scale")
            self._scale = np.ascontiguousarray(self.act_scale, dtype=np.float64)
            assert self._scale.shape == self.scale_shape(), self._scale.shape
            c.act_scale = _dptr(self._scale)
        if amax is not None:
            assert amax.shape == self.scale_shape() and amax.dtype == np.float64
            assert amax.flags.c_contiguous
            c.act_amax = _dptr(amax)
        return c

    def grown(self, delta: int) -> "Config":
        """The configuration after appending `delta` S rows: L0 and every
        query tail longer by delta (pyramid windows anchored at their first
        row)."""
        return Config(self.layers, self.d, self.heads, self.ffn, self.n_ns, self.L0 + delta,
                      [v + delta for v in self.q], self.eps, self.fp8, self.act_scale,
                      self.full_attn, self.moe_experts, self.moe_topk)

    def kv_user_elems(self) -> int:
        return int(lib().orc_kv_user_elems(C.byref(self._c())))

    def kv_layer_offset(self, l: int) -> int:
        return int(lib().orc_kv_layer_offset(C.byref(self._c()), l))


def _f32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().float().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().double().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _fptr(a):
    return a.ctypes.data_as(C.POINTER(C.c_float))


def _dptr(a):
    return a.ctypes.data_as(C.POINTER(C.c_double))


class Weights:
    """Holds float32 copies of the weights and the C struct pointing at them."""

    def __init__(self, w: dict):
        self.arrays = {n: _f32(w[n]) for n in _WNAMES}
        self.arrays.update({n: _f32(w[n]) for n in _MOE_NAMES if w.get(n) is not None})
        self.c = _W(**{n: _fptr(a) for n, a in self.arrays.items()})


def _weights(w):
    return w if isinstance(w, Weights) else Weights(w)


def kv_layer(cfg: Config, kv_user: np.ndarray, l: int):
    """(K, V) of layer l, each [L_l, d], from one user's packed cache."""
    off, L, d = cfg.kv_layer_offset(l), cfg.rows_at(l), cfg.d
    K = kv_user[off: off + L * d].reshape(L, d)
    V = kv_user[off + L * d: off + 2 * L * d].reshape(L, d)
    return K, V


def encode_user(cfg: Config, w, S, amax=None):
    """S [U, L0, d] -> (kv [U, kv_user_elems], s_out [U, q_last, d]).
    ``amax``: optional float64 array of cfg.scale_shape(), max-accumulated
    with every projection input's max |x| (calibration)."""
    S = _f32(S)
    U = S.shape[0]
    assert S.shape == (U, cfg.L0, cfg.d), S.shape
    W = _weights(w)
    kv = np.zeros((U, cfg.kv_user_elems()))
    s_out = np.zeros((U, cfg.q[-1], cfg.d))
    rc = lib().orc_encode_user(C.byref(cfg._c(amax)), C.byref(W.c), _fptr(S), U, _dptr(kv),
                               _dptr(s_out))
    if rc:
        raise ValueError("oracle rejected the configuration")
    return kv, s_out


def encode_append(cfg: Config, w, kv_old, S_new):
    """Append S_new [U, delta, d] to users encoded with the configuration
    that `cfg` (the grown one) was grown from.  kv_old [U, old kv_user_elems]
    -> (kv [U, kv_user_elems], out_new [U, delta, d]): the grown cache and
    the new rows' outputs of the last layer."""
    S_new, kv_old = _f32(S_new), _f64(kv_old)
    U, delta = S_new.shape[0], S_new.shape[1]
    assert S_new.shape == (U, delta, cfg.d), S_new.shape
    old = cfg.grown(-delta)
    assert kv_old.shape == (U, old.kv_user_elems()), kv_old.shape
    W = _weights(w)
    kv = np.zeros((U, cfg.kv_user_elems()))
    out = np.zeros((U, delta, cfg.d))
    rc = lib().orc_encode_append(C.byref(cfg._c()), C.byref(W.c), _dptr(kv_old), _fptr(S_new), U,
                                 delta, _dptr(kv), _dptr(out))
    if rc:
        raise ValueError("oracle rejected the configuration")
    return kv, out


def score_candidates(cfg: Config, w, kv, ns, amax=None):
    """kv [U, kv_user_elems], ns [U, C, N, d] -> ns_out [U, C, N, d].
    ``amax`` as for encode_user."""
    kv, ns = _f64(kv), _f64(ns)
    U, Cn = ns.shape[0], ns.shape[1]
    assert ns.shape == (U, Cn, cfg.n_ns, cfg.d) and kv.shape == (U, cfg.kv_user_elems())
    W = _weights(w)
    out = np.zeros_like(ns)
    rc = lib().orc_score_candidates(C.byref(cfg._c(amax)), C.byref(W.c), _dptr(kv), U, _dptr(ns),
                                    Cn, _dptr(out))
    if rc:
        raise ValueError("oracle rejected the configuration")
    return out


def full_forward_joint(cfg: Config, w, S, ns):
    """No-cache joint form.  Returns (s_out [U,C,q_last,d], kv [U,C,kv], ns_out [U,C,N,d])."""
    S, ns = _f32(S), _f64(ns)
    U, Cn = ns.shape[0], ns.shape[1]
    assert S.shape == (U, cfg.L0, cfg.d) and ns.shape == (U, Cn, cfg.n_ns, cfg.d)
    W = _weights(w)
    s_out = np.zeros((U, Cn, cfg.q[-1], cfg.d))
    kv = np.zeros((U, Cn, cfg.kv_user_elems()))
    ns_out = np.zeros_like(ns)
    rc = lib().orc_full_forward_joint(C.byref(cfg._c()), C.byref(W.c), _fptr(S), U, _dptr(ns),
                                      Cn, _dptr(s_out), _dptr(kv), _dptr(ns_out))
    if rc:
        raise ValueError("oracle rejected the configuration")
    return s_out, kv, ns_out


def auto_split(x, W_split, n_ns: int, d: int):
    """x [..., F], W_split [N*d, F] -> NS tokens [..., N, d] (fp64)."""
    x = _f32(x)
    lead, F = x.shape[:-1], x.shape[-1]
    x2 = x.reshape(-1, F)
    Wsp = _f32(W_split)
    assert Wsp.shape == (n_ns * d, F)
    out = np.zeros((x2.shape[0], n_ns * d))
    lib().orc_auto_split(_fptr(x2), x2.shape[0], F, _fptr(Wsp), n_ns * d, _dptr(out))
    return out.reshape(*lead, n_ns, d)


def embed_gather(table, ids):
    table = _f32(table)
    ids = np.ascontiguousarray(np.asarray(ids), dtype=np.int64)
    out = np.zeros(ids.shape + (table.shape[1],))
    rc = lib().orc_embed_gather(_fptr(table), table.shape[0], table.shape[1],
                                ids.ctypes.data_as(C.POINTER(C.c_longlong)), ids.size, _dptr(out))
    if rc:
        raise IndexError("embedding id out of range")
    return out


def e4m3_round(v: float) -> float:
    return float(lib().orc_e4m3_round(float(v)))


def project_rows(x, W, fp8=FP8_OFF, xs=1.0, amax=None):
    """One projection y = x W^T of rows x [R, in] by W [out, in] under an FP8
    rule, through the same code the block's projections use (weights
    quantised with one scale amax(W)/448; inputs per row or with the
    per-tensor scale xs).  ``amax``: optional float64 [1] accumulator."""
    x = _f64(np.atleast_2d(_f64(x)))
    Wf = _f32(W)
    R, k = x.shape
    assert Wf.shape[1] == k
    y = np.zeros((R, Wf.shape[0]))
    am = None
    if amax is not None:
        assert amax.dtype == np.float64 and amax.size == 1
        am = _dptr(amax)
    rc = lib().orc_project_rows(_dptr(x), R, k, _fptr(Wf), Wf.shape[0], int(fp8), float(xs), am,
                                _dptr(y))
    if rc:
        raise ValueError("oracle rejected the projection")
    return y


def calibrate(cfg: Config, w, S, ns):
    """Per-tensor FP8 scales from a calibration sample: the encode of users S
    and the scoring of their candidates ns with per-row FP8 scales, recording
    each projection input's max |x|; scale = amax / 448 (1 where amax is 0).
    Returns (scales, amax), each [layers][1 + n_ns][4]."""
    c1 = Config(cfg.layers, cfg.d, cfg.heads, cfg.ffn, cfg.n_ns, cfg.L0, list(cfg.q), cfg.eps,
                FP8_ROW)
    amax = np.zeros(c1.scale_shape())
    W = _weights(w)
    kv, _ = encode_user(c1, W, S, amax=amax)
    score_candidates(c1, W, kv, ns, amax=amax)
    # the scales as the GPU holds them (fp32), so both sides quantise alike
    scales = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32).astype(np.float64)
    return scales, amax


def full_forward(cfg: Config, w, S, ns):
    """The oracle's full forward: encode the S-side once, then score every
    candidate against it.  Returns (s_out [U,q_last,d], kv [U,kv], ns_out)."""
    W = _weights(w)
    kv, s_out = encode_user(cfg, W, S)
    return s_out, kv, score_candidates(cfg, W, kv, ns)


def rel_l2(got, ref) -> float:
    """||got - ref||_2 / ||ref||_2 in fp64."""
    got = _f64(got).ravel()
    ref = _f64(ref).ravel()
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    return float(num / den) if den > 0 else float(num)
