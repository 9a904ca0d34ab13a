"""ctypes binding of libonetrans.so (argument marshalling only).

The functions keep the C names (``ot_model_create``, ``ot_encode_user``, ...)
and take plain integers / pointers; :class:`Model` wraps them for torch CUDA
tensors.  Every step of the forward runs in the library's CUDA kernels: there
is no CPU or PyTorch fallback, and a missing or unloadable library raises.
"""

from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# OT_CHECKED=1: the debug build with device bounds checks (build --checked)
LIB_PATH = os.path.join(HERE, "_lib", "libonetrans_checked.so" if os.environ.get("OT_CHECKED") == "1"
                        else "libonetrans.so")
MAX_LAYERS = 32

OT_OK = 0
STATUS = {0: "OT_OK", 1: "OT_ERR_ARG", 2: "OT_ERR_SHAPE", 3: "OT_ERR_DTYPE", 4: "OT_ERR_ALIGN",
          5: "OT_ERR_CACHE_TOO_SMALL", 6: "OT_ERR_WORKSPACE_TOO_SMALL", 7: "OT_ERR_CUDA",
          8: "OT_ERR_DEVICE_TIMEOUT", 9: "OT_ERR_DEVICE_BOUNDS", 10: "OT_ERR_UNSUPPORTED"}
DTYPES = {"f32": 0, "bf16": 1, "fp8": 2}

# Every function the header declares, with (restype, argtypes).
_vp, _i, _l, _ll, _sz = C.c_void_p, C.c_int, C.c_long, C.c_longlong, C.c_size_t


class OtConfig(C.Structure):
    _fields_ = [("layers", C.c_int), ("d", C.c_int), ("heads", C.c_int), ("ffn", C.c_int),
                ("n_ns", C.c_int), ("L0", C.c_int), ("q", C.c_int * MAX_LAYERS), ("F", C.c_int),
                ("eps", C.c_float), ("dtype", C.c_int), ("full_attn", C.c_int),
                ("moe_experts", C.c_int), ("moe_topk", C.c_int)]


WEIGHT_NAMES = ("Wqkv_s", "Wo_s", "W1_s", "W2_s", "g1_s", "g2_s", "Wqkv_ns", "Wo_ns", "W1_ns",
                "W2_ns", "g1_ns", "g2_ns", "W_split")
# a mixture of experts as the S-side FFN (ot_config.moe_experts > 0)
MOE_WEIGHT_NAMES = ("W_router", "W1_moe", "W2_moe")


class OtWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in WEIGHT_NAMES + MOE_WEIGHT_NAMES]


# the tensors ot_full_backward differentiates (fp32, gains not folded)
GRAD_NAMES = WEIGHT_NAMES[:12]


class OtGrads(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in GRAD_NAMES + MOE_WEIGHT_NAMES]


class OtLaunchRecord(C.Structure):
    _fields_ = [("kind", C.c_int), ("role", C.c_int), ("ms", C.c_float), ("flops", C.c_double),
                ("bytes", C.c_double)]


KINDS = {0: "gemm_tc", 1: "gemm_simt", 2: "attn_tc", 3: "attn_simt", 4: "gather", 5: "quant",
         6: "ffn_tc", 7: "attn_ns", 8: "kv_grow", 9: "moe"}
ROLES = {0: "S_QKV", 1: "S_attn", 2: "S_O", 3: "S_FFN1", 4: "S_FFN2", 5: "NS_QKV", 6: "NS_attn",
         7: "NS_O", 8: "NS_FFN1", 9: "NS_FFN2", 10: "auto_split", 11: "other", 12: "S_FFN",
         13: "NS_FFN", 14: "O", 15: "FFN", 16: "QKV", 17: "S_MoE"}

SIGNATURES = {
    "ot_model_create": (_i, [C.POINTER(OtConfig), C.POINTER(OtWeights), C.POINTER(_vp)]),
    "ot_model_destroy": (None, [_vp]),
    "ot_kv_cache_bytes": (_sz, [_vp, _i]),
    "ot_workspace_bytes": (_sz, [_vp, _i, _i]),
    "ot_auto_split": (_i, [_vp, _vp, _l, _vp, _vp]),
    "ot_embed_gather": (_i, [_vp, _l, _i, _vp, _l, _vp, _vp, _vp]),
    "ot_encode_user": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _sz, _vp]),
    "ot_score_candidates": (_i, [_vp, _vp, _i, _vp, _i, _vp, _vp, _sz, _vp]),
    "ot_full_forward": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "ot_host_workspace_bytes": (_sz, [_vp, _i, _i]),
    "ot_full_forward_host": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "ot_poll_device_error": (_i, [_vp, _vp]),
    "ot_set_wait_limit": (_i, [_vp, _ll]),
    "ot_set_kernel_path": (_i, [_vp, _i]),
    "ot_status_str": (C.c_char_p, [_i]),
    "ot_launch_count": (_ll, [_vp]),
    "ot_profile_enable": (_i, [_vp, _i]),
    "ot_profile_read": (_i, [_vp, C.POINTER(OtLaunchRecord), _i]),
    "ot_score_candidates_noalloc": (_i, [_vp, _vp, _i, _vp, _i, _vp, _vp]),
    "ot_encode_append": (_i, [_vp, _vp, _i, _vp, _i, _vp, _vp, _vp, _sz, _vp]),
    "ot_append_workspace_bytes": (_sz, [_vp, _i, _i]),
    "ot_set_act_scales": (_i, [_vp, _vp]),
    "ot_kv_pages_per_user": (_i, [_vp]),
    "ot_kv_page_bytes": (_sz, [_vp]),
    "ot_encode_user_paged": (_i, [_vp, _vp, _i, _vp, _ll, _vp, _vp, _vp, _sz, _vp]),
    "ot_score_candidates_paged": (_i, [_vp, _vp, _ll, _vp, _i, _vp, _i, _vp, _vp, _sz, _vp]),
    "ot_fp8_calibrate": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp, _sz, _vp]),
    "ot_backward_workspace_bytes": (_sz, [C.POINTER(OtConfig), _i, _i]),
    "ot_backward_launches": (_ll, [C.POINTER(OtConfig), _i, _i]),
    "ot_full_backward": (_i, [C.POINTER(OtConfig), C.POINTER(OtWeights), _vp, _vp, _i, _i, _vp,
                              _vp, _vp, _vp, C.POINTER(OtGrads), _vp, _vp, _vp, _sz, _vp]),
}

_lib = None


def lib():
    """Load libonetrans.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libonetrans.so not built ({LIB_PATH}); run "
                              "python -m unified_transformer_recommender_onetrans_b200.build")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class OtError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


def check(code: int, where: str) -> None:
    if code != OT_OK:
        raise OtError(code, where)


def pyramid_schedule(L0: int, q_end: int | None, layers: int) -> list[int]:
    """S query tail per layer, linear from L0 to q_end (ties to even).

    Integer form of q_l = L0 - (L0 - q_end) * l / (layers - 1): numerator
    num = L0 * (layers - 1) - (L0 - q_end) * l over den = layers - 1."""
    if q_end is None or layers == 1:
        return [L0] * layers
    den = layers - 1
    out = []
    for l in range(layers):
        num = L0 * den - (L0 - q_end) * l
        qd, rem = divmod(num, den)
        if 2 * rem > den or (2 * rem == den and qd % 2 == 1):
            qd += 1
        out.append(qd)
    return out


# ------------------------------------------------------------------ torch face
def _host_ptr(t) -> int:
    """Address of a pinned, contiguous host tensor (ot_full_forward_host)."""
    if t.is_cuda or not t.is_pinned():
        raise ValueError("host buffers passed to the library must be pinned CPU tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _ptr(t) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


class Model:
    """A OneTrans block stack living on the current CUDA device.

    ``weights``: dict of CUDA tensors in the storage dtype (see
    include/onetrans.h for layouts).  ``q``: S query tail per layer.
    """

    def __init__(self, *, layers, d, heads, ffn, n_ns, L0, q, F=0, eps=1e-6, dtype="bf16",
                 weights: dict, full_attn: bool = False, moe_experts: int = 0, moe_topk: int = 1):
        import torch
        if not torch.cuda.is_available():
            raise RuntimeError("the OneTrans library needs a CUDA GPU")
        self.layers, self.d, self.heads, self.ffn, self.n_ns, self.L0 = (layers, d, heads, ffn,
                                                                         n_ns, L0)
        self.q, self.F, self.eps, self.dtype = list(q), F, eps, dtype
        self.storage = torch.float32 if dtype == "f32" else torch.bfloat16
        cfg = OtConfig()
        cfg.layers, cfg.d, cfg.heads, cfg.ffn, cfg.n_ns, cfg.L0 = layers, d, heads, ffn, n_ns, L0
        for i, v in enumerate(self.q):
            cfg.q[i] = int(v)
        cfg.F, cfg.eps, cfg.dtype = F, eps, DTYPES[dtype]
        cfg.full_attn = int(bool(full_attn))
        self.full_attn = bool(full_attn)
        cfg.moe_experts, cfg.moe_topk = int(moe_experts), int(moe_topk)
        self.moe_experts, self.moe_topk = int(moe_experts), int(moe_topk)
        self._cfg = cfg
        self._w = {k: weights[k].contiguous() for k in WEIGHT_NAMES + MOE_WEIGHT_NAMES
                   if weights.get(k) is not None}
        for k, t in self._w.items():
            if t.dtype != self.storage:
                raise ValueError(f"weight {k} must be {self.storage}")
        w = OtWeights(**{k: _ptr(self._w.get(k)) for k in WEIGHT_NAMES + MOE_WEIGHT_NAMES})
        h = C.c_void_p()
        check(lib().ot_model_create(C.byref(cfg), C.byref(w), C.byref(h)), "ot_model_create")
        self.handle = h
        self._w = None  # the library holds its own copies

    def close(self):
        if getattr(self, "handle", None):
            lib().ot_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # sizes
    def kv_cache_bytes(self, users: int) -> int:
        return int(lib().ot_kv_cache_bytes(self.handle, users))

    def workspace_bytes(self, users: int, cands: int = 0) -> int:
        return int(lib().ot_workspace_bytes(self.handle, users, cands))

    def rows_at(self, l: int) -> int:
        return self.L0 if l == 0 else self.q[l - 1]

    def kv_layer_offset(self, l: int) -> int:
        return sum(2 * self.d * self.rows_at(j) for j in range(l))

    def kv_layer(self, kv_user, l: int):
        """(K, V) views [L_l, d] of layer l from one user's cache row."""
        off, L, d = self.kv_layer_offset(l), self.rows_at(l), self.d
        return (kv_user[off: off + L * d].view(L, d), kv_user[off + L * d: off + 2 * L * d].view(L, d))

    def _ws(self, ws, nbytes):
        import torch
        if ws is None:
            ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
        return ws

    def set_kernel_path(self, path: int):
        check(lib().ot_set_kernel_path(self.handle, path), "ot_set_kernel_path")

    def set_wait_limit(self, polls: int):
        check(lib().ot_set_wait_limit(self.handle, polls), "ot_set_wait_limit")

    def profile(self, enable: bool = True):
        check(lib().ot_profile_enable(self.handle, int(enable)), "ot_profile_enable")

    def profile_read(self, max_records: int = 1 << 16):
        """List of dicts (kind, role, ms, flops, bytes) since the last read."""
        buf = (OtLaunchRecord * max_records)()
        n = lib().ot_profile_read(self.handle, buf, max_records)
        if n < 0:
            raise OtError(-n, "ot_profile_read")
        return [dict(kind=KINDS.get(r.kind, r.kind), role=ROLES.get(r.role, r.role), ms=r.ms,
                     flops=r.flops, bytes=r.bytes) for r in buf[:n]]

    def launch_count(self) -> int:
        return int(lib().ot_launch_count(self.handle))

    def poll(self, stream=None):
        check(lib().ot_poll_device_error(self.handle, _stream(stream)), "device")

    # calls
    def new_kv_cache(self, users: int):
        import torch
        elems = self.kv_cache_bytes(users) // (4 if self.dtype == "f32" else 2)
        return torch.empty((users, elems // max(users, 1)), dtype=self.storage, device="cuda")

    def auto_split(self, x, ns=None, stream=None):
        import torch
        lead = x.shape[:-1]
        M = x.numel() // x.shape[-1]
        if ns is None:
            ns = torch.empty(*lead, self.n_ns, self.d, dtype=self.storage, device=x.device)
        check(lib().ot_auto_split(self.handle, _ptr(x), M, _ptr(ns), _stream(stream)),
              "ot_auto_split")
        return ns

    def encode_user(self, S, kv=None, out_s_tail=None, ws=None, want_s_tail=True, stream=None):
        import torch
        U = S.shape[0]
        if kv is None:
            kv = self.new_kv_cache(U)
        if out_s_tail is None and want_s_tail:
            out_s_tail = torch.empty(U, self.q[-1], self.d, dtype=self.storage, device=S.device)
        nb = self.workspace_bytes(U, 0)
        ws = self._ws(ws, nb)
        check(lib().ot_encode_user(self.handle, _ptr(S), U, _ptr(kv), _ptr(out_s_tail), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)),
              "ot_encode_user")
        return kv, out_s_tail

    def append_workspace_bytes(self, users: int, delta: int) -> int:
        return int(lib().ot_append_workspace_bytes(self.handle, users, delta))

    def encode_append(self, kv_old, S_new, kv=None, out_new=None, ws=None, stream=None):
        """Append S_new [U, delta, d] to users whose cache kv_old was written
        by a model with L0 - delta and q[l] - delta (ot_encode_append); this
        model is the grown one.  Returns (grown cache, the new rows' outputs
        of the last layer [U, delta, d])."""
        import torch
        U, delta = S_new.shape[0], S_new.shape[1]
        if kv is None:
            kv = self.new_kv_cache(U)
        if out_new is None:
            out_new = torch.empty(U, delta, self.d, dtype=self.storage, device=S_new.device)
        ws = self._ws(ws, self.append_workspace_bytes(U, delta))
        check(lib().ot_encode_append(self.handle, _ptr(kv_old), U, _ptr(S_new), delta, _ptr(kv),
                                     _ptr(out_new), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(stream)), "ot_encode_append")
        return kv, out_new

    def score_candidates(self, kv, ns, out=None, ws=None, stream=None):
        import torch
        U, Cn = ns.shape[0], ns.shape[1]
        if out is None:
            out = torch.empty_like(ns)
        ws = self._ws(ws, self.workspace_bytes(U, Cn))
        check(lib().ot_score_candidates(self.handle, _ptr(kv), U, _ptr(ns), Cn, _ptr(out),
                                        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
              "ot_score_candidates")
        return out

    def score_candidates_noalloc(self, kv, ns, out=None, stream=None):
        """score_candidates into the library's fixed device scratch (no
        workspace, no allocation inside the call); see the header for the
        size limit and the sharing rules."""
        import torch
        U, Cn = ns.shape[0], ns.shape[1]
        if out is None:
            out = torch.empty_like(ns)
        check(lib().ot_score_candidates_noalloc(self.handle, _ptr(kv), U, _ptr(ns), Cn, _ptr(out),
                                                _stream(stream)), "ot_score_candidates_noalloc")
        return out

    def full_forward(self, S, ns, kv=None, out_s_tail=None, out_ns=None, ws=None, stream=None):
        import torch
        B, Cn = ns.shape[0], ns.shape[1]
        if out_s_tail is None:
            out_s_tail = torch.empty(B, self.q[-1], self.d, dtype=self.storage, device=S.device)
        if out_ns is None:
            out_ns = torch.empty_like(ns)
        ws = self._ws(ws, self.workspace_bytes(B, Cn))
        check(lib().ot_full_forward(self.handle, _ptr(S), _ptr(ns), B, Cn, _ptr(out_s_tail),
                                    _ptr(out_ns), _ptr(kv), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)),
              "ot_full_forward")
        return out_s_tail, out_ns

    # paged KV cache
    PAGE_ROWS = 128

    def kv_pages_per_user(self) -> int:
        return int(lib().ot_kv_pages_per_user(self.handle))

    def kv_page_bytes(self) -> int:
        return int(lib().ot_kv_page_bytes(self.handle))

    def new_page_pool(self, n_pages: int):
        """A pool of n_pages pages ([n_pages, 2, 128, d]: K rows, then V rows)."""
        import torch
        return torch.empty((n_pages, 2, self.PAGE_ROWS, self.d), dtype=self.storage, device="cuda")

    def encode_user_paged(self, S, pool, pages, out_s_tail=None, ws=None, want_s_tail=True,
                          stream=None):
        """ot_encode_user into a paged cache: pool from new_page_pool, pages an
        int32 CUDA tensor [U, kv_pages_per_user()] of page ids."""
        import torch
        U = S.shape[0]
        if out_s_tail is None and want_s_tail:
            out_s_tail = torch.empty(U, self.q[-1], self.d, dtype=self.storage, device=S.device)
        ws = self._ws(ws, self.workspace_bytes(U, 0))
        check(lib().ot_encode_user_paged(self.handle, _ptr(S), U, _ptr(pool), pool.shape[0],
                                         _ptr(pages), _ptr(out_s_tail), _ptr(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)),
              "ot_encode_user_paged")
        return out_s_tail

    def score_candidates_paged(self, pool, pages, ns, out=None, ws=None, stream=None):
        import torch
        U, Cn = ns.shape[0], ns.shape[1]
        if out is None:
            out = torch.empty_like(ns)
        ws = self._ws(ws, self.workspace_bytes(U, Cn))
        check(lib().ot_score_candidates_paged(self.handle, _ptr(pool), pool.shape[0], _ptr(pages), U,
                                              _ptr(ns), Cn, _ptr(out), _ptr(ws),
                                              ws.numel() * ws.element_size(), _stream(stream)),
              "ot_score_candidates_paged")
        return out

    def kv_from_pages(self, pool, pages_u, l: int):
        """(K, V) [L_l, d] of layer l of one user, gathered from its pages."""
        import torch
        L = self.rows_at(l)
        off = sum((self.rows_at(j) + self.PAGE_ROWS - 1) // self.PAGE_ROWS for j in range(l))
        nb = (L + self.PAGE_ROWS - 1) // self.PAGE_ROWS
        pg = pages_u[off: off + nb].long()
        K = pool[pg, 0].reshape(-1, self.d)[:L]
        V = pool[pg, 1].reshape(-1, self.d)[:L]
        return K, V

    # fp8 per-tensor scales
    def act_scale_shape(self) -> tuple:
        return (self.layers, 1 + self.n_ns, 4)

    def set_act_scales(self, scales):
        """Per-tensor FP8 activation scales [layers, 1 + n_ns, 4] (a CPU tensor
        or array; None: back to per-row scales)."""
        import numpy as np
        if scales is None:
            check(lib().ot_set_act_scales(self.handle, None), "ot_set_act_scales")
            return
        a = np.ascontiguousarray(np.asarray(scales, dtype=np.float32))
        if a.shape != self.act_scale_shape():
            raise ValueError(f"scales must have shape {self.act_scale_shape()}")
        check(lib().ot_set_act_scales(self.handle, a.ctypes.data_as(C.c_void_p)),
              "ot_set_act_scales")

    def fp8_calibrate(self, S, ns, amax=None, ws=None, stream=None):
        """Max-accumulate every projection input's max |x| over users S [U, L0,
        d] and candidates ns [U, C, N, d] into amax (a CUDA float32 tensor of
        act_scale_shape(), zeros if None) and return it."""
        import torch
        U, Cn = ns.shape[0], ns.shape[1]
        if amax is None:
            amax = torch.zeros(self.act_scale_shape(), dtype=torch.float32, device=S.device)
        ws = self._ws(ws, self.workspace_bytes(U, Cn))
        check(lib().ot_fp8_calibrate(self.handle, _ptr(S), _ptr(ns), U, Cn, _ptr(amax), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)),
              "ot_fp8_calibrate")
        return amax

    def host_workspace_bytes(self, users: int, cands: int) -> int:
        return int(lib().ot_host_workspace_bytes(self.handle, users, cands))

    def full_forward_host(self, S_host, x_host, out_s_tail_host, out_ns_host, kv=None, ws=None,
                          stream=None):
        """Auto-Split + full forward from pinned host tensors S_host [B, L0, d] and
        x_host [B, C, F] into pinned host outputs [B, q_last, d] and [B, C, N, d]
        (ot_full_forward_host).  Consecutive calls on one stream with the same
        workspace overlap the next call's input copy with this call's work."""
        B, Cn = x_host.shape[0], x_host.shape[1]
        ws = self._ws(ws, self.host_workspace_bytes(B, Cn))
        check(lib().ot_full_forward_host(self.handle, _host_ptr(S_host), _host_ptr(x_host), B, Cn,
                                         _host_ptr(out_s_tail_host), _host_ptr(out_ns_host), _ptr(kv),
                                         _ptr(ws), ws.numel() * ws.element_size(),
                                         _stream(stream)),
              "ot_full_forward_host")
        return out_s_tail_host, out_ns_host


def embed_gather(table, ids, out=None, err=None, stream=None):
    import torch
    n = ids.numel()
    d = table.shape[1]
    if out is None:
        out = torch.empty(*ids.shape, d, dtype=table.dtype, device=table.device)
    check(lib().ot_embed_gather(_ptr(table), table.shape[0], d, _ptr(ids), n, _ptr(out),
                                _ptr(err), _stream(stream)), "ot_embed_gather")
    return out


# ------------------------------------------------------------------ training
def make_config(*, layers, d, heads, ffn, n_ns, L0, q, F=0, eps=1e-6, dtype="f32",
                full_attn=False, moe_experts=0, moe_topk=1) -> OtConfig:
    cfg = OtConfig()
    cfg.layers, cfg.d, cfg.heads, cfg.ffn, cfg.n_ns, cfg.L0 = layers, d, heads, ffn, n_ns, L0
    for i, v in enumerate(q):
        cfg.q[i] = int(v)
    cfg.F, cfg.eps, cfg.dtype = F, eps, DTYPES[dtype]
    cfg.full_attn, cfg.moe_experts, cfg.moe_topk = int(bool(full_attn)), moe_experts, moe_topk
    return cfg


def backward_workspace_bytes(cfg: OtConfig, users: int, cands: int) -> int:
    return lib().ot_backward_workspace_bytes(C.byref(cfg), users, cands)


def backward_launches(cfg: OtConfig, users: int, cands: int) -> int:
    return lib().ot_backward_launches(C.byref(cfg), users, cands)


def _expect(t, shape, name):
    """A tensor handed to ot_full_backward: None, or fp32 of exactly this shape."""
    import torch
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if t.dtype != torch.float32:
        raise ValueError(f"{name} must be float32, not {t.dtype}")


def _backward_shapes(cfg: OtConfig, U: int, Cn: int) -> dict:
    """Shapes of every tensor of ot_full_backward (include/onetrans.h layouts)."""
    L, d, f, N, E = cfg.layers, cfg.d, cfg.ffn, cfg.n_ns, cfg.moe_experts
    q_last = cfg.q[L - 1]
    return {
        "Wqkv_s": (L, 3 * d, d), "Wo_s": (L, d, d), "W1_s": (L, f, d), "W2_s": (L, d, f),
        "g1_s": (L, d), "g2_s": (L, d),
        "Wqkv_ns": (L, N, 3 * d, d), "Wo_ns": (L, N, d, d), "W1_ns": (L, N, f, d),
        "W2_ns": (L, N, d, f), "g1_ns": (L, N, d), "g2_ns": (L, N, d),
        "W_router": (L, E, d), "W1_moe": (L, E, f, d), "W2_moe": (L, E, d, f),
        "S": (U, cfg.L0, d), "dS": (U, cfg.L0, d), "ns": (U, Cn, N, d), "dns": (U, Cn, N, d),
        "G_ns": (U, Cn, N, d), "out_ns": (U, Cn, N, d), "G_s": (U, q_last, d), "out_s_tail": (U, q_last, d),
    }


def full_backward(cfg: OtConfig, weights: dict, S, ns, G_s, G_ns, *, grads=None, dS=None,
                  dns=None, out_s_tail=None, out_ns=None, ws=None, want_outputs=True,
                  want_input_grads=True, stream=None):
    """ot_full_backward on fp32 CUDA tensors.  ``weights``: the twelve dense
    tensors of GRAD_NAMES (gains not folded) and, for a mixture of experts,
    those of MOE_WEIGHT_NAMES (W1_s / W2_s may then be absent).  Returns
    (s_tail, ns_out, grads, dS, dns); the gradients are those of
    sum(s_tail * G_s) + sum(ns_out * G_ns)."""
    import torch
    U, Cn = S.shape[0], (ns.shape[1] if ns is not None else 0)
    dev = S.device
    present = [k for k in GRAD_NAMES + MOE_WEIGHT_NAMES if weights.get(k) is not None]
    nbytes = backward_workspace_bytes(cfg, U, Cn)
    if nbytes > 0:
        # a configuration the library accepts (else its own status is
        # reported below): every tensor given must have its shape and fp32
        shapes = _backward_shapes(cfg, U, Cn)
        for k in present:
            _expect(weights[k], shapes[k], k)
            if grads is not None:
                _expect(grads.get(k), shapes[k], f"grads[{k}]")
        for name, t in (("S", S), ("ns", ns), ("G_s", G_s), ("G_ns", G_ns), ("out_s_tail", out_s_tail),
                        ("out_ns", out_ns), ("dS", dS), ("dns", dns)):
            _expect(t, shapes[name], name)
    if grads is None:
        grads = {k: torch.empty_like(weights[k]) for k in present}
    if want_outputs:
        if out_s_tail is None:
            out_s_tail = torch.empty(U, cfg.q[cfg.layers - 1], cfg.d, dtype=torch.float32, device=dev)
        if out_ns is None and Cn:
            out_ns = torch.empty_like(ns)
    if want_input_grads:
        if dS is None:
            dS = torch.empty_like(S)
        if dns is None and Cn:
            dns = torch.empty_like(ns)
    if ws is None:
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    w = OtWeights(**{k: _ptr(weights.get(k)) for k in GRAD_NAMES + MOE_WEIGHT_NAMES})
    g = OtGrads(**{k: _ptr(grads.get(k)) for k in GRAD_NAMES + MOE_WEIGHT_NAMES})
    check(lib().ot_full_backward(C.byref(cfg), C.byref(w), _ptr(S), _ptr(ns) if Cn else 0, U, Cn,
                                 _ptr(G_s), _ptr(G_ns) if Cn else 0, _ptr(out_s_tail),
                                 _ptr(out_ns) if Cn else 0, C.byref(g), _ptr(dS),
                                 _ptr(dns) if Cn else 0, _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)),
          "ot_full_backward")
    return out_s_tail, out_ns, grads, dS, dns
