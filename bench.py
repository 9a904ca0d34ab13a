"""Throughput of the OneTrans block-stack forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload onetrans_s_full]

One step = one pass of the whole hot path over one batch: Auto-Split of the
static features into NS tokens, then the full forward (every layer's S QKV
GEMM with the KV-cache store, pyramid-tail S attention, O / FFN GEMMs, and the
NS side: grouped private-weight GEMMs and NS attention against the cache).
Default workload: OneTransS-shaped full forward, 6 layers, d=256, 4 heads,
16 NS tokens, 1190 S tokens (1190 -> 12 pyramid), 64 users x 1 candidate.
Metric: S-tokens/s = users * L0 / step time.

N > 1 (one process per GPU, launched by torch.distributed.run): every rank runs
its own replica on its own 64 users (weak scaling, no data-path collective);
timing is the max over ranks of the device time.

--impl reference times the CPU fp64 oracle on this machine's cores on a
bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of the dominant kernel (dram__bytes_read.sum + dram__bytes_write.sum),
# summed over the launches of one step, from one ncu capture of the default
# workload (the capture is summarised in profiles/, with its command).  It is
# reported only while the kernel's source is the one that was captured.
CAPTURED_TRAFFIC = {
    # kernel kind -> (source file, its sha256 at capture time, bytes per step, launches per step)
    # attn_tc: ncu dram__bytes_read.sum + dram__bytes_write.sum of the six S-attention launches
    # of one onetrans_s_full step (651.1 MB read + 34.4 MB written)
    "attn_tc": ("ot_attn_tc.cu", "4e9ab25b647c2a37ce94733adfd370f3024a6f8845cc1d9215fbd9a7504b1ec8",
                685544192, 6),
    # ffn_tc: the six fused O-projection + FFN launches of one onetrans_s_full step
    # (363.4 MB read + 20.6 MB written)
    "ffn_tc": ("ot_ffn_tc.cu", "675fae658dab54517d2954da43f31073cedb641fd3c4be7f406e1fea356bc07d",
               383966464, 6),
}


def metric_name(wl) -> str:
    """The headline metric's name: the same string in both arms."""
    return f"S-tokens/s ({wl.name} full forward)"


def captured_traffic(kind: str):
    """(bytes per step, note) of the last ncu capture of `kind`, or (None, why)."""
    import hashlib
    ent = CAPTURED_TRAFFIC.get(kind)
    if ent is None:
        return None, "no ncu capture recorded for this kernel"
    src, sha, nbytes, launches = ent
    path = os.path.join(ROOT, "unified_transformer_recommender_onetrans_b200", "csrc", src)
    with open(path, "rb") as fh:
        if hashlib.sha256(fh.read()).hexdigest() != sha:
            return None, f"{src} changed since the ncu capture"
    return nbytes, f"ncu dram__bytes_read.sum + dram__bytes_write.sum over {launches} launches"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled while active: the
    nvidia-smi query loop (every 200 ms) plus an NVML poll every 10 ms, so a
    timed region of a few tens of milliseconds still holds samples."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int, uuid: str | None = None):
        self.gpu = gpu_index
        self.uuid = uuid
        self.proc = None
        self.lines = []     # (host time, nvidia-smi csv line)
        self.nvml = []      # (host time, sm MHz, max MHz, reason names)
        self.t0, self.t1 = float("-inf"), float("inf")
        self._stop = threading.Event()
        self._poll = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.uuid:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            except pynvml.NVMLError:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll_nvml(self):
        try:
            nv, h = self._nvml_handle()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            while not self._stop.is_set():
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.nvml.append((time.monotonic(), sm, mx,
                                  [k for k, v in bits.items() if r & v]))
                self._stop.wait(0.01)
        except Exception:  # NVML missing or refused: nvidia-smi samples remain
            return

    def start(self):
        """Start both samplers and wait (up to 10 s) for nvidia-smi's first
        line, so sampling is running when the timed region opens."""
        self._poll = threading.Thread(target=self._poll_nvml, daemon=True)
        self._poll.start()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t_end = time.monotonic() + 10.0
        while not self.lines and time.monotonic() < t_end and self.proc.poll() is None:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def window(self, t0: float, t1: float):
        """Restrict the summary to samples taken between host times t0 and t1."""
        self.t0, self.t1 = t0, t1

    def stop(self):
        self._stop.set()
        if self._poll is not None:
            self._poll.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)
        sm, mx, reasons, n_smi = [], None, set(), 0
        for ts, ln in self.lines:
            if not self.t0 <= ts <= self.t1:
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            n_smi += 1
            for nm, v in zip(self.NAMES, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        n_nvml = 0
        for ts, f, m, rs in self.nvml:
            if self.t0 <= ts <= self.t1:
                sm.append(f)
                mx = m
                reasons.update(rs)
                n_nvml += 1
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "samples_nvidia_smi": n_smi, "samples_nvml": n_nvml,
                "sm_mhz_min": sm[0]}


def device_uuid(local: int):
    """NVML-style UUID of the CUDA device `local`, or None."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


def user_shard(world: int, rank: int, users_per_rank: int) -> range:
    """The users rank `rank` of `world` works on: a disjoint block of
    `users_per_rank` user indices (inputs are seeded per user, so a rank's
    block is generated exactly as that slice of one big batch would be)."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of {world}")
    return range(rank * users_per_rank, (rank + 1) * users_per_rank)


def max_over_ranks(value: float, world: int, dist, device) -> float:
    """The largest `value` over all ranks (every rank calls it, in the same
    order); the step time of a weak-scaling job is the slowest rank's."""
    if world == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ---------------------------------------------------------------- oracle (CPU)
def oracle_sample(wl, users=1, threads=0):
    """Time the oracle's full forward on `users` users of the workload (full
    sequence length, all candidates of those users).  Returns (seconds,
    S tokens processed, threads used)."""
    import torch  # noqa: F401

    from oracle import oracle as O
    from synth import gen_auto_split_features, gen_s_tokens, gen_weights

    wl1 = wl.with_(users=users)
    w = gen_weights(wl1)
    S = gen_s_tokens(wl1, weights=w)
    x = gen_auto_split_features(wl1)
    nthreads = O.set_threads(threads)
    cfg = O.Config.of(wl1)
    W = O.Weights(w)
    t0 = time.perf_counter()
    ns = O.auto_split(x, w["W_split"], wl.n_ns, wl.d)
    O.full_forward(cfg, W, S, ns)
    dt = time.perf_counter() - t0
    return dt, users * wl.L0, nthreads


def run_reference(args, wl):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    # bounded sample: one user of the workload per step (under a second on a
    # many-core host); the timed steps stop early after 150 s of oracle time
    per = []
    for _ in range(args.warmup_ref):
        oracle_sample(wl, users=1)
    cores = 0
    spent = 0.0
    for _ in range(args.steps_ref):
        dt, toks, cores = oracle_sample(wl, users=1)
        per.append(dt / toks)
        spent += dt
        if spent > 150.0:
            break
    sec_per_tok = sum(per) / len(per)
    value = 1.0 / sec_per_tok
    line = {
        "impl": "reference", "metric": metric_name(wl), "value": value,
        "unit": "S-tokens/s", "n_gpus": ws, "steps": len(per), "warmup": args.warmup_ref,
        "ms_per_step": 1e3 * sec_per_tok * wl.L0, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "users": wl.users, "cands": wl.cands, "L0": wl.L0,
                   "layers": wl.layers, "d": wl.d},
        "cpu_baseline": {"value": value, "unit": "S-tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"1 user x {wl.cands} candidate(s) of {wl.name} at full "
                                   f"length per step, C fp64 oracle, OpenMP"},
        "e2e": {"value": value, "unit": "S-tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- serving arms
def _time_device(fn, steps, flush, world, dist, dev):
    """Median device ms of `fn` over `steps` calls (CUDA events on the current
    stream, L2 flushed between calls), max over ranks."""
    import torch
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for e0, e1 in ev:
        e0.record(stream)
        fn()
        e1.record(stream)
        flush.zero_()
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(b) for a, b in ev)
    return max_over_ranks(t[len(t) // 2], world, dist, dev)


def _score_point(m, wl, U, C, x, kv, steps, flush, world, dist, dev, peaks, tensor_peak):
    """Time score_candidates (with the candidates' Auto-Split) at C candidates
    per user against an encoded cache; its roofline is the slower of the
    bytes the call must move once over HBM and its FLOPs on the tensor cores."""
    import torch

    ns = torch.empty(U, C, wl.n_ns, wl.d, dtype=m.storage, device=dev)
    out_ns = torch.empty_like(ns)
    ws = torch.empty(m.workspace_bytes(U, C), dtype=torch.uint8, device=dev)

    def score():
        m.auto_split(x, ns)
        m.score_candidates(kv, ns, out=out_ns, ws=ws)

    for _ in range(10):
        score()
    m.poll()
    ms = _time_device(score, steps, flush, world, dist, dev)
    m.poll()
    m.profile(True)
    score()
    recs = m.profile_read()
    m.profile(False)
    flops = sum(r["flops"] for r in recs)
    gemm_flops = sum(r["flops"] for r in recs if r["kind"] != "attn_tc")
    # bytes a score call must move at least once: every NS weight, the users'
    # cache, the candidates' features in, NS tokens out and W_split
    d, f, N, L = wl.d, wl.ffn, wl.n_ns, wl.layers
    wbytes = (1 if wl.dtype == "fp8" else 2) * L * N * (3 * d * d + d * d + 2 * d * f)
    min_bytes = wbytes + m.kv_cache_bytes(U) + x.numel() * 2 + out_ns.numel() * 2 + \
        N * d * wl.F * 2
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    t_hbm = min_bytes / (hbm * 1e9)
    # GEMMs at the GEMM dtype's peak, attention (always bf16) at the bf16 peak
    t_tc = gemm_flops / (tensor_peak["gemm"] * 1e12) + \
        (flops - gemm_flops) / (tensor_peak["attn"] * 1e12)
    roles = {}
    for r in recs:
        roles[r["role"]] = roles.get(r["role"], 0.0) + r["ms"]
    return {
        "cands": C,
        "roles_ms_profiled": roles,
        "candidates_per_s": world * U * C / (ms / 1e3),
        "ms": ms,
        "tflops": flops / (ms / 1e3) / 1e12,
        "min_hbm_bytes": min_bytes,
        "hbm_gbs_min_bytes": min_bytes / (ms / 1e3) / 1e9,
        "hbm_frac": min_bytes / (ms / 1e3) / 1e9 / hbm,
        "tensor_frac": t_tc / (ms / 1e3),
        "bound": "hbm" if t_hbm >= t_tc else "tensor",
        "roofline_ms": 1e3 * max(t_hbm, t_tc),
        "roofline_frac": 1e3 * max(t_hbm, t_tc) / ms,
    }


def measure_fp8_peak(dev, n=8192, seconds=2.0):
    """Dense e4m3 x e4m3 -> bf16 GEMM throughput of the library GEMM
    (torch._scaled_mm, cuBLASLt), n^3: best of 10 (burst) and back to back
    for `seconds` (sustained).  The denominator for the e4m3 GEMMs."""
    import torch
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev)
        mm = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one,  # noqa: E731
                                      out_dtype=torch.bfloat16)
        for _ in range(3):
            mm()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mm()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(1, int(seconds * 1e3 / best))
        e0.record()
        for _ in range(reps):
            mm()
        e1.record()
        torch.cuda.synchronize()
        sus = e0.elapsed_time(e1) / reps
        fl = 2.0 * n ** 3
        return {"tflops_burst": fl / (best / 1e3) / 1e12, "tflops_sustained": fl / (sus / 1e3) / 1e12,
                "how": f"torch._scaled_mm e4m3 {n}^3, best of 10 / {reps} back to back"}
    except Exception as e:  # no fp8 GEMM in this torch build
        return {"error": str(e).splitlines()[0][:200]}


def _append_point(m, wl, w, q, S, kv, delta, steps, flush, world, dist, dev):
    """Append `delta` new S tokens per user to the encoded users
    (ot_encode_append on the grown model: only the new rows run, against the
    cached K/V) against encoding the grown sequences from scratch."""
    import torch

    import unified_transformer_recommender_onetrans_b200 as ot
    from unified_transformer_recommender_onetrans_b200.binding import WEIGHT_NAMES

    U = S.shape[0]
    m2 = ot.Model(layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns,
                  L0=wl.L0 + delta, q=[v + delta for v in q], F=wl.F, eps=wl.eps, dtype=wl.dtype,
                  weights={k: w[k].to(dev) for k in WEIGHT_NAMES})
    g = torch.Generator().manual_seed(7)
    S_new = torch.randn(U, delta, wl.d, generator=g).to(S.dtype).to(dev)
    S_all = torch.cat([S, S_new], dim=1).contiguous()
    kv2 = m2.new_kv_cache(U)
    out_new = torch.empty(U, delta, wl.d, dtype=S.dtype, device=dev)
    ws_a = torch.empty(m2.append_workspace_bytes(U, delta), dtype=torch.uint8, device=dev)
    ws_e = torch.empty(m2.workspace_bytes(U, 0), dtype=torch.uint8, device=dev)

    def append():
        m2.encode_append(kv, S_new, kv=kv2, out_new=out_new, ws=ws_a)

    def reencode():
        m2.encode_user(S_all, kv=kv2, ws=ws_e, want_s_tail=False)

    for _ in range(10):
        append()
        reencode()
    m2.poll()
    app_ms = _time_device(append, steps, flush, world, dist, dev)
    enc_ms = _time_device(reencode, steps, flush, world, dist, dev)
    m2.poll()
    del m2, kv2, ws_a, ws_e
    return {"delta": delta, "ms": app_ms, "new_s_tokens_per_s": world * U * delta / (app_ms / 1e3),
            "reencode_ms": enc_ms, "speedup_vs_reencode": enc_ms / app_ms}


def run_serving(name, steps, flush, world, dist, dev, peaks, cands=None, sweep=None, append_rows=0):
    """Encode once per user, then score every candidate against the cache
    (Auto-Split of the candidates' features included in scoring); with
    `sweep`, score the same cache again at each candidate count in it; with
    `append_rows`, also time appending that many S tokens per user."""
    import torch

    import unified_transformer_recommender_onetrans_b200 as ot
    from synth import (WORKLOADS, gen_auto_split_features, gen_embedding_table, gen_s_tokens,
                       gen_weights, gen_zipf_ids)
    from unified_transformer_recommender_onetrans_b200.binding import WEIGHT_NAMES

    wl = WORKLOADS[name]
    if cands is not None:
        wl = wl.with_(cands=cands)
    w = gen_weights(wl)
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers)
    m = ot.Model(layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns, L0=wl.L0,
                 q=q, F=wl.F, eps=wl.eps, dtype=wl.dtype,
                 weights={k: w[k].to(dev) for k in WEIGHT_NAMES})
    U, C = wl.users, wl.cands
    out = {"workload": name, "users": U, "cands": C, "dtype": wl.dtype}
    if wl.zipf_s is not None:
        table = gen_embedding_table(wl).to(dev)
        ids = gen_zipf_ids(wl).to(dev)
        S = torch.empty(U, wl.L0, wl.d, dtype=torch.bfloat16, device=dev)
        gather = lambda: ot.embed_gather(table, ids, out=S)  # noqa: E731
        del w
    else:
        S = gen_s_tokens(wl, weights=w).to(dev)
        gather = None
    x = gen_auto_split_features(wl).to(dev)
    kv = m.new_kv_cache(U)
    if wl.dtype == "fp8":
        # per-tensor activation scales from a calibration sample (user 0 and
        # 8 of its candidates): amax of every projection input / 448
        if gather:
            gather()
        ns_cal = m.auto_split(x[:1, :8].contiguous())
        amax = m.fp8_calibrate(S[:1].contiguous(), ns_cal)
        m.poll()
        scales = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).cpu()
        m.set_act_scales(scales)
        out["fp8_scales"] = "per-tensor, calibrated on user 0 x 8 candidates (ot_fp8_calibrate)"
        del ns_cal
    ws = torch.empty(m.workspace_bytes(U, 0), dtype=torch.uint8, device=dev)

    def encode():
        if gather:
            gather()
        m.encode_user(S, kv=kv, ws=ws, want_s_tail=False)

    for _ in range(10):
        encode()
    m.poll()
    enc_ms = _time_device(encode, steps, flush, world, dist, dev)
    m.poll()
    m.profile(True)
    encode()
    enc_flops = sum(r["flops"] for r in m.profile_read())
    m.profile(False)
    out.update({
        "encode_s_tokens_per_s": world * U * wl.L0 / (enc_ms / 1e3),
        "encode_ms": enc_ms,
        "encode_tflops": enc_flops / (enc_ms / 1e3) / 1e12,
    })
    if append_rows and gather is None:
        out["append"] = _append_point(m, wl, w, q, S, kv, append_rows, steps, flush, world, dist, dev)
    bf16_peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    tensor_peak = {"gemm": bf16_peak, "attn": bf16_peak}
    peak_note = f"{peaks['_source']} bf16 dense sustained"
    if wl.dtype == "fp8":
        fp8 = measure_fp8_peak(dev)
        out["fp8_peak"] = fp8
        if fp8.get("tflops_sustained"):
            tensor_peak["gemm"] = fp8["tflops_sustained"]
            peak_note += "; GEMMs: e4m3 measured here (cuBLASLt, sustained)"
    del ws
    pt = _score_point(m, wl, U, C, x, kv, steps, flush, world, dist, dev, peaks, tensor_peak)
    out.update({"score_" + k: v for k, v in pt.items()})
    out["score_peak_source"] = peak_note
    if sweep:
        out["score_c_sweep"] = []
        for c in sweep:
            wc = wl.with_(cands=c)
            xc = gen_auto_split_features(wc).to(dev)
            out["score_c_sweep"].append(
                _score_point(m, wc, U, c, xc, kv, steps, flush, world, dist, dev, peaks,
                             tensor_peak))
            del xc
            torch.cuda.empty_cache()
    m.close()
    return out


def run_moe_point(name, experts, topk, steps, flush, world, dist, dev, peaks):
    """The workload's full forward with a sparse mixture of `experts` experts
    (top-`topk`) as the S-side FFN: router, experts and combine timed with
    the rest of the step; seeded random router and experts of the dense FFN's
    shape."""
    import torch

    import unified_transformer_recommender_onetrans_b200 as ot
    from synth import WORKLOADS, gen_auto_split_features, gen_s_tokens, gen_weights
    from unified_transformer_recommender_onetrans_b200.binding import MOE_WEIGHT_NAMES, WEIGHT_NAMES

    wl = WORKLOADS[name]
    w = gen_weights(wl)
    g = torch.Generator().manual_seed(11)
    L, d, f, E = wl.layers, wl.d, wl.ffn, experts
    w["W_router"] = (torch.randn(L, E, d, generator=g) * d ** -0.5).to(torch.bfloat16)
    w["W1_moe"] = (torch.randn(L, E, f, d, generator=g) * d ** -0.5).to(torch.bfloat16)
    w["W2_moe"] = (torch.randn(L, E, d, f, generator=g) * f ** -0.5).to(torch.bfloat16)
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers)
    m = ot.Model(layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns, L0=wl.L0,
                 q=q, F=wl.F, eps=wl.eps, dtype=wl.dtype, moe_experts=E, moe_topk=topk,
                 weights={k: w[k].to(dev) for k in WEIGHT_NAMES + MOE_WEIGHT_NAMES})
    U, C = wl.users, wl.cands
    S = gen_s_tokens(wl, weights=w).to(dev)
    x = gen_auto_split_features(wl).to(dev)
    del w
    ns = torch.empty(U, C, wl.n_ns, wl.d, dtype=m.storage, device=dev)
    out_ns = torch.empty_like(ns)
    s_tail = torch.empty(U, q[-1], wl.d, dtype=m.storage, device=dev)
    kv = m.new_kv_cache(U)
    ws = torch.empty(m.workspace_bytes(U, C), dtype=torch.uint8, device=dev)

    def step():
        m.auto_split(x, ns)
        m.full_forward(S, ns, kv=kv, out_s_tail=s_tail, out_ns=out_ns, ws=ws)

    for _ in range(5):
        step()
    m.poll()
    ms = _time_device(step, steps, flush, world, dist, dev)
    m.poll()
    m.profile(True)
    step()
    recs = m.profile_read()
    m.profile(False)
    m.close()
    by_role = {}
    for r in recs:
        by_role[r["role"]] = by_role.get(r["role"], 0.0) + r["ms"]
    flops = sum(r["flops"] for r in recs)
    return {"workload": name, "moe_experts": E, "moe_topk": topk, "users": U, "cands": C,
            "full_forward_ms": ms, "full_forward_s_tokens_per_s": world * U * wl.L0 / (ms / 1e3),
            "algorithmic_tflops": flops / (ms / 1e3) / 1e12,
            "ms_by_role_serialised": by_role}


def forward_flops(wl, q, U, C):
    """Algorithmic FLOPs of one forward of U users x C candidates: (all,
    attention only).  The projections and FFNs of both sides, and 4 d FLOPs
    per attended (query, key) pair (Q K^T and P V)."""
    d, f, N = wl.d, wl.ffn, wl.n_ns
    L, total, attn = wl.L0, 0.0, 0.0
    RN = U * C * N
    for ql in q:
        pairs_s = ql * (L - ql) + ql * (ql + 1) // 2
        pairs_ns = N * L + N * (N + 1) // 2
        a = 4.0 * d * U * pairs_s + 4.0 * d * U * C * pairs_ns
        attn += a
        # S side: K and V of all L rows, Q, O and the FFN of the ql tail rows
        total += a + 2.0 * U * (2 * L + ql) * d * d + 2.0 * U * ql * d * d + 4.0 * U * ql * d * f
        total += 2.0 * RN * 3 * d * d + 2.0 * RN * d * d + 4.0 * RN * d * f
        L = ql
    return total, attn


def run_backward_point(name, users, steps, flush, world, dist, dev, peaks):
    """One training step of the workload's shapes in fp32 through
    ot_full_backward: checkpointing forward, then per layer (top first) the
    recomputed forward and the gradients of every weight, gain and input.
    Synthetic S rows of the workload, seeded NS rows and upstream gradients."""
    import torch

    import unified_transformer_recommender_onetrans_b200 as ot
    from synth import WORKLOADS, gen_s_tokens, gen_weights

    wl = WORKLOADS[name].with_(dtype="f32", users=users, cands=1)
    w = gen_weights(wl)
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers)
    cfg = ot.make_config(layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns,
                         L0=wl.L0, q=q, eps=wl.eps)
    U, C = wl.users, wl.cands
    g = torch.Generator().manual_seed(21)
    S = gen_s_tokens(wl, weights=w).to(dev)
    ns = torch.randn(U, C, wl.n_ns, wl.d, generator=g).to(dev)
    G_s = torch.randn(U, q[-1], wl.d, generator=g).to(dev)
    G_ns = torch.randn(U, C, wl.n_ns, wl.d, generator=g).to(dev)
    wd = {k: w[k].to(dev) for k in ot.GRAD_NAMES}
    del w
    grads = {k: torch.empty_like(wd[k]) for k in ot.GRAD_NAMES}
    dS, dns = torch.empty_like(S), torch.empty_like(ns)
    s_tail = torch.empty(U, q[-1], wl.d, device=dev)
    out_ns = torch.empty_like(ns)
    ws = torch.empty(ot.backward_workspace_bytes(cfg, U, C), dtype=torch.uint8, device=dev)

    def step():
        ot.full_backward(cfg, wd, S, ns, G_s, G_ns, grads=grads, dS=dS, dns=dns,
                         out_s_tail=s_tail, out_ns=out_ns, ws=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ms = _time_device(step, steps, flush, world, dist, dev)
    F, F_attn = forward_flops(wl, q, U, C)
    # fp32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 FLOPs x max SM clock
    fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12
    model = 3 * F / (ms / 1e3) / 1e12
    executed = (4 * F - F_attn) / (ms / 1e3) / 1e12
    return {"workload": name, "dtype": "f32", "training_step": "ot_full_backward (checkpointed)",
            "users": U, "cands": C, "ms": ms, "s_tokens_per_s": world * U * wl.L0 / (ms / 1e3),
            "launches": ot.backward_launches(cfg, U, C),
            "model_tflops": model, "executed_tflops": executed,
            "fp32_peak_tflops": fp32_peak, "executed_frac_fp32_peak": executed / fp32_peak,
            "flops_rule": "model = 3 x forward FLOPs (forward + backward); executed adds the "
                          "recomputed forward without its attention (kept from the checkpointing "
                          "pass)"}


def run_full_point(name, steps, flush, world, dist, dev, peaks):
    """Auto-Split + full forward of a whole workload batch (C candidates per
    user, S and NS sides in one call), 10 warm-ups + median of `steps` calls."""
    import torch

    import unified_transformer_recommender_onetrans_b200 as ot
    from synth import WORKLOADS, gen_auto_split_features, gen_s_tokens, gen_weights
    from unified_transformer_recommender_onetrans_b200.binding import WEIGHT_NAMES

    wl = WORKLOADS[name]
    w = gen_weights(wl)
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers)
    m = ot.Model(layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns, L0=wl.L0,
                 q=q, F=wl.F, eps=wl.eps, dtype=wl.dtype,
                 weights={k: w[k].to(dev) for k in WEIGHT_NAMES})
    U, C = wl.users, wl.cands
    S = gen_s_tokens(wl, weights=w).to(dev)
    x = gen_auto_split_features(wl).to(dev)
    del w
    ns = torch.empty(U, C, wl.n_ns, wl.d, dtype=m.storage, device=dev)
    out_ns = torch.empty_like(ns)
    s_tail = torch.empty(U, q[-1], wl.d, dtype=m.storage, device=dev)
    kv = m.new_kv_cache(U)
    ws = torch.empty(m.workspace_bytes(U, C), dtype=torch.uint8, device=dev)

    def step():
        m.auto_split(x, ns)
        m.full_forward(S, ns, kv=kv, out_s_tail=s_tail, out_ns=out_ns, ws=ws)

    for _ in range(10):
        step()
    m.poll()
    ms = _time_device(step, steps, flush, world, dist, dev)
    m.poll()
    m.profile(True)
    step()
    flops = sum(r["flops"] for r in m.profile_read())
    m.profile(False)
    m.close()
    tf = flops / (ms / 1e3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    return {"workload": name, "users": U, "cands": C, "dtype": wl.dtype, "full_forward_ms": ms,
            "full_forward_s_tokens_per_s": world * U * wl.L0 / (ms / 1e3),
            "full_forward_tflops": tf, "full_forward_tensor_frac": tf / peak,
            "peak_source": f"{peaks['_source']} bf16 dense sustained (whole calls back to back)"}


# ---------------------------------------------------------------- our arm
def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    import unified_transformer_recommender_onetrans_b200 as ot
    from synth import gen_auto_split_features, gen_s_tokens, gen_weights
    from unified_transformer_recommender_onetrans_b200.binding import WEIGHT_NAMES

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    ot.lib()
    dev = torch.device("cuda", local)

    w = gen_weights(wl)
    shard = user_shard(world, rank, wl.users)
    S_cpu = gen_s_tokens(wl, users=shard, weights=w)
    x_cpu = gen_auto_split_features(wl, users=shard)
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers)
    m = ot.Model(layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns, L0=wl.L0,
                 q=q, F=wl.F, eps=wl.eps, dtype=wl.dtype,
                 weights={k: w[k].to(dev) for k in WEIGHT_NAMES})
    U, C = wl.users, wl.cands
    S = S_cpu.to(dev)
    x = x_cpu.to(dev)
    ns = torch.empty(U, C, wl.n_ns, wl.d, dtype=m.storage, device=dev)
    out_ns = torch.empty_like(ns)
    s_tail = torch.empty(U, q[-1], wl.d, dtype=m.storage, device=dev)
    kv = m.new_kv_cache(U)
    ws = torch.empty(m.workspace_bytes(U, C), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream()

    def step():
        m.auto_split(x, ns)
        m.full_forward(S, ns, kv=kv, out_s_tail=s_tail, out_ns=out_ns, ws=ws)

    for _ in range(args.warmup):
        step()
        flush.zero_()
    m.poll()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- device-timed steps, inputs resident in HBM, L2 flushed between steps
    clocks = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                          if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit()
                          else local, device_uuid(local))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    launches0 = m.launch_count()
    clocks.start()
    barrier()
    t_host0 = time.monotonic()
    for e0, e1 in ev:
        e0.record(stream)
        step()
        e1.record(stream)
        flush.zero_()
    barrier()
    clocks.window(t_host0, time.monotonic())
    clk = clocks.stop()
    launches = m.launch_count() - launches0
    m.poll()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), world, dist, dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = U * wl.L0 * world
    value = tokens_per_step / (ms_per_step / 1e3)

    # ---- end to end through the public API: pinned host inputs -> device -> host outputs.
    # ot_full_forward_host copies each call's inputs on the model's copy stream into
    # one of two staging slots, so back-to-back calls overlap the next input copy
    # with this call's work, as a serving loop would; the number is the span of
    # all K calls (L2 flushes between calls included) divided by K.
    S_h = S_cpu.pin_memory()
    x_h = x_cpu.pin_memory()
    s_tail_h = torch.empty(s_tail.shape, dtype=s_tail.dtype).pin_memory()
    out_ns_h = torch.empty(out_ns.shape, dtype=out_ns.dtype).pin_memory()
    ws_host = torch.empty(m.host_workspace_bytes(U, C), dtype=torch.uint8, device=dev)

    def step_e2e():
        m.full_forward_host(S_h, x_h, s_tail_h, out_ns_h, kv=kv, ws=ws_host)

    for _ in range(3):
        step_e2e()
        flush.zero_()
    barrier()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(args.steps):
        step_e2e()
        flush.zero_()
    e_end.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / args.steps, world, dist, dev)
    del ws_host
    h2d = S_h.numel() * S_h.element_size() + x_h.numel() * x_h.element_size()
    d2h = s_tail_h.numel() * s_tail_h.element_size() + out_ns_h.numel() * out_ns_h.element_size()

    # ---- per-kernel times: the same steps again with per-launch events on the
    # launching streams; profiling runs every kernel alone (no S/NS overlap),
    # so each event pair brackets exactly one kernel
    prof_steps = min(args.steps, 20)
    m.profile(True)
    barrier()
    for _ in range(prof_steps):
        step()
        flush.zero_()
    barrier()
    recs = m.profile_read()
    m.profile(False)

    peaks = load_peaks()
    serving = []
    if not args.no_serving:
        del ws, kv
        torch.cuda.empty_cache()
        sweep = [1, 2, 4, 8, 16, 64, 512] if args.c_sweep else None
        for name, cands, sw in (("onetrans_s_serve", None, sweep), ("onetrans_l_full", 8, sweep),
                                ("long_fp8", None, None)):
            # 10 warm-up calls, median of 50 per call
            serving.append(run_serving(name, 50, flush, world, dist, dev, peaks, cands, sw,
                                       append_rows=64 if name == "onetrans_s_serve" else 0))
            torch.cuda.empty_cache()
        serving.append(run_full_point("onetrans_l_full", 50, flush, world, dist, dev, peaks))
        torch.cuda.empty_cache()
        serving.append(run_moe_point("onetrans_s_full", 8, 2, 20, flush, world, dist, dev, peaks))
        serving.append(run_backward_point("onetrans_s_full", 16, 5, flush, world, dist, dev, peaks))
        torch.cuda.empty_cache()

    # ---- roofline of the dominant kernel (from the live per-launch events)
    by_kind, by_role = {}, {}
    for r in recs:
        for key, tab in ((r["kind"], by_kind), (r["role"], by_role)):
            t = tab.setdefault(key, {"ms": 0.0, "flops": 0.0, "bytes": 0.0, "launches": 0})
            t["ms"] += r["ms"]
            t["flops"] += r["flops"]
            t["bytes"] += r["bytes"]
            t["launches"] += 1
    dom = max(by_kind, key=lambda k: by_kind[k]["ms"])
    dk = by_kind[dom]
    tf = dk["flops"] / (dk["ms"] / 1e3) / 1e12
    # each launch is timed alone by its own event pair: the burst peak applies
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    traffic, traffic_note = captured_traffic(dom)
    roofline = {"kernel": dom, "bound": "tensor", "achieved": tf, "peak": peak_tf,
                "unit": "TFLOP/s", "frac": tf / peak_tf,
                "traffic": None if traffic is None else traffic * prof_steps / dk["launches"],
                "traffic_unit": "bytes per launch (mean over the step's launches)",
                "traffic_source": traffic_note,
                "algorithmic_bytes_per_launch": dk["bytes"] / dk["launches"],
                "peak_source": f"{peaks['_source']} bf16 dense burst",
                "launches_per_step": dk["launches"] / prof_steps,
                "algorithmic_tflop_per_step": dk["flops"] / prof_steps / 1e12}
    # The S attention at head_dim 64 needs one exponential per visible (query,
    # key) pair against 4 * 64 FLOPs: on B200 the special-function unit (16
    # exp2 per clock per SM) is slower than the tensor core at that ratio, so
    # its exponential rate is the kernel's binding roofline.
    sa = by_role.get("S_attn")
    if sa and sa["ms"] > 0:
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        mhz = clk.get("sm_max_mhz") or 1965.0
        exp_peak = 16 * sms * mhz * 1e6
        exps = sa["flops"] / (4 * 64)
        roofline["s_attention_exp"] = {
            "bound": "sfu", "achieved": exps / (sa["ms"] / 1e3), "peak": exp_peak, "unit": "exp2/s",
            "frac": exps / (sa["ms"] / 1e3) / exp_peak,
            "peak_source": f"16 exp2 per clock per SM x {sms} SMs x {mhz:.0f} MHz",
            "exps_per_step": exps / prof_steps,
            "tensor_floor_ms": sa["flops"] / prof_steps / (peak_tf * 1e12) * 1e3,
            "exp_floor_ms": exps / prof_steps / exp_peak * 1e3}
    step_flops = sum(v["flops"] for v in by_kind.values()) / prof_steps
    kernels = {k: {"ms_per_step": v["ms"] / prof_steps,
                   "share": v["ms"] / max(sum(x["ms"] for x in by_kind.values()), 1e-9),
                   "tflops": v["flops"] / max(v["ms"], 1e-9) / 1e9,
                   "gbs": v["bytes"] / max(v["ms"], 1e-9) / 1e6}
               for k, v in by_kind.items()}
    roles = {k: {"ms_per_step": v["ms"] / prof_steps,
                 "tflops": v["flops"] / max(v["ms"], 1e-9) / 1e9}
             for k, v in by_role.items()}

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            dt, toks, cores = oracle_sample(wl, users=args.cpu_users)
            cpu = {"value": toks / dt, "unit": "S-tokens/s", "cores": cores, "kind": "oracle",
                   "sample": f"{args.cpu_users} users of {wl.name} (full length, {wl.cands} "
                             f"candidate each), "
                             f"Auto-Split + encode + score, C fp64 oracle, OpenMP"}
        line = {
            "metric": metric_name(wl), "value": value, "unit": "S-tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "users_per_gpu": U, "cands": C, "L0": wl.L0,
                       "pyramid": q, "layers": wl.layers, "d": wl.d, "heads": wl.heads,
                       "ffn": wl.ffn, "n_ns": wl.n_ns, "parallelism": f"replicas{world}",
                       "l2": "flushed between steps (256 MB write)"},
            "step_tflops": step_flops / (ms_per_step / 1e3) / 1e12,
            "roofline": roofline,
            "kernels": kernels, "roles": roles,
            "cpu_baseline": cpu,
            "e2e": {"value": tokens_per_step / (e2e_ms / 1e3), "unit": "S-tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clk,
            "serving": serving,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="onetrans_s_full")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-users", type=int, default=8)
    ap.add_argument("--no-serving", action="store_true")
    ap.add_argument("--users", type=int, default=0,
                    help="users per GPU instead of the workload's (a small case for profiling)")
    ap.add_argument("--c-sweep", action="store_true",
                    help="also score the serving caches at C = 1, 2, 4, 8, 16, 64, 512")
    ap.add_argument("--training", action="store_true",
                    help="time only the fp32 training step (ot_full_backward) at the workload's "
                         "shapes, --users users (default 16), and print its JSON object")
    args = ap.parse_args()
    args.steps_ref = max(1, args.steps)
    args.warmup_ref = args.warmup
    from synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.users > 0:
        wl = wl.with_(users=args.users)
    if args.training:
        import torch
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        res = run_backward_point(args.workload, args.users or 16, args.steps, flush, 1, None, dev,
                                 load_peaks())
        print(json.dumps(res))
    elif args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
