"""Benchmark of the AnchorKV codec on B200.

One step = the whole hot path over one synthetic cache: compress every layer
(observation score, anchors, assignment, coefficients, utilities, top-R
residual selection, 2-bit codec) and then one decode-attention step over every
compressed layer at batch 1.  The default workload is the Llama-3.1-8B-shaped
cache (32 layers, 8 KV / 32 query heads, D = 128, N = 32768 tokens, bf16,
theta = 0.05).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl anchorkv|reference]
        python bench.py --sweep      (theta/length sweep of one 8B-shaped layer:
                                      counts, speed, Theorem-1 bound vs measured
                                      output error, ranking and codec ablations)
Under torchrun (N > 1) every rank compresses its own independent cache (weak
scaling, no collective on the data path); the timed region is bracketed by a
barrier and device synchronisation and its duration is the max over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compress Mtok/s per layer-head; compressed decode attn µs/step and HBM GB/s"
UNIT = "Mtok/s per layer-head"
WORKLOAD = "llama8b-n32k-bf16"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d.get("bf16_tflops_sustained"),
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, sm_max_mhz=1965.0, source="fallback")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons of the benchmark's GPU, sampled every
    10 ms from a thread through NVML while the timed region runs (read-only;
    nvidia-smi at 200 ms when NVML is unavailable)."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.thread = None
        self.rows = []

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(self.dev)
        bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
        except Exception:
            nv = None
        if nv is not None:
            self.stop_flag = threading.Event()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        clk = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.rows.append((float(clk), float(mx), [n for n, c in self.REASONS
                                                                   if rs & getattr(nv, c, 0)]))
                    except Exception:
                        pass
                    self.stop_flag.wait(0.01)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict | None:
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            rows = self.rows
        elif self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = [n for n, _ in self.REASONS[:4]]
            rows = [(float(r[1]), float(r[2]), [n for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"])
                    for r in (x.split(",") for x in out.strip().splitlines()) if len(r) >= 9]
        else:
            return None
        if not rows:
            return None
        mx = max(r[1] for r in rows)
        sm = [r[0] for r in rows]
        loaded = [v for v in sm if v > 0.5 * mx] or sm
        reasons = sorted({n for r in rows for n in r[2]})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


# ---------------------------------------------------------------- algorithmic units per stage

def stage_units(spec, theta, L):
    """Algorithmic work of one launch of each timed stage (one layer):
    {stage: (kind, amount, bound)}.  kind 'flops' (tensor contractions, counted
    once even where the kernel splits an operand into bf16 hi/lo parts or
    recomputes Q K^T) or 'bytes' (the bytes the stage must move at least)."""
    H, N, D, G, W = spec.n_kv_heads, spec.n_tokens, spec.head_dim, spec.n_q_heads // spec.n_kv_heads, spec.window
    e = 2 if spec.dtype == "bf16" else 4
    k = L["n_anchors"]
    R = L["n_residuals"]
    GW = G * W
    kv = 2 * H * N * D * e
    n_t = (N + 127) // 128
    return {
        "obs_pass1": ("flops", 2 * H * GW * N * D, "tensor"),          # S = Q K^T
        "obs_alpha": ("flops", 2 * H * GW * N * D, "tensor"),          # ybar = alpha V
        "obs_key_term": ("flops", 2 * H * GW * N * D, "tensor"),       # V ybar^T
        "assign": ("flops", 2 * 2 * H * N * k * D, "tensor"),          # X A^T, both sides
        "project": ("bytes", kv + 4 * 2 * H * N * 3, "hbm"),           # K, V; records, utilities
        "select_topR": ("bytes", 4 * 2 * H * N + 16 * 2 * H * n_t, "hbm"),   # utilities, bitmap
        "quantize": ("bytes", R * (2 * D * e + 34), "hbm"),            # residual rows, records
        "decode_attn": ("bytes", L["total_bytes"], "hbm"),            # one compressed layer
    }


def recorded_traffic(stage):
    """DRAM bytes per launch of `stage` from profiles/traffic.txt, or None when
    there is no capture or the kernel source changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) < 5 or line.startswith("#") or parts[0] != stage:
                continue
            src = os.path.join(ROOT, parts[3])
            if not os.path.exists(src):
                return None
            with open(src, "rb") as g:
                if hashlib.sha256(g.read()).hexdigest() != parts[4]:
                    return None
            return int(parts[2])
    return None


def stage_roofline(stage, units, ms_per_launch, peaks):
    kind, amount, bound = units[stage]
    s = ms_per_launch / 1e3
    if kind == "flops":
        # per-launch event times run at full clock: the burst bf16 peak
        achieved, peak, unit = amount / s / 1e12, peaks["bf16"], "TFLOP/s"
    else:
        achieved, peak, unit = amount / s / 1e9, peaks["hbm"], "GB/s"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak}


# ---------------------------------------------------------------- ranks (host logic, also used by the gloo tests)

def rank_spec(spec, rank: int, layers: int = 0, shard: str = "replicas"):
    """The cache rank `rank` works on: with replicas, an independent cache per
    rank (its own seed); with layer sharding, the one model's cache, the same
    on every rank.  Optionally fewer layers."""
    out = type(spec)(**{**spec.__dict__, "seed": spec.seed + (rank if shard == "replicas" else 0)})
    if layers:
        out = type(spec)(**{**out.__dict__, "n_layers": min(layers, out.n_layers)})
    return out


def rank_layers(n_layers: int, rank: int, world: int, shard: str = "replicas") -> list:
    """Layer indices rank `rank` compresses and decodes: every layer of its own
    cache (replicas), or layers l = rank (mod world) of the shared model
    (layer sharding: each layer's budget is its own, so no layer needs
    another rank's data and no collective runs on the data path)."""
    if shard == "replicas" or world <= 1:
        return list(range(n_layers))
    return [l for l in range(n_layers) if l % world == rank]


def reduce_max(x: float, world: int, device) -> float:
    """Maximum of x over the ranks of the default process group (x itself
    when running alone)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def graph_us_over_ranks(local_ms, steps: int, world: int, device):
    """Microseconds per step of a replayed graph, the max over ranks, or None
    when any rank has no time (its capture failed: local_ms is None).  One
    collective on every rank either way."""
    ms = reduce_max(local_ms if local_ms is not None else 1e30, world, device)
    return 1e3 * ms / steps if ms < 1e29 else None


def job_value(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput in Mtok/s: every rank's layer-head tokens over the
    slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3) / 1e6


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="anchorkv", choices=["anchorkv", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the 70B-shaped compress + 128-step decode and the batch-16 decode blocks")
    ap.add_argument("--layers", type=int, default=0, help="compress only the first L layers (profiling runs)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "layers"],
                    help="under torchrun: every rank its own cache (replicas, weak scaling) or the layers "
                         "of one model split over the ranks (layers, strong scaling)")
    ap.add_argument("--compress-streams", type=int, default=4,
                    help="compress layers round-robin on this many streams (independent layers overlap)")
    ap.add_argument("--sweep", action="store_true",
                    help="theta/length sweep with output error vs the Theorem-1 bound and the ablations "
                         "(one JSON line per point; not the benchmark line)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="batched decode of one 8B-shaped layer (theta = 0.1) for B sequences: "
                         "µs per layer and HBM GB/s over the compressed bytes (one JSON line; not the benchmark line)")
    ap.add_argument("--sweep-point", default="",
                    help="with --sweep: only the theta-length point N,THETA (e.g. 32768,0.05; profiling runs)")
    args = ap.parse_args()
    if args.sweep:
        return run_sweep(args)
    if args.decode_batch > 0:
        return run_batched_decode(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args)
    return run_gpu(args, world, rank, local)


# ---------------------------------------------------------------- sweep and ablations

def _output_error(p, comp, K, V, n_queries, seed):
    """Output error of the compressed cache on n_queries N(0, I) queries per
    KV head and the two Theorem-1 bounds (review, "What carries the argument",
    Eq. 17: ||y^ - y|| <= sum_t alpha_t ||V^_t - V_t|| + 2 V_max tanh(mu),
    mu = ||q|| max_t ||K_t - K^_t|| / sqrt(D); both pairings of weights and
    V_max are provable and both are checked).  y^ comes from the library's
    decode kernel on the compressed bytes; the exact attention and the bound
    terms are evaluated in fp64 with torch (evaluation only)."""
    import torch
    from kv_cache_compression_anchorkv_b200 import api
    from kv_cache_compression_anchorkv_b200.synthetic import gaussian_queries
    H, Hq, D = p.n_kv_heads, p.n_q_heads, p.head_dim
    G = Hq // H
    dev = K.device
    Kh, Vh = api.reconstruct(p, comp)
    qs = gaussian_queries(H * n_queries, D, seed, device=dev).reshape(H, n_queries, D)
    # the decode kernel takes Hq queries per call: G per KV head
    yhat = torch.empty(H, n_queries, D, dtype=torch.float64, device=dev)
    for c in range(0, n_queries, G):
        q = qs[:, c:c + G].reshape(1, Hq, D).to(p.torch_dtype)
        o = api.decode_attn(p, comp, q)
        yhat[:, c:c + G] = o.reshape(H, G, D).double()
    qd = qs.to(p.torch_dtype).double()          # the queries the kernel saw
    err, rel, ba, bb, dks = [], [], [], [], []
    for h in range(H):
        k, v = K[h].double(), V[h].double()
        kh, vh = Kh[h].double(), Vh[h].double()
        dK = (k - kh).norm(dim=1).max()
        dV = (v - vh).norm(dim=1)
        vmax, vhmax = v.norm(dim=1).max(), vh.norm(dim=1).max()
        a = torch.softmax(qd[h] @ k.T / D ** 0.5, dim=1)
        ah = torch.softmax(qd[h] @ kh.T / D ** 0.5, dim=1)
        y = a @ v
        mu = qd[h].norm(dim=1) * dK / D ** 0.5
        e = (yhat[h] - y).norm(dim=1)
        err.append(e)
        rel.append(e / y.norm(dim=1))
        ba.append(ah @ dV + 2 * vmax * torch.tanh(mu))
        bb.append(a @ dV + 2 * vhmax * torch.tanh(mu))
        dks.append(float(dK))
    err, rel, ba, bb = (torch.cat(x) for x in (err, rel, ba, bb))
    bound = torch.minimum(ba, bb)
    return {"queries": int(err.numel()), "err_mean": float(err.mean()), "err_max": float(err.max()),
            "rel_err_mean": float(rel.mean()), "bound_a_mean": float(ba.mean()), "bound_b_mean": float(bb.mean()),
            "bound_holds": float(((err <= ba) & (err <= bb)).double().mean()),
            "err_over_bound_max": float((err / bound).max()), "max_key_error": max(dks)}


def _time_ms(fn, reps, warm=2):
    import torch
    for _ in range(warm):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def run_sweep(args):
    """Theta/length sweep of one 8B-shaped layer (8 KV / 32 query heads,
    D = 128, bf16, window 32; N in {8K, 32K, 128K} x theta in {0.05, 0.1,
    0.2}): anchor and residual counts, compress Mtok/s per layer-head, decode
    at batch 1 (µs, GB/s over the compressed bytes; also the decode with
    rotary positions, keys taken as stored before RoPE), and the Theorem-1 bound
    vs the measured output error on 256 N(0, I) queries per KV head.  Then,
    at N = 32768 and theta = 0.05, the same error for every residual ranking
    criterion and for the unrotated codec (the ablation of the review's
    Figure 5).  Synthetic data as in the benchmark; one JSON line per point."""
    import torch
    from kv_cache_compression_anchorkv_b200 import api
    from kv_cache_compression_anchorkv_b200.synthetic import CacheSpec, make_decode_queries, make_layer
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    n_queries = 256

    def point(N, theta, mode, tag):
        spec = CacheSpec(1, 8, 32, N, n_dirs=128, seed=0)
        K, V, Q = make_layer(spec, 0, device=dev)
        p = api.AnchorKVParams(n_tokens=N, n_kv_heads=8, n_q_heads=32, theta=theta, mode=mode)
        L = api.anchorkv_bytes(p)
        out, ws = api.compress(p, K, V, Q)
        ms = _time_ms(lambda: api.compress(p, K, V, Q, out=out, workspace=ws), reps=5)
        q = make_decode_queries(spec, 0, step=0, batch=1, device=dev)
        dec_ms = _time_ms(lambda: api.decode_attn(p, out, q), reps=20)
        rope_ms = _time_ms(lambda: api.decode_attn_rope(p, out, q, 500000.0), reps=10)
        st = api.read_status(ws)
        line = {"sweep": tag, "n_tokens": N, "theta": theta, "mode": mode, "anchors": L["n_anchors"],
                "residuals": L["n_residuals"], "residual_share": L["n_residuals"] / (2 * 8 * N),
                "compressed_bytes": L["total_bytes"], "ratio": L["uncompressed_bytes"] / L["total_bytes"],
                "compress_mtok_s_per_layer_head": 8 * N / (ms * 1e-3) / 1e6, "compress_ms": ms,
                "decode_us": dec_ms * 1e3, "decode_gbs": L["total_bytes"] / (dec_ms * 1e-3) / 1e9,
                "decode_rope_us": rope_ms * 1e3,
                "refined_rows": st[1]}
        line.update(_output_error(p, out, K, V, n_queries, seed=1000 + N))
        print(json.dumps(line), flush=True)

    if args.sweep_point:
        N, theta = args.sweep_point.split(",")
        point(int(N), float(theta), 0, "theta-length")
        return 0
    for N in (8192, 32768, 131072):
        for theta in (0.05, 0.1, 0.2):
            point(N, theta, 0, "theta-length")
    for name, mode in [("utility", 0), ("residual-norm", api.mode_bits(rank=api.RANK_RESIDUAL_NORM)),
                       ("attention", api.mode_bits(rank=api.RANK_ATTENTION)),
                       ("cosine", api.mode_bits(rank=api.RANK_COSINE)),
                       ("random", api.mode_bits(rank=api.RANK_RANDOM)),
                       ("naive-2bit", api.mode_bits(naive_codec=True)),
                       ("key-queries", api.mode_bits(key_queries=True))]:
        point(32768, 0.05, mode, "ablation:" + name)
    return 0


def run_batched_decode(args):
    """Batched decode of one layer: `--decode-batch` sequences of the 8B shape
    (8 KV / 32 query heads, N = 32768, bf16, theta = 0.1), each compressed on
    its own, decoded in one launch.  Plain decode and decode with rotary
    positions (keys taken as stored before RoPE); µs per layer, and GB/s over
    the compressed bytes the launch reads, against the measured HBM copy peak.
    The batch's layouts (13.4 MB per sequence) exceed L2 from batch 10 on."""
    import torch
    from kv_cache_compression_anchorkv_b200 import api
    from kv_cache_compression_anchorkv_b200.synthetic import CacheSpec, make_decode_queries, make_layer
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    batch, theta = args.decode_batch, 0.1
    spec = CacheSpec(32, 8, 32, 32768, n_dirs=128, seed=0)
    p = api.AnchorKVParams(n_tokens=spec.n_tokens, n_kv_heads=spec.n_kv_heads, n_q_heads=spec.n_q_heads,
                           theta=theta)
    L = api.anchorkv_bytes(p)
    stride = (L["total_bytes"] + 255) // 256 * 256
    comp = torch.zeros(batch, stride, dtype=torch.uint8, device=dev)
    ws, status = None, 0
    for b in range(batch):
        sb = CacheSpec(**{**spec.__dict__, "seed": 1000 + b})
        K, V, Q = make_layer(sb, 0, device=dev)
        out, ws = api.compress(p, K, V, Q, workspace=ws)
        status = status or api.read_status(ws)[0]
        comp[b, :L["total_bytes"]] = out
        del K, V, Q, out
    q = make_decode_queries(spec, 0, step=0, batch=batch, device=dev)
    o = torch.empty(batch, spec.n_q_heads, spec.head_dim, dtype=torch.float32, device=dev)
    dws = torch.empty(api.decode_workspace_bytes(p, batch), dtype=torch.uint8, device=dev)
    rws = torch.empty(api.decode_rope_workspace_bytes(p, batch), dtype=torch.uint8, device=dev)
    reps = max(1, args.steps) * 10
    # layouts below the L2 size would be re-read from L2 between repetitions:
    # flush it with a write larger than L2 before every repetition then, and
    # time the flush alone to take it out
    nbytes = batch * L["total_bytes"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if nbytes < (160 << 20) else None

    def timed(fn):
        if flush is None:
            return _time_ms(fn, reps=reps, warm=max(3, args.warmup))
        both = _time_ms(lambda: (flush.zero_(), fn()), reps=reps, warm=max(3, args.warmup))
        return both - _time_ms(lambda: flush.zero_(), reps=reps, warm=2)

    ms = timed(lambda: api.decode_attn(p, comp, q, out=o, workspace=dws))
    finite = bool(torch.isfinite(o).all())
    # the same decode with the key-residual logits forced onto each path: the
    # tensor-core pre-pass (the default from two slices per head down) and
    # inside the decode
    alt = {}
    for flag, name in (("1", "prepass_key_logits"), ("0", "in_kernel_key_logits")):
        os.environ["ANCHORKV_DECODE_KLOGIT"] = flag
        kws = torch.empty(api.decode_workspace_bytes(p, batch), dtype=torch.uint8, device=dev)
        ok_ = torch.empty_like(o)
        k_ms = timed(lambda: api.decode_attn(p, comp, q, out=ok_, workspace=kws))
        del os.environ["ANCHORKV_DECODE_KLOGIT"]
        alt[f"decode_{name}_us_per_layer"] = k_ms * 1e3
        alt[f"decode_{name}_gbs"] = nbytes / (k_ms * 1e-3) / 1e9
        alt[f"decode_{name}_max_abs_diff"] = float((ok_ - o).abs().max())
    rope_ms = timed(lambda: api.decode_attn_rope(p, comp, q, 500000.0, out=o, workspace=rws))
    finite = finite and bool(torch.isfinite(o).all())
    peaks = _peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {"decode_batch": batch, "n_tokens": spec.n_tokens, "kv_heads": spec.n_kv_heads,
            "q_heads": spec.n_q_heads, "theta": theta, "compressed_bytes_per_sequence": L["total_bytes"],
            "uncompressed_bytes_per_layer": batch * L["uncompressed_bytes"], "reps": reps,
            "decode_us_per_layer": ms * 1e3, "decode_launch": api.decode_config(p, batch),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm"], "traffic": None, "algorithmic_bytes": nbytes,
                         "peak_source": peaks["source"] + " (copy)"},
            **alt,
            "decode_rope_us_per_layer": rope_ms * 1e3,
            "decode_rope_gbs": nbytes / (rope_ms * 1e-3) / 1e9,
            "l2": "layouts larger than L2" if flush is None else "L2 flushed before every repetition",
            "output_finite": finite, "device_status": status, "data": "synthetic"}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- other configurations (one GPU)

def _event_ms(fn, stream, reps):
    """Milliseconds per call of fn() (all calls on `stream`, CUDA events)."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def run_config2(args, dev):
    """Llama-3-70B-shaped cache: 80 layers, 8 KV / 64 query heads, D = 128,
    N = 131072, bf16, theta = 0.05 (43 GB of K/V resident in HBM).  The full
    compress pass (layers on four streams, as in the main step), then a
    128-step decode at batch 1 in which step i sees i + 1 exact tokens
    appended after the compressed prefix; per layer launch, and as one CUDA
    graph holding all 128 steps x 80 layers."""
    import torch
    from kv_cache_compression_anchorkv_b200 import api
    from kv_cache_compression_anchorkv_b200.synthetic import WORKLOADS, make_decode_queries, make_layer, make_tail
    wl = WORKLOADS["llama70b-n128k-bf16"]
    spec, theta = wl["spec"], wl["theta"]
    Lr, H, N, n_steps = spec.n_layers, spec.n_kv_heads, spec.n_tokens, 128
    stream = torch.cuda.current_stream(dev)
    Ks, Vs, Qs, qs, tails = [], [], [], [], []
    for l in range(Lr):
        K, V, Q = make_layer(spec, l, device=dev)
        Ks.append(K); Vs.append(V); Qs.append(Q)
        qs.append(make_decode_queries(spec, l, step=0, batch=n_steps, device=dev))   # row i: step i's query
        tails.append(make_tail(spec, l, n_steps, batch=1, device=dev))
    params = [api.AnchorKVParams(n_tokens=N, n_kv_heads=H, n_q_heads=spec.n_q_heads, theta=theta, layer=l)
              for l in range(Lr)]
    L = api.anchorkv_bytes(params[0])
    outs = [torch.empty(L["total_bytes"], dtype=torch.uint8, device=dev) for _ in range(Lr)]
    n_cs = 4
    cstreams = [torch.cuda.Stream(dev) for _ in range(n_cs)]
    wss = [torch.empty(api.compress_workspace(params[0])["total_bytes"], dtype=torch.uint8, device=dev)
           for _ in range(n_cs)]

    def compress_all():
        fork = torch.cuda.Event()
        fork.record(stream)
        for cs in cstreams:
            cs.wait_event(fork)
        for l in range(Lr):
            with torch.cuda.stream(cstreams[l % n_cs]):
                api.compress(params[l], Ks[l], Vs[l], Qs[l], out=outs[l], workspace=wss[l % n_cs])
        for cs in cstreams:
            j = torch.cuda.Event()
            j.record(cs)
            stream.wait_event(j)

    compress_all()
    status = max((api.read_status(w)[0] for w in wss), key=abs)
    reps = max(1, min(args.steps, 3))
    c_ms = _event_ms(compress_all, stream, reps)
    del Ks, Vs, Qs, wss
    torch.cuda.empty_cache()

    dws = torch.empty(api.decode_workspace_bytes(params[0], 1), dtype=torch.uint8, device=dev)
    dout = torch.empty(1, spec.n_q_heads, spec.head_dim, dtype=torch.float32, device=dev)

    def decode_all():
        for i in range(n_steps):
            for l in range(Lr):
                api.decode_attn(params[l], outs[l], qs[l][i:i + 1], tails[l][0], tails[l][1], tail_len=i + 1,
                                out=dout, workspace=dws)

    decode_all()
    d_ms = _event_ms(decode_all, stream, 1)
    ok = bool(torch.isfinite(dout).all())
    graph_us, note = None, None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            decode_all()
        g.replay()
        torch.cuda.synchronize()
        graph_us = 1e3 * _event_ms(g.replay, stream, max(1, min(args.steps, 3))) / n_steps
        del g
    except Exception as e:
        note = f"{type(e).__name__}: {e}"[:200]
    peaks = _peaks()
    step_bytes = Lr * L["total_bytes"]
    dec_us = 1e3 * d_ms / n_steps
    return {"workload": "llama70b-n128k-bf16", "layers": Lr, "kv_heads": H, "q_heads": spec.n_q_heads,
            "n_tokens": N, "theta": theta, "anchors": L["n_anchors"], "residuals_per_layer": L["n_residuals"],
            "compressed_bytes_per_layer": L["total_bytes"],
            "compress_ms": c_ms, "compress_mtok_s_per_layer_head": Lr * H * N / (c_ms / 1e3) / 1e6,
            "decode_steps": n_steps, "decode_tail": "step i decodes N compressed + (i + 1) exact tokens",
            "decode_us_per_step": dec_us, "decode_us_per_layer": dec_us / Lr,
            "decode_graph_us_per_step": graph_us,
            **({"decode_graph_unavailable": note} if note else {}),
            "decode_hbm_gbs": step_bytes / (dec_us / 1e6) / 1e9,
            "decode_hbm_frac": step_bytes / (dec_us / 1e6) / 1e9 / peaks["hbm"],
            "output_finite": ok, "device_status": status,
            "l2": "inputs larger than L2 (43 GB of K/V; 2.1 GB of layouts per decode step)"}


def run_config3(args, dev):
    """Batched decode: 16 sequences of the 8B shape (32 layers, 8 KV / 32 query
    heads, N = 32768, bf16), each compressed on its own at theta = 0.1; one
    decode step = 32 layer launches of batch 16.  Microseconds per step and
    GB/s over the compressed bytes the step reads, next to the bytes an
    uncompressed cache would read."""
    import torch
    from kv_cache_compression_anchorkv_b200 import api
    from kv_cache_compression_anchorkv_b200.synthetic import WORKLOADS, make_decode_queries, make_layer
    wl = WORKLOADS["llama8b-n32k-bf16-batch16"]
    spec, theta, batch = wl["spec"], wl["theta"], wl["batch"]
    Lr, H, N = spec.n_layers, spec.n_kv_heads, spec.n_tokens
    stream = torch.cuda.current_stream(dev)
    params = [api.AnchorKVParams(n_tokens=N, n_kv_heads=H, n_q_heads=spec.n_q_heads, theta=theta, layer=l)
              for l in range(Lr)]
    L = api.anchorkv_bytes(params[0])
    stride = (L["total_bytes"] + 255) // 256 * 256
    comp = torch.zeros(Lr, batch, stride, dtype=torch.uint8, device=dev)
    ws, status = None, 0
    for l in range(Lr):
        for b in range(batch):
            sb = type(spec)(**{**spec.__dict__, "seed": 1000 + b})
            K, V, Q = make_layer(sb, l, device=dev)
            out, ws = api.compress(params[l], K, V, Q, out=comp[l, b, :L["total_bytes"]], workspace=ws)
        status = status or api.read_status(ws)[0]
    del K, V, Q, ws
    torch.cuda.empty_cache()
    q = [make_decode_queries(spec, l, step=0, batch=batch, device=dev) for l in range(Lr)]
    dws = torch.empty(api.decode_workspace_bytes(params[0], batch), dtype=torch.uint8, device=dev)
    o = torch.empty(Lr, batch, spec.n_q_heads, spec.head_dim, dtype=torch.float32, device=dev)

    def step():
        for l in range(Lr):
            api.decode_attn(params[l], comp[l], q[l], out=o[l], workspace=dws)

    for _ in range(max(3, args.warmup)):
        step()
    ok = bool(torch.isfinite(o).all())
    us = 1e3 * _event_ms(step, stream, max(3, args.steps))
    graph_us = None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        g.replay()
        graph_us = 1e3 * _event_ms(g.replay, stream, max(3, args.steps))
        del g
    except Exception:
        pass
    # the same step with the key-residual logits forced onto each path: the
    # tensor-core pre-pass (this shape's default) and inside the decode
    peaks = _peaks()
    step_bytes = Lr * batch * L["total_bytes"]
    alt = {}
    for flag, name in (("1", "prepass_key_logits"), ("0", "in_kernel_key_logits")):
        os.environ["ANCHORKV_DECODE_KLOGIT"] = flag
        kws = torch.empty(api.decode_workspace_bytes(params[0], batch), dtype=torch.uint8, device=dev)
        ko = torch.empty_like(o)

        def kstep():
            for l in range(Lr):
                api.decode_attn(params[l], comp[l], q[l], out=ko[l], workspace=kws)

        kstep()
        k_us = 1e3 * _event_ms(kstep, stream, max(3, args.steps))
        alt[f"decode_{name}_us_per_step"] = k_us
        alt[f"decode_{name}_hbm_frac"] = step_bytes / (k_us / 1e6) / 1e9 / peaks["hbm"]
        alt[f"decode_{name}_max_abs_diff"] = float((ko - o).abs().max())
        del os.environ["ANCHORKV_DECODE_KLOGIT"], kws, ko
    gbs = step_bytes / (us / 1e6) / 1e9
    return {"workload": "llama8b-n32k-bf16-batch16", "layers": Lr, "batch": batch, "theta": theta,
            **alt,
            "compressed_bytes_per_sequence_layer": L["total_bytes"],
            "decode_us_per_step": us, "decode_us_per_layer": us / Lr, "decode_graph_us_per_step": graph_us,
            "decode_hbm_gbs": gbs, "decode_hbm_frac": gbs / peaks["hbm"],
            "decode_launch": api.decode_config(params[0], batch),
            "uncompressed_bytes_per_step": Lr * batch * L["uncompressed_bytes"],
            "output_finite": ok, "device_status": status,
            "l2": "layouts larger than L2 (%.1f GB per step)" % (step_bytes / 1e9)}


# ---------------------------------------------------------------- oracle (CPU) arm

def _oracle_sample(spec, theta, n_heads):
    """Compress one layer of the workload (the first n_heads KV heads with
    their query heads) with the CPU oracle; returns (seconds, layer-head tokens)."""
    from kv_cache_compression_anchorkv_b200.synthetic import CacheSpec, make_layer
    from oracle import anchorkv_oracle as O
    sub = CacheSpec(1, n_heads, n_heads * (spec.n_q_heads // spec.n_kv_heads), spec.n_tokens, spec.head_dim,
                    spec.window, spec.n_dirs, spec.dtype, spec.seed)
    K, V, Q = make_layer(sub, 0)
    K, V, Q = (x.double().numpy() for x in (K, V, Q))
    p = O.Params(n_tokens=spec.n_tokens, n_kv_heads=n_heads, n_q_heads=sub.n_q_heads, theta=theta,
                 dtype=spec.dtype)
    t0 = time.perf_counter()
    O.compress_layer(K, V, Q, p)
    dt = time.perf_counter() - t0
    return dt, spec.n_tokens * n_heads


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(spec, theta, min_seconds=10.0, max_reps=4):
    """The oracle on one full layer (all KV heads) of the workload, repeated
    until about `min_seconds` of CPU work have been timed."""
    total, toks, reps = 0.0, 0, 0
    while reps < max_reps and (reps == 0 or total < min_seconds):
        dt, t = _oracle_sample(spec, theta, spec.n_kv_heads)
        total += dt
        toks += t
        reps += 1
    out = {"value": toks / total / 1e6, "unit": UNIT, "cores": _threads(), "kind": "oracle",
           "sample": f"{reps} x one layer, all {spec.n_kv_heads} KV heads (N={spec.n_tokens}), fp64 numpy, "
                     f"{total:.1f} s"}
    # the same oracle on one thread (its parallelism is numpy's BLAS threads)
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            dt, t = _oracle_sample(spec, theta, 1)
        out["single_thread"] = {"value": t / dt / 1e6, "unit": UNIT, "cores": 1,
                                "sample": f"one layer, 1 of {spec.n_kv_heads} KV heads, {dt:.1f} s"}
    except ImportError:
        pass
    return out


def run_reference(args):
    from kv_cache_compression_anchorkv_b200.synthetic import WORKLOADS
    wl = WORKLOADS[WORKLOAD]
    spec, theta = wl["spec"], wl["theta"]
    for _ in range(max(0, min(args.warmup, 1))):
        _oracle_sample(spec, theta, 1)
    times, toks = [], 0
    for _ in range(args.steps):
        dt, toks = _oracle_sample(spec, theta, 1)
        times.append(dt)
    total = sum(times)
    value = toks * args.steps / total / 1e6
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": "one layer, 1 KV head (4 query heads) per step",
                       "n_tokens": spec.n_tokens, "theta": theta},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _threads(), "kind": "oracle",
                             "sample": "one layer, 1 of 8 KV heads per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm

def run_gpu(args, world, rank, local):
    import torch
    import torch.distributed as dist

    from kv_cache_compression_anchorkv_b200 import api
    from kv_cache_compression_anchorkv_b200.synthetic import WORKLOADS, make_decode_queries, make_layer

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wl = WORKLOADS[WORKLOAD]
    spec, theta = wl["spec"], wl["theta"]
    spec = rank_spec(spec, rank, args.layers, args.shard)
    ids = rank_layers(spec.n_layers, rank, world, args.shard)    # this rank's layers
    Lr, H, N = len(ids), spec.n_kv_heads, spec.n_tokens
    # layer-heads of the whole job per step: every rank's own cache, or the one model
    job_layers = Lr * world if args.shard == "replicas" else spec.n_layers

    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_base = cpu_baseline(spec, theta)

    # inputs resident in HBM: every layer's K, V, Q_obs (4.3 GB at the 8B shape)
    Ks, Vs, Qs, qd = [], [], [], []
    for l in ids:
        K, V, Q = make_layer(spec, l, device=dev)
        Ks.append(K); Vs.append(V); Qs.append(Q)
        qd.append(make_decode_queries(spec, l, step=0, batch=1, device=dev))
    params = [api.AnchorKVParams(n_tokens=N, n_kv_heads=H, n_q_heads=spec.n_q_heads, theta=theta,
                                 window=spec.window, dtype=spec.dtype, seed=spec.seed, layer=l) for l in ids]
    L = api.anchorkv_bytes(params[0])
    outs = [torch.empty(L["total_bytes"], dtype=torch.uint8, device=dev) for _ in range(Lr)]
    ws = torch.empty(api.compress_workspace(params[0])["total_bytes"], dtype=torch.uint8, device=dev)
    dws = torch.empty(api.decode_workspace_bytes(params[0], 1), dtype=torch.uint8, device=dev)
    dout = [torch.empty(1, spec.n_q_heads, spec.head_dim, dtype=torch.float32, device=dev) for _ in range(Lr)]
    stream = torch.cuda.current_stream(dev)
    # layers are independent compression problems: optionally several streams,
    # each with its own workspace; decode stays sequential over layers (a
    # layer's query depends on the previous layer's output)
    n_cs = max(1, args.compress_streams)
    cstreams = [torch.cuda.Stream(dev) for _ in range(n_cs)] if n_cs > 1 else []
    wss = [ws] + [torch.empty_like(ws) for _ in range(n_cs - 1)]

    dstream = torch.cuda.Stream(dev) if n_cs > 1 else None

    def step(single=False):
        if single or not cstreams:
            for l in range(Lr):
                api.compress(params[l], Ks[l], Vs[l], Qs[l], out=outs[l], workspace=ws)
            for l in range(Lr):
                api.decode_attn(params[l], outs[l], qd[l], out=dout[l], workspace=dws)
            return
        # compress layer l on stream l % n_cs; the decode step runs on its own
        # stream, layer after layer, each layer once its compression is done
        fork = torch.cuda.Event()
        fork.record(stream)
        for cs in cstreams + [dstream]:
            cs.wait_event(fork)
        done = []
        for l in range(Lr):
            i = l % n_cs
            with torch.cuda.stream(cstreams[i]):
                api.compress(params[l], Ks[l], Vs[l], Qs[l], out=outs[l], workspace=wss[i])
                ev = torch.cuda.Event()
                ev.record(cstreams[i])
                done.append(ev)
        with torch.cuda.stream(dstream):
            for l in range(Lr):
                dstream.wait_event(done[l])
                api.decode_attn(params[l], outs[l], qd[l], out=dout[l], workspace=dws)
        for cs in cstreams + [dstream]:
            join = torch.cuda.Event()
            join.record(cs)
            stream.wait_event(join)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    status = [api.read_status(w)[0] for w in wss]
    status = [max(status, key=abs)]
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    n0 = api.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    barrier()
    launches = api.launch_count() - n0
    clk = clocks.stop()
    ms = reduce_max(ev0.elapsed_time(ev1), world, dev)
    ms_step = ms / args.steps

    # decode alone and compress alone (same stream, CUDA events) for the metric's parts
    ev2, ev3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    ev2.record(stream)
    for _ in range(args.steps):
        for l in range(Lr):
            api.decode_attn(params[l], outs[l], qd[l], out=dout[l], workspace=dws)
    ev3.record(stream)
    barrier()
    dec_us = 1e3 * reduce_max(ev2.elapsed_time(ev3), world, dev) / args.steps

    # the same decode step captured once as one CUDA graph over the layers
    # (no collective inside the try, so every rank takes the same steps)
    graph, graph_note = None, None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for l in range(Lr):
                api.decode_attn(params[l], outs[l], qd[l], out=dout[l], workspace=dws)
    except Exception as e:  # reported in the line, not fatal to the bench
        graph, graph_note = None, f"{type(e).__name__}: {e}"[:200]
    barrier()
    graph_local = 0.0
    if graph is not None:
        graph.replay()
        torch.cuda.synchronize(dev)
        ev4, ev5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev4.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev5.record(stream)
        torch.cuda.synchronize(dev)
        graph_local = ev4.elapsed_time(ev5)
    barrier()
    dec_graph_us = graph_us_over_ranks(graph_local if graph is not None else None, args.steps, world, dev)
    del graph

    # per-stage event timing over the same steps, for the roofline of the dominant kernel
    api.stage_timing(True)
    barrier()
    for _ in range(args.steps):
        step(single=True)     # one stream: stage events do not overlap
    barrier()
    stages = api.stage_times()
    api.stage_timing(False)

    peaks = _peaks()
    units = stage_units(spec, theta, L)
    per_launch = {st: stages[st][0] / stages[st][1] for st in stages if st in units and stages[st][1]}
    dom = max(per_launch, key=lambda st: stages[st][0])
    roof = stage_roofline(dom, units, per_launch[dom], peaks)
    roof["traffic"] = recorded_traffic(dom)
    roof["kernel"] = dom
    roof["peak_source"] = ("measured" if peaks["source"] == "measured" else "fallback") + (
        " (burst bf16)" if roof["unit"] == "TFLOP/s" else " (copy)")
    stage_roofs = {st: {**{kk: (round(v, 4) if isinstance(v, float) else v)
                           for kk, v in stage_roofline(st, units, per_launch[st], peaks).items()},
                        "traffic": recorded_traffic(st)}
                   for st in per_launch}

    dec_bytes = Lr * L["total_bytes"]
    value = job_value(N * job_layers * H, 1, ms_step)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, spec, theta, params, ids, job_layers, dev, stream, barrier, world)

    # the other single-GPU configurations, on this GPU alone (not under torchrun)
    extra = {}
    if world == 1 and not args.no_configs:
        del Ks, Vs, Qs, outs, wss, ws
        torch.cuda.empty_cache()
        extra["config2"] = run_config2(args, dev)
        torch.cuda.empty_cache()
        extra["config3"] = run_config3(args, dev)
        torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak" if args.shard == "replicas" else "strong",
            "vs_baseline": None, "dtype": spec.dtype, "data": "synthetic",
            "config": {"workload": WORKLOAD, "layers": Lr, "kv_heads": H, "q_heads": spec.n_q_heads,
                       "head_dim": spec.head_dim, "n_tokens": N, "window": spec.window, "theta": theta,
                       "decode_batch": 1, "parallelism": f"{args.shard}{world}", "compress_streams": n_cs,
                       "l2": "inputs larger than L2 (%.1f GB of K/V per step)" % (Lr * 2 * H * N * 128 * 2 / 1e9)},
            "decode_us_per_step": dec_us,
            "decode_graph_us_per_step": dec_graph_us,
            "decode_launch": api.decode_config(params[0], 1),
            "decode_hbm_gbs": dec_bytes / (dec_us / 1e6) / 1e9,
            "decode_graph": ({"note": "one CUDA graph holding the 32 per-layer launches, replayed per step"}
                             if dec_graph_us is not None else {"unavailable": graph_note or "capture failed on a rank"}),
            "compressed_bytes_per_layer": L["total_bytes"],
            "uncompressed_bytes_per_layer": L["uncompressed_bytes"],
            "compression_ratio": L["uncompressed_bytes"] / L["total_bytes"],
            "roofline": roof,
            "stage_ms_per_step": {s: v[0] / args.steps for s, v in stages.items() if v[1]},
            "stage_roofline": stage_roofs,
            "gpu_launches": launches,
            "clocks": clk,
            "device_status": status[0],
            "e2e": e2e,
            **extra,
        }
        if cpu_base is not None:
            line["cpu_baseline"] = cpu_base
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(args, spec, theta, params, ids, job_layers, dev, stream, barrier, world):
    """Same step through the public API with host buffers: per layer, the
    C ABI's anchorkv_compress_host copies the pinned K, V, Q_obs in, compresses
    and copies the layout back (the copies inside the library); then the
    decode step copies each layer's query in and its output back."""
    import torch

    from kv_cache_compression_anchorkv_b200 import api
    from kv_cache_compression_anchorkv_b200.synthetic import make_decode_queries, make_layer
    Lr = len(ids)
    # host copies of the layers (pinned); the step moves all of them
    host = []
    for l in ids:
        K, V, Q = make_layer(spec, l, device=dev)
        host.append(tuple(x.cpu().pin_memory() for x in (K, V, Q)))
    qh = [make_decode_queries(spec, l, 0, 1, device=dev).cpu().pin_memory() for l in ids]
    n_cs = max(1, args.compress_streams)
    comps = [api.HostCompressor(api.AnchorKVParams(**{**params[0].__dict__}), device=dev) for _ in range(n_cs)]
    cstreams = [torch.cuda.Stream(dev) for _ in range(n_cs)]
    dstream = torch.cuda.Stream(dev)
    outs_h = [torch.empty_like(comps[0].host_out).pin_memory() for _ in range(Lr)]
    qdev = torch.empty(1, spec.n_q_heads, spec.head_dim, dtype=params[0].torch_dtype, device=dev)
    odev = torch.empty(1, spec.n_q_heads, spec.head_dim, dtype=torch.float32, device=dev)
    oh = torch.empty(Lr, 1, spec.n_q_heads, spec.head_dim, dtype=torch.float32).pin_memory()
    layouts = [torch.empty_like(comps[0].out) for _ in range(Lr)]
    dws = torch.empty(api.decode_workspace_bytes(params[0], 1), dtype=torch.uint8, device=dev)

    def step():
        # compress: layer l on stream l % n_cs (copies of one layer overlap the
        # compression of another); decode: sequential over layers
        fork = torch.cuda.Event()
        fork.record(stream)
        for cs in cstreams + [dstream]:
            cs.wait_event(fork)
        done = []
        for l in range(Lr):
            i = l % n_cs
            with torch.cuda.stream(cstreams[i]):
                comps[i](*host[l], layer=ids[l], host_out=outs_h[l])
                layouts[l].copy_(comps[i].out)
                ev = torch.cuda.Event()
                ev.record(cstreams[i])
                done.append(ev)
        with torch.cuda.stream(dstream):
            for l in range(Lr):
                dstream.wait_event(done[l])
                qdev.copy_(qh[l], non_blocking=True)
                api.decode_attn(params[l], layouts[l], qdev, out=odev, workspace=dws)
                oh[l].copy_(odev, non_blocking=True)
        for cs in cstreams + [dstream]:
            join = torch.cuda.Event()
            join.record(cs)
            stream.wait_event(join)

    steps = max(1, min(args.steps, 3))
    step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    barrier()
    ms = reduce_max(e0.elapsed_time(e1), world, dev) / steps
    h2d = sum(x.numel() * x.element_size() for t3 in host for x in t3) + sum(q.numel() * q.element_size() for q in qh)
    d2h = sum(o.numel() for o in outs_h) + oh.numel() * 4
    return {"value": job_value(spec.n_tokens * job_layers * spec.n_kv_heads, 1, ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms, "steps": steps}


if __name__ == "__main__":
    sys.exit(main())
