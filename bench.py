#!/usr/bin/env python
"""KronQ per-layer quantization throughput on B200.

One step = the whole per-layer path over one synthetic layer's calibration
batch: H_X = X^T X / N and H_G = G^T G / N (tensor cores), BiIP (rescale +
randomized Hadamard on both sides of W, H_X, H_G), s = tr(H_G) tr(H_X),
damped inverse Cholesky, column-wise OBS quantization, packing.

Prints one JSON line (rank 0).  `value` is whole-job Mweights/s with X, G, W
resident in HBM; `e2e` is the same metric through the public Python API with
pinned host buffers (H2D of X, G, W and D2H of the packed result inside the
timed region).  `--impl reference` times the fp64 CPU oracle on a bounded
sample of the same workload instead.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import pathlib
import statistics
import subprocess
import sys
import threading
import time

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "layer quantize Mweights/s end-to-end; H_X/H_G GEMM % of bf16 tensor peak"
UNIT = "Mweights/s"
DEFAULT_CONFIG = "llama3-70b-mlp"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--act-order", action="store_true",
                    help="quantize columns in descending H_X' diagonal order (README --act_order)")
    ap.add_argument("--w-clip", action="store_true",
                    help="clip-ratio search for every grid (README --w_clip)")
    ap.add_argument("--deploy", action="store_true",
                    help="time the deployment matvec (kronq_deploy_matvec, batch 1) of the "
                         "quantized layer instead of the quantization step")
    ap.add_argument("--tokens", type=int, default=None,
                    help="calibration tokens per X/G (default: the workload's; smaller only for "
                         "profiler captures)")
    ap.add_argument("--kernel", choices=["covariance", "cholesky", "solver", "biip"], default=None,
                    help="time one stage alone (for profiler captures on small cases): "
                         "kronq_covariance of a --tokens x --width bf16 matrix, "
                         "kronq_cholesky_inv of a --width x --width covariance, "
                         "kronq_quantize_layer of a --rows x --width layer, or "
                         "kronq_biip_rotate of that layer with its two covariances")
    ap.add_argument("--rows", type=int, default=4096, help="layer rows for --kernel solver")
    ap.add_argument("--width", type=int, default=None,
                    help="feature width for --kernel (default: the workload's widest)")
    ap.add_argument("--gptaq", action="store_true",
                    help="time the step with GPTAQ's asymmetric calibration: the drift covariance "
                         "of [X~ | X] in place of H_X, the correction P and the solver with it")
    ap.add_argument("--oracle-full-chain", action="store_true",
                    help="time the fp64 oracle's whole chain once on the host cores (every "
                         "token, every row) for the configuration and print one line; no GPU")
    return ap.parse_args()


def workload_desc(cfg) -> str:
    subs = ", ".join(f"{s.name} {s.m}x{s.n}" for s in cfg.sublayers)
    g = "per-channel" if cfg.sublayers[0].group == -1 else f"group-{cfg.sublayers[0].group}"
    bits = "mixed 2/3/4 at 3.0 avg" if cfg.mixed_avg_bits else f"W{cfg.sublayers[0].bits}"
    return (f"{cfg.name}: {subs}; X/G {cfg.tokens} tokens bf16 ({cfg.x_dist} X with outlier "
            f"channels x{cfg.x_outlier_scale:g}, G scales over {cfg.g_decades:g} decades); "
            f"{bits} asymmetric {g}; BiIP alpha {cfg.alpha}, damp {cfg.damp}")


def l2_note(cfg) -> str:
    sizes = [cfg.tokens * s.width * 2 for s in cfg.sites] + [cfg.tokens * s.m * 2 for s in cfg.sublayers]
    small = min(sizes)
    verdict = "larger than" if small > 126 * 2 ** 20 else "NOT larger than"
    return (f"inputs {verdict} L2, no flush: each X/G is {small / 2 ** 30:.2f} GiB or more "
            f"({cfg.tokens} tokens, bf16)")


# ---------------------------------------------------- ranks (N > 1)
def rank_config(cfg0, rank: int):
    """Each rank quantizes its own layer (weak scaling): the seed is offset
    by the rank, so no two ranks draw the same inputs."""
    import dataclasses
    return dataclasses.replace(cfg0, seed=cfg0.seed + rank)


def reduce_max_ms(ms: float, world: int, device) -> float:
    """The job's time: the slowest rank's (a MAX all-reduce; every rank calls it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(weights: int, world: int, steps: int, ms: float) -> float:
    """Whole-job Mweights/s: every rank's layer, all timed steps, over the max time."""
    return weights * world * steps / (ms / 1e3) / 1e6


# ------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while running (clocks and throttle reasons)."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None
        self.cut = None

    def mark_end(self):
        """The samples so far are the timed region's; later ones (the
        end-to-end leg, the CPU baseline) stay out of the summary."""
        self.cut = len(self.lines)

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[:self.cut]:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 8:
                continue
            try:
                sm.append(float(p[0]))
                mx = float(p[1])
            except ValueError:
                continue
            for nm, v in zip(names, p[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for(dev_index: int) -> str | None:
    import torch
    try:
        u = torch.cuda.get_device_properties(dev_index).uuid
        s = str(u)
        return s if s.startswith("GPU-") else f"GPU-{s}"
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[dev_index] if vis else None


# -------------------------------------------------------- peaks / traffic
def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "MEASURED_PEAKS.json"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("covariance.cu", "common.cuh"):
        h.update((ROOT / "post_quantization_02_b200" / "csrc" / f).read_bytes())
    return h.hexdigest()[:16]


def load_traffic(workload: str):
    """DRAM bytes per launch of the covariance kernel from a committed ncu
    summary, only while the kernel source is the one that was profiled."""
    p = ROOT / "profiles" / "cov_pair_kernel.traffic.json"
    if not p.exists():
        return None
    d = json.loads(p.read_text())
    if d.get("source_sha") != kernel_source_sha() or d.get("workload") != workload:
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------- oracle side
# The fixed oracle sample both CPU legs time (the cpu_baseline of the GPU
# run and every step of --impl reference): the same stages on the same
# sample sizes, scaled to the whole layer the same way, so the two agree.
SAMPLE_TOKENS = 2048       # covariance rows, scaled by tokens
SAMPLE_COV_COLS = 4096     # covariance of the leading columns, scaled by (width / cols)^2
SAMPLE_ROT_ROWS = 64       # rows through each rotation, scaled by rows
SAMPLE_CHOL_N = 1024       # inverse Cholesky size, scaled by n^3
SAMPLE_OBS_COLS = 4096     # column-loop width, scaled by cols^2 above it
SAMPLE_OBS_ROWS = 32       # column-loop rows per host thread, scaled by rows


def oracle_sample(cfg):
    """Time the fp64 oracle, as it stands, on a bounded sample of the workload
    and extrapolate to the whole job.  Returns (seconds_full, sample_text)."""
    import numpy as np
    import synth
    from oracle import cholesky as ochol, quantizer as oq, pack as opack
    from oracle import covariance as ocov
    from oracle import transform as otr

    tok = SAMPLE_TOKENS
    rows_rot = SAMPLE_ROT_ROWS
    total = 0.0
    parts = []
    r = np.random.default_rng(0)
    for sub in cfg.sublayers:
        site = cfg.site(sub.site)
        m, n = sub.m, sub.n
        # covariances: tok tokens of the leading cx (cg) columns of X (G),
        # scaled to all tokens and to the whole width by (width / cx)^2 -- the
        # product's cost; the full d x d output of a small sample would be
        # written at memory speed and, scaled by tokens, overstate it
        xb = synth.x_chunk(cfg, site, 0, tokens=tok)
        gb = synth.g_chunk(cfg, sub, 0, tokens=tok)
        cx, cg = min(site.width, SAMPLE_COV_COLS), min(m, SAMPLE_COV_COLS)
        t0 = time.perf_counter()
        ocov.covariance(synth.bf16_bits_to_f32(xb[:, :cx]).astype(np.float64))
        t_x = time.perf_counter() - t0
        t0 = time.perf_counter()
        ocov.covariance(synth.bf16_bits_to_f32(gb[:, :cg]).astype(np.float64))
        t_g = time.perf_counter() - t0
        t_cov = (t_x * (site.width / cx) ** 2 + t_g * (m / cg) ** 2) * cfg.tokens / tok
        # BiIP: the transform on rows_rot rows of each width, scaled to the
        # row and column passes of W (m x n), H_X (n x n), H_G (m x m)
        su, sv = synth.make_signs(cfg, sub)
        t0 = time.perf_counter()
        otr.apply(r.standard_normal((rows_rot, n)), sv)
        t_rn = (time.perf_counter() - t0) / rows_rot
        t0 = time.perf_counter()
        otr.apply(r.standard_normal((rows_rot, m)), su)
        t_rm = (time.perf_counter() - t0) / rows_rot
        t_rot = t_rn * (m + 2 * n) + t_rm * (n + 2 * m)
        # damped inverse Cholesky at SAMPLE_CHOL_N, scaled by n^3
        nc = min(n, SAMPLE_CHOL_N)
        A = r.standard_normal((nc, nc))
        H = A @ A.T / nc + np.eye(nc)
        t0 = time.perf_counter()
        ochol.inverse_cholesky(ochol.damp(H, cfg.damp))
        t_chol = (time.perf_counter() - t0) * (n / nc) ** 3
        # column loop: one 64-row chunk per host thread at up to 4096 columns,
        # scaled by rows and by cols^2 beyond (the loop's cost does not depend
        # on the factor's values: any upper triangular matrix with a positive
        # diagonal serves for timing)
        nn = min(n, SAMPLE_OBS_COLS)
        U = np.triu(r.standard_normal((nn, nn)) * 0.01) + np.eye(nn)
        bits = sub.bits or 3
        grp = sub.group if sub.group == -1 or nn % sub.group == 0 else -1
        rows_obs = min(m, SAMPLE_OBS_ROWS * max(1, min(32, os.cpu_count() or 1)))
        Wr = r.standard_normal((rows_obs, nn)) * 0.02
        t0 = time.perf_counter()
        res = oq.obs_quantize_rows(Wr, U, bits, grp)
        t_obs = (time.perf_counter() - t0) * (m / rows_obs) * (n / nn) ** 2
        t0 = time.perf_counter()
        if bits in (2, 4):
            opack.pack(res["codes"], bits)
        t_pack = (time.perf_counter() - t0) * (m / rows_obs) * (n / nn)
        total += t_cov + t_rot + t_chol + t_obs + t_pack
        parts.append(f"{sub.name}: cov {tok} of {cfg.tokens} tokens x {cx} of {site.width} (X) and "
                     f"{cg} of {m} (G) columns, rotation {rows_rot} rows, "
                     f"inverse Cholesky n={nc}, OBS {rows_obs} of {m} rows x {nn} cols")
    sample = ("fp64 oracle stages timed on a fixed sample and scaled to the whole layer (covariance "
              "x tokens x (width / columns)^2, rotation x rows, inverse Cholesky x n^3, OBS x rows, "
              f"x cols^2 above {SAMPLE_OBS_COLS}): " + "; ".join(parts))
    return total, sample


def host_cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.lower().startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_full_chain(args):
    """The whole fp64 oracle chain of the configuration, timed once on the
    host cores: covariances over every token, BiIP, s, damped inverse
    Cholesky, the unblocked column loop on every row, packing."""
    import synth
    from oracle import pipeline as opipe
    cfg = synth.get_config(args.config)
    t0 = time.perf_counter()
    stages = {}
    for sub in cfg.sublayers:
        t = time.perf_counter()
        hx = opipe.x_covariance(cfg, cfg.site(sub.site))
        hg = opipe.g_covariance(cfg, sub)
        stages["covariance"] = stages.get("covariance", 0.0) + time.perf_counter() - t
        t = time.perf_counter()
        opipe.quantize_sublayer(cfg, sub, hx, hg, sub.bits or 3)
        stages["biip_to_pack"] = stages.get("biip_to_pack", 0.0) + time.perf_counter() - t
    wall = time.perf_counter() - t0
    line = {"impl": "reference", "kind": "oracle full chain", "metric": METRIC,
            "value": cfg.weights / wall / 1e6, "unit": UNIT, "seconds": wall,
            "stages_s": {k: round(v, 2) for k, v in stages.items()},
            "config": {"workload": workload_desc(cfg)}, "cores": blas_threads(),
            "host_cpus": os.cpu_count(), "cpu_model": host_cpu_model(), "dtype": "f64"}
    print(json.dumps(line), flush=True)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, rank, world):
    import synth
    if rank != 0:
        return
    cfg = synth.get_config(args.config)
    weights = cfg.weights
    for _ in range(args.warmup):
        oracle_sample(cfg)
    t0 = time.perf_counter()
    ests = []
    sample = ""
    for _ in range(args.steps):
        est, sample = oracle_sample(cfg)
        ests.append(est)
    wall = time.perf_counter() - t0
    full = statistics.mean(ests)
    value = weights / full / 1e6
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": full * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded generator)",
        "config": {"workload": workload_desc(cfg), "sample_wall_s_per_step": wall / max(1, args.steps)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                         "host_cpus": os.cpu_count(), "cpu_model": host_cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- GPU side
class Layer:
    """Device buffers of one sublayer for the timed steps (allocated once)."""

    def __init__(self, cfg, sub, dev, seed_offset, G, act_order=False):
        import torch
        import synth
        from post_quantization_02_b200 import abi
        self.sub = sub
        m, n = sub.m, sub.n
        self.W0 = torch.from_numpy(synth.make_w(cfg, sub)).to(dev)
        su, sv = synth.make_signs(cfg, sub)
        self.su = torch.from_numpy(su).to(dev)
        self.sv = torch.from_numpy(sv).to(dev)
        self.G = G
        self.W = torch.empty_like(self.W0)
        self.HX = torch.empty((n, n), dtype=torch.float32, device=dev)
        self.HG = torch.empty((m, m), dtype=torch.float32, device=dev)
        self.SX = torch.empty(n, dtype=torch.float32, device=dev)
        self.SG = torch.empty(m, dtype=torch.float32, device=dev)
        self.U = torch.empty((n, n), dtype=torch.float32, device=dev)
        self.sens = torch.zeros(3, dtype=torch.float64, device=dev)
        self.info = torch.zeros(1, dtype=torch.int32, device=dev)
        self.codes = torch.empty((m, n), dtype=torch.uint8, device=dev)
        G = 1 if sub.group == -1 else n // sub.group
        self.scales = torch.empty((m, G), dtype=torch.float32, device=dev)
        self.zeros = torch.empty((m, G), dtype=torch.uint8, device=dev)
        # room for 4-bit words; 2-bit codes use the first m x n/16 words as one
        # contiguous m x (n/16) matrix (packed_view)
        self.packed_store = torch.empty(m * abi.packed_words(n, 4), dtype=torch.int32, device=dev)
        self.bits = sub.bits
        self.perm = self.Hp = self.Wp = self.codes_p = None
        if act_order:
            self.perm = torch.empty(n, dtype=torch.int32, device=dev)
            self.Hp = torch.empty((n, n), dtype=torch.float32, device=dev)
            self.Wp = torch.empty((m, n), dtype=torch.float32, device=dev)
            self.codes_p = torch.empty((m, n), dtype=torch.uint8, device=dev)


def packed_view(L, bits):
    words = abi_packed_words(L.sub.n, bits)
    return L.packed_store[: L.sub.m * words].view(L.sub.m, words)


def abi_packed_words(n, bits):
    from post_quantization_02_b200 import abi
    return abi.packed_words(n, bits)


def host_input_bytes(cfg) -> int:
    """Bytes of one rank's host inputs: X per input site and G per sublayer
    (bf16, every token)."""
    return sum(cfg.tokens * s_.width * 2 for s_ in cfg.sites) + \
        sum(cfg.tokens * s_.m * 2 for s_ in cfg.sublayers)


def needs_lean_inputs(cfg, world: int, e2e: bool, ram: int) -> bool:
    """True when every rank's host inputs (and, with the end-to-end leg, their
    pinned copies) would take more than 60 % of the host's memory."""
    return world * host_input_bytes(cfg) * (2 if e2e else 1) > 0.6 * ram


def draw_to_device(chunk_fn, tokens, width, dev, threads):
    """A token-major bf16 input drawn chunk by chunk (synth's seeded chunks)
    straight into device memory; at most `threads` chunks on the host at once."""
    import numpy as np
    import torch
    import synth
    from concurrent.futures import ThreadPoolExecutor
    A = torch.empty((tokens, width), dtype=torch.bfloat16, device=dev)
    nch = synth.n_chunks(tokens)
    with ThreadPoolExecutor(threads) as ex:
        for c0 in range(0, nch, threads):
            for c, bits in zip(range(c0, nch), ex.map(chunk_fn, range(c0, min(nch, c0 + threads)))):
                r0 = c * synth.CHUNK_TOKENS
                A[r0:r0 + bits.shape[0]].copy_(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
    return A


class StageMarks:
    """CUDA events at stage boundaries of one step; each mark closes the
    stage named by it (the time since the previous mark)."""

    def __init__(self, stream):
        self.stream = stream
        self.events = []

    def mark(self, name):
        import torch
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        self.events.append((name, e))

    def totals(self):
        out = {}
        for (_, e0), (name, e1) in zip(self.events, self.events[1:]):
            out[name] = out.get(name, 0.0) + e0.elapsed_time(e1)
        return out


def solve_layer(cfg, L, ws, stream, act_order=False, clip=False, mark=None):
    """Damped inverse Cholesky and the column loop of one sublayer, with the
    README's --act_order (column order by the H_X' diagonal, results back in
    the original order) and --w_clip (clip-ratio search) when asked for."""
    from post_quantization_02_b200 import abi
    opts = abi.QUANT_CLIP if clip else 0
    mark = mark or (lambda name: None)
    if not act_order:
        abi.kronq_cholesky_inv(L.HX, cfg.damp, L.U, L.info, ws, stream=stream)
        mark("inverse_cholesky")
        abi.kronq_quantize_layer_opt(L.W, L.U, L.bits, L.sub.group, cfg.block, opts, L.codes,
                                     L.scales, L.zeros, None, L.info, ws, stream=stream)
        mark("solver")
        return
    abi.kronq_act_order(L.HX, L.perm, stream=stream)
    abi.kronq_permute(L.HX, L.Hp, L.perm, abi.PERM_SYM, L.info, stream=stream)
    abi.kronq_permute(L.W, L.Wp, L.perm, abi.PERM_COLS, L.info, stream=stream)
    abi.kronq_cholesky_inv(L.Hp, cfg.damp, L.U, L.info, ws, stream=stream)
    mark("inverse_cholesky")
    abi.kronq_quantize_layer_opt(L.Wp, L.U, L.bits, L.sub.group, cfg.block, opts, L.codes_p,
                                 L.scales, L.zeros, None, L.info, ws, stream=stream)
    abi.kronq_permute(L.codes_p, L.codes, L.perm, abi.UNPERM_COLS, L.info, stream=stream)
    mark("solver")


def gpu_step(cfg, layers, X, ws, stream, cov_events=None, act_order=False, clip=False,
             marks=None):
    """One pass of the whole path over every sublayer of the config."""
    import torch
    from post_quantization_02_b200 import abi, alloc
    N = cfg.tokens
    ev = iter(cov_events) if cov_events is not None else None
    mark = marks.mark if marks is not None else (lambda name: None)
    mark("start")

    def cov(A, H):
        if ev is not None:
            next(ev).record(stream)
        abi.kronq_covariance(A, H, 1.0 / N, 0.0, stream=stream)
        if ev is not None:
            next(ev).record(stream)

    hx_site = {}
    for L in layers:
        site = L.sub.site
        if site not in hx_site:
            cov(X[site], layers[[l.sub.site for l in layers].index(site)].HX)
            hx_site[site] = layers[[l.sub.site for l in layers].index(site)].HX
        cov(L.G, L.HG)
    for L in layers:
        if L.HX is not hx_site[L.sub.site]:
            L.HX.copy_(hx_site[L.sub.site])
    for L in layers:
        L.W.copy_(L.W0)
    mark("covariance")
    # H_X of a shared site is rotated per sublayer: rotate copies, the site's own last
    for L in layers:
        abi.kronq_biip_rotate(L.W, L.HX, L.HG, L.su, L.sv, cfg.alpha, cfg.mode, 0, L.SX, L.SG, ws,
                              stream=stream)
        abi.kronq_sensitivity(L.HX, L.HG, L.sens, stream=stream)
    if cfg.mixed_avg_bits:
        scores = torch.stack([L.sens[0] for L in layers]).cpu().tolist()
        bits = alloc.allocate_bits(scores, [L.sub.m * L.sub.n for L in layers], cfg.mixed_avg_bits)
        for L, b in zip(layers, bits):
            L.bits = b
    mark("biip_sensitivity")
    for L in layers:
        solve_layer(cfg, L, ws, stream, act_order, clip, mark)
        if L.bits in (2, 4):
            abi.kronq_pack(L.codes, L.bits, packed_view(L, L.bits), stream=stream)
        mark("pack")


def run_deploy(args):
    """Batch-1 decode through the packed layer: y = W_hat x with the BiIP
    transforms applied to x and y (kronq_deploy_matvec).  The layer is
    quantized once on the GPU; `copies` distinct copies of its packed codes
    (more bytes than L2) are cycled so that every matvec reads its weights
    from HBM; the calls are captured in one CUDA graph (one replay = all
    copies) and timed with CUDA events."""
    import dataclasses
    import numpy as np
    import torch
    import synth
    from post_quantization_02_b200 import abi
    from post_quantization_02_b200 import pipeline as gpipe
    dev = torch.device("cuda", 0)
    cfg = dataclasses.replace(synth.get_config(args.config), tokens=args.tokens or 16384)
    sub = cfg.sublayers[0]
    m, n, bits, group = sub.m, sub.n, (sub.bits if sub.bits in (2, 4) else 4), sub.group
    site = cfg.site(sub.site)
    X = torch.from_numpy(synth.make_x(cfg, site).view(np.int16)).to(dev).view(torch.bfloat16)
    G_ = torch.from_numpy(synth.make_g(cfg, sub).view(np.int16)).to(dev).view(torch.bfloat16)
    HX, HG = gpipe.covariance(X), gpipe.covariance(G_)
    del X, G_
    su, sv = synth.make_signs(cfg, sub)
    su_d, sv_d = torch.from_numpy(su).to(dev), torch.from_numpy(sv).to(dev)
    W = torch.from_numpy(synth.make_w(cfg, sub)).to(dev)
    res = gpipe.quantize_sublayer(W, HX, HG, su_d, sv_d, bits, group, cfg.alpha, cfg.mode,
                                  cfg.damp, cfg.block)
    torch.cuda.synchronize()
    layer_bytes = res.packed.numel() * 4 + res.scales.numel() * 4 + res.zeros.numel()
    copies = max(2, int(4 * 126 * 2 ** 20 // layer_bytes) + 1)
    packs = [res.packed.clone() for _ in range(copies)]
    x = torch.randn((1, n), device=dev)
    ys = [torch.empty((1, m), device=dev) for _ in range(copies)]
    ws = abi.deploy_workspace(m, n, 1, dev)
    stream = torch.cuda.Stream(dev)

    def call(k):
        abi.kronq_deploy_matvec(packs[k], n, bits, group, res.scales, res.zeros, res.S_X, res.S_G,
                                su_d, sv_d, cfg.mode, x, ys[k], ws, stream=stream)

    with torch.cuda.stream(stream):
        for k in range(copies):
            call(k)
    torch.cuda.synchronize()
    launches0 = abi.kronq_launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for k in range(copies):
            call(k)
    launches_per_replay = abi.kronq_launch_count() - launches0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):          # replay() runs on the current stream
        for _ in range(max(3, args.warmup)):
            g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (args.steps * copies)
    peaks, src = load_peaks()
    algo = layer_bytes + (n + m) * 4
    achieved = algo / (us * 1e-6) / 1e9
    line = {
        "metric": "deploy matvec us per layer (batch 1, packed weights from HBM)", "value": us,
        "unit": "us", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": us * copies / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded generator)",
        "config": {"workload": f"{cfg.name} {sub.name} {m}x{n} W{bits} "
                               f"{'per-channel' if group == -1 else f'g{group}'} BiIP {cfg.mode}",
                   "copies_cycled": copies, "bytes_per_layer": int(algo),
                   "l2": "distinct copies larger than L2 in total, no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": float(peaks["hbm_gbs"]),
                     "unit": "GB/s", "frac": achieved / float(peaks["hbm_gbs"]), "traffic": None,
                     "kernel": "kronq_deploy_matvec (transforms + dequant_matvec_kernel)",
                     "peak_source": src},
        "gpu_launches": launches_per_replay * args.steps,
    }
    print(json.dumps(line), flush=True)


# fp32 CUDA-core peak of a B200 (no measured figure exists for it): 148 SMs x
# 128 fp32 lanes x 2 flops per FMA x the 1965 MHz maximum SM clock.
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1965e6 / 1e12


def stage_rooflines(cfg, layers, steps, stages, inner, peaks, peak_src, peak, peak_kind):
    """Per-kernel roofline entries from the live CUDA-event timings of the
    timed region: the lazy-update GEMMs and the inverse Cholesky's panels and
    updates (library event pairs around their launches, over `steps` steps),
    the inverse Cholesky and BiIP stages (the stage marks, per step).  Algorithmic
    work: lazy update m n (n - 128) flops per sublayer; inverse Cholesky
    2 n^3 / 3 flops; BiIP 8 bytes per element per pass, two passes over each
    of W, H_X, H_G (16 (m n + n^2 + m^2) bytes)."""
    out = {}
    ms, cnt = inner["lazy_update"]
    lazy_flops = sum(L.sub.m * L.sub.n * max(0, L.sub.n - 128) for L in layers)
    if cnt and ms > 0:
        ach = lazy_flops * steps / (ms / 1e3) / 1e12
        out["lazy_update"] = {
            "bound": "tensor", "kernel": "gemm_nt_tc_kernel (solver lazy updates)",
            "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
            "peak_source": f"{peak_src} {peak_kind}", "flops_per_step": lazy_flops,
            "ms_per_step": ms / steps, "launches_per_step": cnt / steps,
            "avg_launch_ms": ms / cnt,
            "note": "each product as three bf16 tensor-core MMAs of hi / lo planes (hi*hi + hi*lo + "
                    "lo*hi, ~2^-17 relative), so the algorithmic ceiling is 1/3 of the bf16 peak"}
    chol_ms = stages.get("inverse_cholesky", 0.0)
    chol_flops = sum(2 * L.sub.n ** 3 / 3 for L in layers)
    # the panel kernels' own work: per 128-wide panel of the padded order np,
    # the slice products (np rows x 128 x 128) and the diagonal block's factor
    # and inverse (2 x 128^3 / 3); the update GEMMs carry the rest
    panel_flops = sum((-(-L.sub.n // 128)) * (2 * 128 * 128 * (-(-L.sub.n // 128) * 128)
                                              + 2 * 128 ** 3 / 3) for L in layers)
    if chol_ms > 0:
        ach = chol_flops / (chol_ms / 1e3) / 1e12
        pan_ms, pan_cnt = inner["chol_panel"]
        upd_ms, upd_cnt = inner["chol_update"]
        entry = {
            "bound": "tensor", "kernel": "panel_kernel + gemm_nt_tc_kernel (kronq_cholesky_inv)",
            "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
            "peak_source": f"{peak_src} {peak_kind}",
            "flops_per_step": chol_flops, "ms_per_step": chol_ms,
            "note": "2 n^3 / 3 per factorisation (Cholesky and triangular inverse); nearly all of it "
                    "in the update GEMMs, whose products run as three tensor-core MMAs of hi / lo "
                    "planes, so the algorithmic ceiling is 1/3 of the 16-bit peak"}
        if pan_cnt and pan_ms > 0:
            pa = panel_flops * steps / (pan_ms / 1e3) / 1e12
            entry["panels"] = {
                "bound": "alu", "achieved": pa, "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                "frac": pa / FP32_ALU_TFLOPS,
                "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz",
                "flops_per_step": panel_flops, "ms_per_step": pan_ms / steps,
                "launches_per_step": pan_cnt / steps,
                "note": "latency-bound: 128 sequential pivots per diagonal block"}
        if upd_cnt and upd_ms > 0:
            ua = (chol_flops - panel_flops) * steps / (upd_ms / 1e3) / 1e12
            entry["updates"] = {
                "bound": "tensor", "achieved": ua, "peak": peak, "unit": "TFLOP/s",
                "frac": ua / peak, "peak_source": f"{peak_src} {peak_kind}",
                "flops_per_step": chol_flops - panel_flops, "ms_per_step": upd_ms / steps,
                "launches_per_step": upd_cnt / steps}
        out["inverse_cholesky"] = entry
    biip_ms = stages.get("biip_sensitivity", 0.0)
    biip_bytes = sum(16 * (L.sub.m * L.sub.n + L.sub.n ** 2 + L.sub.m ** 2) for L in layers)
    if biip_ms > 0:
        hbm = float(peaks["hbm_gbs"])
        ach = biip_bytes / (biip_ms / 1e3) / 1e9
        out["biip"] = {"bound": "hbm", "kernel": "row / column transform passes (kronq_biip_rotate)",
                       "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                       "peak_source": f"{peak_src} hbm_gbs", "bytes_per_step": biip_bytes,
                       "ms_per_step": biip_ms,
                       "note": "stage time includes the norm reductions and the trace sums"}
    obs_ms, obs_cnt = inner["obs_block"]
    if obs_cnt:
        out["obs_block"] = {"bound": "latency", "ms_per_step": obs_ms / steps,
                            "launches_per_step": obs_cnt / steps}
    return out


def run_kernel(args):
    """One kernel alone on a seeded input: --kernel covariance times
    kronq_covariance of a (tokens x width) bf16 matrix (X drawn like the
    workload's widest input site), after untimed warm-up launches."""
    import numpy as np
    import torch
    import dataclasses
    import synth
    from post_quantization_02_b200 import abi
    dev = torch.device("cuda", 0)
    cfg = synth.get_config(args.config)
    site = max(cfg.sites, key=lambda s_: s_.width)
    if args.width:
        site = dataclasses.replace(site, width=args.width)
    tokens = args.tokens or 16384
    cfg = dataclasses.replace(cfg, tokens=tokens)
    X = torch.from_numpy(synth.make_x(cfg, site).view(np.int16)).to(dev).view(torch.bfloat16)
    d = site.width
    H = torch.empty((d, d), dtype=torch.float32, device=dev)
    abi.kronq_covariance(X, H, 1.0 / tokens, 0.0)
    info = torch.zeros(1, dtype=torch.int32, device=dev)
    if args.kernel == "covariance":
        def call():
            abi.kronq_covariance(X, H, 1.0 / tokens, 0.0)
        flops, what = tokens * d * d, "kronq_covariance"
    elif args.kernel == "cholesky":
        del X
        U = torch.empty_like(H)
        ws = abi.workspace(d, d, device=dev)

        def call():
            abi.kronq_cholesky_inv(H, 0.01, U, info, ws)
        flops, what = 2 * d ** 3 / 3, "kronq_cholesky_inv"
    elif args.kernel == "biip":
        del X
        m = args.rows
        G_ = torch.randn((tokens, m), generator=torch.Generator(device=dev).manual_seed(1),
                         device=dev).to(torch.bfloat16)
        HG = torch.empty((m, m), dtype=torch.float32, device=dev)
        abi.kronq_covariance(G_, HG, 1.0 / tokens, 0.0)
        del G_
        W0 = torch.randn((m, d), generator=torch.Generator(device=dev).manual_seed(0),
                         device=dev) * 0.02
        W, HXr, HGr = torch.empty_like(W0), torch.empty_like(H), torch.empty_like(HG)
        su = (torch.randint(0, 2, (m,), device=dev, dtype=torch.int8) * 2 - 1).to(torch.int8)
        sv = (torch.randint(0, 2, (d,), device=dev, dtype=torch.int8) * 2 - 1).to(torch.int8)
        SX = torch.empty(d, device=dev)
        SG = torch.empty(m, device=dev)
        ws = abi.workspace(m, d, device=dev)

        def call():
            W.copy_(W0)
            HXr.copy_(H)
            HGr.copy_(HG)
            abi.kronq_biip_rotate(W, HXr, HGr, su, sv, 0.25, "full", 0, SX, SG, ws)
        flops, what = 16 * (m * d + d * d + m * m), "kronq_biip_rotate (algorithmic bytes)"
    else:
        del X
        U = torch.empty_like(H)
        ws = abi.workspace(args.rows, d, device=dev)
        abi.kronq_cholesky_inv(H, 0.01, U, info, ws)
        sub = cfg.sublayers[0]
        W0 = torch.randn((args.rows, d), generator=torch.Generator(device=dev).manual_seed(0),
                         device=dev) * 0.02
        W = torch.empty_like(W0)
        codes = torch.empty((args.rows, d), dtype=torch.uint8, device=dev)
        G = 1 if sub.group == -1 else d // sub.group
        scales = torch.empty((args.rows, G), device=dev)
        zeros = torch.empty((args.rows, G), dtype=torch.uint8, device=dev)

        def call():
            W.copy_(W0)
            abi.kronq_quantize_layer(W, U, sub.bits or 4, sub.group, 128, codes, scales, zeros,
                                     None, info, ws)
        flops, what = args.rows * d * (d - 128), "kronq_quantize_layer (lazy-update flops)"
    for _ in range(max(1, args.warmup)):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    if info.item() != 0:
        raise RuntimeError(f"device status {info.item()}")
    ms = e0.elapsed_time(e1) / args.steps
    peaks, src = load_peaks()
    rate = flops / (ms / 1e3) / 1e12
    if args.kernel == "biip":
        out = {"tb_per_s": rate, "frac_of_hbm": rate * 1e3 / float(peaks["hbm_gbs"])}
    else:
        out = {"tflops": rate, "frac_of_burst_peak": rate / float(peaks["bf16_tflops"])}
    print(json.dumps({"kernel": what, "tokens": tokens, "width": d, "rows": args.rows, "ms": ms,
                      **out, "peak_source": src}), flush=True)


def run_gptaq(args):
    """One step per sublayer: H~, Delta X X^T = kronq_drift_covariance([X~ | X]),
    H_G, BiIP, the drift covariance rotated like H~, inverse Cholesky, P,
    the column loop with the P term, packing.  Inputs resident in HBM."""
    import dataclasses
    import numpy as np
    import torch
    import synth
    from post_quantization_02_b200 import abi
    from concurrent.futures import ThreadPoolExecutor
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = synth.get_config(args.config)
    if args.tokens:
        cfg = dataclasses.replace(cfg, tokens=args.tokens)
    N = cfg.tokens
    t_gen = time.perf_counter()
    xqx, gs = {}, {}
    for site in cfg.sites:
        buf = torch.empty((N, 2 * site.width), dtype=torch.bfloat16, device=dev)

        def pair(c, site=site):
            xb = synth.x_chunk(cfg, site, c)
            return c, np.concatenate([synth.xq_chunk(cfg, site, c, x_bits=xb), xb], axis=1)

        with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
            for c, bits in ex.map(pair, range(synth.n_chunks(N))):
                r0 = c * synth.CHUNK_TOKENS
                buf[r0:r0 + len(bits)].copy_(torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
                                             .view(torch.bfloat16))
        xqx[site.name] = buf
    for sub in cfg.sublayers:
        gs[sub.name] = torch.from_numpy(synth.make_g(cfg, sub).view(np.int16)).to(dev).view(torch.bfloat16)
    t_gen = time.perf_counter() - t_gen
    L = []
    for sub in cfg.sublayers:
        m, n = sub.m, sub.n
        su, sv = synth.make_signs(cfg, sub)
        G = 1 if sub.group == -1 else n // sub.group
        L.append(dict(sub=sub, W0=torch.from_numpy(synth.make_w(cfg, sub)).to(dev),
                      W=torch.empty((m, n), device=dev), HX=torch.empty((n, n), device=dev),
                      A=torch.empty((n, n), device=dev), HG=torch.empty((m, m), device=dev),
                      U=torch.empty((n, n), device=dev), P=torch.empty((n, n), device=dev),
                      SX=torch.empty(n, device=dev), SG=torch.empty(m, device=dev),
                      su=torch.from_numpy(su).to(dev), sv=torch.from_numpy(sv).to(dev),
                      codes=torch.empty((m, n), dtype=torch.uint8, device=dev),
                      scales=torch.empty((m, G), device=dev),
                      zeros=torch.empty((m, G), dtype=torch.uint8, device=dev),
                      packed=torch.empty((m, abi.packed_words(n, sub.bits or 4)), dtype=torch.int32,
                                         device=dev)))
    ws = abi.gptaq_workspace(max(s.m for s in cfg.sublayers), max(s.n for s in cfg.sublayers), dev)
    info = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = {}

    def step(marks=None):
        def mark(k):
            if marks is not None:
                e = torch.cuda.Event(enable_timing=True)
                e.record(stream)
                marks.append((k, e))
        mark("start")
        for d in L:
            sub = d["sub"]
            abi.kronq_drift_covariance(xqx[sub.site], d["HX"], d["A"], info, ws)
            abi.kronq_covariance(gs[sub.name], d["HG"], 1.0 / N, 0.0)
        mark("covariances")
        for d in L:
            sub = d["sub"]
            d["W"].copy_(d["W0"])
            abi.kronq_biip_rotate(d["W"], d["HX"], d["HG"], d["su"], d["sv"], cfg.alpha, cfg.mode, 0,
                                  d["SX"], d["SG"], ws)
            abi.kronq_biip_rotate_input(d["A"], d["SX"], d["sv"], cfg.mode, ws)
            abi.kronq_cholesky_inv(d["HX"], cfg.damp, d["U"], info, ws)
            abi.kronq_gptaq_correction(d["A"], d["U"], 0.25, d["P"], info, ws)
        mark("biip_cholesky_correction")
        for d in L:
            sub = d["sub"]
            abi.kronq_quantize_layer_gptaq(d["W"], d["U"], d["P"], sub.bits, sub.group, cfg.block,
                                           d["codes"], d["scales"], d["zeros"], None, info, ws)
            if sub.bits in (2, 4):
                abi.kronq_pack(d["codes"], sub.bits, d["packed"])
        mark("solver_pack")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if info.item() != 0:
        raise RuntimeError(f"device status {info.item()} in warm-up")
    marks_all = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        marks = []
        step(marks)
        marks_all.append(marks)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    stages = {}
    for marks in marks_all:
        for (_, a), (k, b2) in zip(marks, marks[1:]):
            stages[k] = stages.get(k, 0.0) + a.elapsed_time(b2) / args.steps
    print(json.dumps({"metric": METRIC + " (GPTAQ asymmetric calibration)", "value":
                      cfg.weights / (ms / 1e3) / 1e6, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                      "dtype": "bf16", "data": "synthetic (seeded generator; drifted X~ = X + noise)",
                      "config": {"workload": workload_desc(cfg) + "; GPTAQ alpha 0.25",
                                 "input_gen_s": round(t_gen, 1)},
                      "stages_ms": {k: round(v, 3) for k, v in stages.items()}}), flush=True)


def main():
    args = parse()
    if args.gptaq:
        run_gptaq(args)
        return
    if args.kernel:
        run_kernel(args)
        return
    if args.deploy:
        run_deploy(args)
        return
    if args.oracle_full_chain:
        oracle_full_chain(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import numpy as np
    import torch
    import torch.distributed as dist
    import synth
    from post_quantization_02_b200 import abi
    from post_quantization_02_b200 import pipeline as gpipe

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    abi.lib()
    import dataclasses
    cfg0 = synth.get_config(args.config)
    if args.tokens:
        cfg0 = dataclasses.replace(cfg0, tokens=args.tokens)
    cfg = rank_config(cfg0, rank)   # each rank: its own layer (weak scaling)

    # ---- seeded inputs on the host (pinned for the end-to-end leg), then HBM.
    # When every rank's host copies (and their pinned twins) would not fit the
    # host's memory, each rank draws its inputs chunk by chunk straight into
    # device memory with its share of the host cores, and has no e2e leg.
    in_bytes = host_input_bytes(cfg)
    ram = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES")
    lean = needs_lean_inputs(cfg, world, not args.no_e2e, ram)
    t_gen = time.perf_counter()
    host = {"X": {}, "G": {}}
    if lean:
        threads = max(1, (os.cpu_count() or 1) // world)
        X = {s_.name: draw_to_device(lambda c, s_=s_: synth.x_chunk(cfg, s_, c), cfg.tokens,
                                     s_.width, dev, threads) for s_ in cfg.sites}
        Gd = {sub.name: draw_to_device(lambda c, sub=sub: synth.g_chunk(cfg, sub, c), cfg.tokens,
                                       sub.m, dev, threads) for sub in cfg.sublayers}
    else:
        for site in cfg.sites:
            host["X"][site.name] = synth.make_x(cfg, site)
        for sub in cfg.sublayers:
            host["G"][sub.name] = synth.make_g(cfg, sub)
        X = {s_: torch.from_numpy(v.view(np.int16)).to(dev).view(torch.bfloat16)
             for s_, v in host["X"].items()}
        Gd = {s_: torch.from_numpy(v.view(np.int16)).to(dev).view(torch.bfloat16)
              for s_, v in host["G"].items()}
    t_gen = time.perf_counter() - t_gen
    layers = [Layer(cfg, sub, dev, rank, Gd[sub.name], args.act_order) for sub in cfg.sublayers]
    mmax = max(s.m for s in cfg.sublayers)
    nmax = max(s.n for s in cfg.sublayers)
    ws = abi.workspace(mmax, nmax, device=dev)
    stream = torch.cuda.current_stream(dev)
    weights = cfg.weights

    ncov = len(cfg.sites) + len(cfg.sublayers)
    for _ in range(args.warmup):
        gpu_step(cfg, layers, X, ws, stream, None, args.act_order, args.w_clip)
    torch.cuda.synchronize()
    for L in layers:
        if L.info.item() != 0:
            raise RuntimeError(f"device status {L.info.item()} in warm-up")

    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()
    time.sleep(0.3)
    cov_events = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * ncov)] for _ in range(args.steps)]
    stage_marks = [StageMarks(stream) for _ in range(args.steps)]
    launches0 = abi.kronq_launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(args.steps):
        if k == args.steps - 1:
            # event pairs around the library's inner launches, in the last timed
            # step only (they cost a little time per launch)
            abi.kronq_timing_enable(True)
        gpu_step(cfg, layers, X, ws, stream, cov_events[k], args.act_order, args.w_clip,
                 stage_marks[k])
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler.mark_end()
    launches = abi.kronq_launch_count() - launches0
    inner = {k: abi.kronq_timing_read(k) for k in abi.TIMERS}
    abi.kronq_timing_enable(False)
    ms = reduce_max_ms(start.elapsed_time(end), world, dev)
    cov_ms = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for ev in cov_events for i in range(ncov)]
    stages = {}
    for sm_ in stage_marks:
        for name, t in sm_.totals().items():
            stages[name] = stages.get(name, 0.0) + t / args.steps

    # ---- end to end through the public API with pinned host buffers
    e2e = None
    e2e_skipped = None
    if lean and not args.no_e2e:
        e2e_skipped = (f"{world} ranks x {2 * in_bytes / 2 ** 30:.0f} GiB of host and pinned input "
                       f"copies exceed 60 % of the host's {ram / 2 ** 30:.0f} GiB")
    if not args.no_e2e and not lean:
        pin = {"X": {s: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory()
                     for s, v in host["X"].items()},
               "G": {s: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory()
                     for s, v in host["G"].items()},
               "W": {L.sub.name: L.W0.cpu().pin_memory() for L in layers}}
        outs = {L.sub.name: (torch.empty(L.packed_store.shape, dtype=torch.int32).pin_memory(),
                             torch.empty(L.scales.shape).pin_memory(),
                             torch.empty(L.zeros.shape, dtype=torch.uint8).pin_memory()) for L in layers}
        copy_stream = torch.cuda.Stream(dev)
        staging = {}

        def cov_host(A_host, H, width):
            if width not in staging:
                staging[width] = [torch.empty((16384, width), dtype=torch.bfloat16, device=dev)
                                  for _ in range(2)]
            return gpipe.covariance_from_host(A_host, H, copy_stream=copy_stream, stream=stream,
                                              staging=staging[width])

        solve_stream = torch.cuda.Stream(dev)

        def finish_layer(L, st):
            """BiIP, s, inverse Cholesky, solver, pack and the D2H copies of one
            sublayer on stream st; returns the bytes copied back."""
            abi.kronq_biip_rotate(L.W, L.HX, L.HG, L.su, L.sv, cfg.alpha, cfg.mode, 0, L.SX, L.SG,
                                  ws, stream=st)
            abi.kronq_sensitivity(L.HX, L.HG, L.sens, stream=st)
            solve_layer(cfg, L, ws, st, args.act_order, args.w_clip)
            pk, sc, zr = outs[L.sub.name]
            n_out = 0
            with torch.cuda.stream(st):
                if L.bits in (2, 4):
                    pv = packed_view(L, L.bits)
                    abi.kronq_pack(L.codes, L.bits, pv, stream=st)
                    pk[: pv.numel()].copy_(pv.view(-1), non_blocking=True)
                    n_out += pv.numel() * 4
                sc.copy_(L.scales, non_blocking=True)
                zr.copy_(L.zeros, non_blocking=True)
            return n_out + L.scales.numel() * 4 + L.zeros.numel()

        def e2e_step():
            """One step from pinned host buffers.  Fixed bit widths: sublayer by
            sublayer (widest input first), each sublayer's chain on a second
            stream as soon as its covariances are done, while the next
            sublayer's inputs stream in (the host-to-device copies bound the
            step).  A mixed 2/3/4-bit allocation needs every score first, so it
            runs stage by stage."""
            h2d = d2h = 0
            Hs = {}

            def site_cov(site):
                nonlocal h2d
                L0 = next(L for L in layers if L.sub.site == site.name)
                h2d += cov_host(pin["X"][site.name], L0.HX, site.width)
                Hs[site.name] = L0.HX
                for L in layers:            # a shared input: every sublayer rotates its own copy
                    if L.sub.site == site.name and L.HX is not L0.HX:
                        L.HX.copy_(L0.HX)

            if cfg.mixed_avg_bits:
                for site in cfg.sites:
                    site_cov(site)
                for L in layers:
                    h2d += cov_host(pin["G"][L.sub.name], L.HG, L.sub.m)
                    L.W.copy_(pin["W"][L.sub.name], non_blocking=True)
                    h2d += L.W.numel() * 4 + L.su.numel() + L.sv.numel()
                for L in layers:
                    d2h += finish_layer(L, stream)
                return h2d, d2h
            # the widest input first: its inverse Cholesky (~n^3) is the
            # longest chain, and it runs while the others' inputs stream in
            for L in sorted(layers, key=lambda L_: -L_.sub.n):
                if L.sub.site not in Hs:
                    site_cov(cfg.site(L.sub.site))
                h2d += cov_host(pin["G"][L.sub.name], L.HG, L.sub.m)
                L.W.copy_(pin["W"][L.sub.name], non_blocking=True)
                h2d += L.W.numel() * 4 + L.su.numel() + L.sv.numel()
                ready = torch.cuda.Event()
                ready.record(stream)
                solve_stream.wait_event(ready)
                d2h += finish_layer(L, solve_stream)
            done = torch.cuda.Event()
            done.record(solve_stream)
            stream.wait_event(done)
            return h2d, d2h

        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.e2e_steps):
            h2d, d2h = e2e_step()
        s1.record(stream)
        torch.cuda.synchronize()
        e_ms = reduce_max_ms(s0.elapsed_time(s1), world, dev)
        e2e = {"value": job_throughput(weights, world, args.e2e_steps, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e_ms / args.e2e_steps}
    time.sleep(0.3)
    sampler.stop()
    clocks = sampler.summary()

    value = job_throughput(weights, world, args.steps, ms)
    peaks, peak_src = load_peaks()
    timed_s = ms / 1e3
    peak_kind = "bf16_tflops_sustained" if timed_s >= 1.0 else "bf16_tflops"
    peak = float(peaks.get(peak_kind, peaks.get("bf16_tflops")))
    cov_flops = []
    for s in cfg.sites:
        cov_flops.append(cfg.tokens * s.width ** 2)
    for sub in cfg.sublayers:
        cov_flops.append(cfg.tokens * sub.m ** 2)
    avg_ms = statistics.mean(cov_ms)
    achieved = statistics.mean(cov_flops) / (avg_ms / 1e3) / 1e12
    workload = workload_desc(cfg0)
    roofline = {"bound": "tensor", "kernel": "cov_pair_kernel (kronq_covariance)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": load_traffic(workload),
                "peak_source": f"{peak_src} {peak_kind}",
                "flops_per_launch": statistics.mean(cov_flops), "avg_launch_ms": avg_ms,
                "launches_timed": len(cov_ms)}
    rooflines = stage_rooflines(cfg0, layers, 1, stages, inner, peaks, peak_src, peak, peak_kind)
    rooflines["covariance"] = {k: roofline[k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                                        "avg_launch_ms", "flops_per_launch")}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        est, sample = oracle_sample(cfg0)
        cpu = {"value": cfg0.weights / est / 1e6, "unit": UNIT, "cores": blas_threads(),
               "kind": "oracle", "sample": sample, "host_cpus": os.cpu_count(),
               "cpu_model": host_cpu_model()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded generator; stands in for WikiText-2 activations and LLaMA weights)",
            "config": {"workload": workload, "parallelism": f"replicas x{world} (one layer per GPU)",
                       "l2": l2_note(cfg0),
                       "solver_dtype": "fp32", "input_gen_s": round(t_gen, 1),
                       "act_order": args.act_order, "w_clip": args.w_clip},
            "roofline": roofline, "rooflines": rooflines, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches,
            **({"e2e_skipped": e2e_skipped} if e2e_skipped else {}),
            "clocks": clocks,
            "stages_ms": {k: round(v, 4) for k, v in stages.items()},
            # the solver alone, given H_X': inverse Cholesky + OBS loop
            "solver_only_mweights_s": (
                weights / ((stages.get("inverse_cholesky", 0.0) + stages.get("solver", 0.0)) / 1e3) / 1e6
                if stages.get("inverse_cholesky", 0.0) + stages.get("solver", 0.0) > 0 else None),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
