#!/usr/bin/env python
"""Benchmark of batched speculative-draft verification on B200.

One step = one pass of the whole hot path over one batch: DVL allocation
(for the workloads with a verify budget), the fused temperature-softmax
statistics of the verify window, the accept tests with first-rejection
ballot, and the residual / bonus Gumbel-max draw. Metric: verified
request-blocks per second (one request-block = one request's verify step),
with the achieved HBM bandwidth against the measured B200 copy peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 5] [--extras 2,3,4]
                    [--impl specv|reference]

The headline workload is the stress case (B=64, L=16, V=151936, K=4
latent-mixture drafts, bf16, DVL budget 544 = half of B(L+1)), the largest
of the five seeded workloads; --extras measures further workloads in the
same run with the same protocol and reports them under "workloads".

Under torchrun every rank verifies its own batch (weak scaling, no
collective on the data path); the time is the max over ranks. Prints one
JSON line on rank 0.

Timing: inputs live in HBM; --sets rotating input sets (4 by default, each
above 160 MB, together far above the 126 MB L2), so each step reads its
logits from HBM. The headline `value` is K CUDA-graph replays of the step
between one pair of CUDA events on the launching stream. The same step is
also timed replay by replay (one event pair each; median and spread), both
as graph replays and as plain stream launches through the public API, which
gives the launch-gap saving of the captured graph. The dominant kernel (row
statistics) is timed alone with events for the roofline fraction. The e2e
leg copies each step's inputs from pinned host memory and reads the results
back inside the timed region.
"""
import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified request-blocks/sec and achieved HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "request-blocks/s"
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 2 ** 20
HEADLINE = 5
EPS_MARGIN = 1e-6


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", type=int, default=HEADLINE, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--extras", default="1,2,3,4",
                    help="comma-separated further workloads measured in the same run ('' for none)")
    ap.add_argument("--sets", type=int, default=4, help="rotating input sets (together above the L2 size)")
    ap.add_argument("--top-p-extras", default="3", help="workloads also measured with top-p filtering ('' for none)")
    ap.add_argument("--top-p", type=float, default=0.95, help="top-p of the filtered measurements")
    ap.add_argument("--impl", default="specv", choices=["specv", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the oracle CPU-baseline sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    args.extra_ids = [int(c) for c in args.extras.split(",") if c.strip()] if args.extras else []
    args.extra_ids = [c for c in args.extra_ids if c != args.workload]
    args.top_p_ids = [int(c) for c in args.top_p_extras.split(",") if c.strip()] if args.top_p_extras else []
    return args


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (1 Gi bf16 copy, burst) of measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback 6.65 TB/s (MEASURED_PEAKS.json absent)"


# ---------------------------------------------------------------- workload

STATS_BURST_REPLAYS = 50  # replays of the statistics graph in its burst timing
STATS_BURST_PAUSE_S = 0.5  # idle time before the burst


def window_bytes(w, verify_len):
    """Algorithmic bytes of the statistics stage: every tested target row and
    the K draft rows of every tested position, read once."""
    e = 2 if w.dtype == "bf16" else 4
    return int(sum((w.K + 1) * int(l) for l in verify_len)) * w.V * e


def step_bytes(w, verify_len, accept_len):
    """Algorithmic bytes of one verify step: the window, one fp32 Gumbel row
    per request, the bonus target row of the requests that accepted every
    tested position, and the small per-request arrays.

    The bonus row is counted only where the method reads it (a request that
    accepted all of its l_b positions draws its last token from target row
    l_b); the survey's byte model counts (l_b + 1) target rows for every
    request, which overstates the bytes of requests that reject."""
    e = 2 if w.dtype == "bf16" else 4
    bonus = sum(1 for l, a in zip(verify_len, accept_len) if a == l)
    small = w.B * (w.L * 4 * 2 + 4 + (w.L + 1) * 4)
    if w.budget is not None:
        small += w.B * w.L * 4 + w.B * 4 + (w.B + 1) * 4 + w.budget * 4
    return window_bytes(w, verify_len) + w.B * w.V * 4 + bonus * w.V * e + small


def set_bytes(w):
    """Device bytes of one input set: target (dense, plus the packed rows with
    a budget), draft, Gumbel noise and the small arrays."""
    e = 2 if w.dtype == "bf16" else 4
    n = w.B * (w.L + 1) * w.V * e + w.B * w.K * w.L * w.V * e + w.B * (w.L + 1) * w.V * 4
    n += w.B * w.L * 8 + (w.B * w.K * 4 if w.K > 1 else 0)
    if w.budget is not None:
        n += w.budget * w.V * e + w.B * w.L * 4
    return n


def l2_note(w, nsets):
    return "%d rotating input sets of %.0f MB (%s the 126 MB L2 together)" % (
        nsets, set_bytes(w) / 1e6, "above" if nsets * set_bytes(w) > L2_BYTES else "NOT above")


def config_of(w, nsets, world):
    """The workload description shared by both arms (same keys and values)."""
    return {"workload": w.name, "B": w.B, "L": w.L, "V": w.V, "K": w.K, "T": w.T, "budget": w.budget,
            "l2": l2_note(w, nsets), "parallelism": "dp%d" % world}


def spread(ms):
    """Median and spread of per-replay times (ms)."""
    a = np.sort(np.asarray(ms, np.float64))
    q = lambda f: float(a[min(len(a) - 1, int(round(f * (len(a) - 1))))])
    return {"median_ms": q(0.5), "p10_ms": q(0.1), "p90_ms": q(0.9), "min_ms": float(a[0]), "max_ms": float(a[-1]),
            "n": int(len(a))}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi in its own process (`-lms`), started before the warm-up and
    stopped after the timed region; the report keeps the samples whose
    timestamps fall inside the timed region. It only reads the clocks."""

    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, cuda_index, period_ms=20):
        import subprocess
        import tempfile
        self.region = None
        self.err = None
        self.proc = None
        self.period_ms = period_ms
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(cuda_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            sel = vis.split(",")[cuda_index] if vis else str(cuda_index)
        cmd = ["nvidia-smi", "-i", sel, "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
               "-lms", str(period_ms)]
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)  # let it take its first samples before the warm-up
        except OSError as exc:
            self.err = repr(exc)

    def stop(self):
        if self.proc is not None:
            time.sleep(0.05)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def report(self):
        import datetime
        if self.proc is None:
            return {"error": self.err}
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) != len(self.FIELDS):
                continue
            try:
                t = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((t, float(f[1]), float(f[2]), f[4:]))
            except ValueError:
                continue
        if not rows:
            return {"error": "no nvidia-smi samples"}
        t0, t1 = self.region
        inside = [r for r in rows if t0 <= r[0] <= t1]
        note = "nvidia-smi -lms %d during the timed region" % self.period_ms
        if not inside:
            inside = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:2]
            note = "nvidia-smi -lms %d, the samples nearest the timed region (region shorter than the period)" \
                   % self.period_ms
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        active = sorted({names[k] for r in inside for k, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": inside[0][2], "reasons": active,
                "samples": len(inside), "source": note}


# ------------------------------------------------------------ the oracle leg

def oracle_sample(x, requests, n_threads, diag=False):
    """One oracle verify over the first `requests` requests of inputs x (with
    a budget: the oracle's own allocation and packing of the whole batch)."""
    import oracle
    w = x.w
    sl = slice(0, requests)
    if w.budget is None:
        return oracle.verify(x.target[sl], x.draft[sl], x.tokens[sl], x.u[sl], x.g[sl], w.T,
                             mix_w=None if x.mix_w is None else x.mix_w[sl], n_threads=n_threads, diag=diag)
    rd = oracle.dvl_allocate(x.scores, w.budget)
    packed = oracle.pack(x.target, rd["verify_len"], rd["offsets"], w.budget)
    r = oracle.verify(packed, x.draft[sl], x.tokens[sl], x.u[sl], x.g[sl], w.T,
                      mix_w=None if x.mix_w is None else x.mix_w[sl], verify_len=rd["verify_len"][sl],
                      target_row_off=rd["offsets"][:w.B][sl], n_threads=n_threads, diag=diag)
    r["verify_len"] = rd["verify_len"][sl]
    return r


def margin_report(acc, out, ref, verify_len):
    """Decisions of one verify call and the low-margin ones among them, as the
    parity rule counts them: every tested accept decision and the terminal
    draw; an accept test is low-margin when |u - min(1, rho)| < 1e-6, a draw
    when the fp64 gap between its two best scores is below 1e-6 * max(1,
    kappa). `mismatches` counts GPU outputs that differ from the oracle's
    outside the low-margin exemption (0 is parity)."""
    n_dec = n_low = n_exempt_diff = n_bad = 0
    L = out.shape[1] - 1
    for b in range(out.shape[0]):
        ja = int(ref["accept_len"][b])
        if ja < 0:
            n_bad += int(not (acc[b] == -1 and np.all(out[b] == -1)))
            continue
        ell = L if verify_len is None else int(verify_len[b])
        tested = ja + 1 if ja < ell else ja
        m = ref["accept_margin"][b]
        n_dec += tested + 1
        low = [i for i in range(tested) if m[i] < EPS_MARGIN]
        same = acc[b] == ja and np.array_equal(out[b], ref["out_tokens"][b])
        if low:  # exempt from the first low-margin test on; the outputs before it must still match
            n_low += 1
            i0 = low[0]
            before_ok = acc[b] >= i0 and np.array_equal(out[b, :i0], ref["out_tokens"][b][:i0])
            n_bad += int(not same and not before_ok)
            n_exempt_diff += int(not same and before_ok)
            continue
        if ref["argmax_gap"][b] < EPS_MARGIN * max(1.0, ref["argmax_kappa"][b]):
            n_low += 1
            same_prefix = acc[b] == ja and np.array_equal(out[b, :ja], ref["out_tokens"][b, :ja])
            n_bad += int(not same_prefix)
            n_exempt_diff += int(same_prefix and not same)
            continue
        n_bad += int(not same)
    return {"decisions": n_dec, "low_margin": n_low, "low_margin_fraction": n_low / max(1, n_dec),
            "exempted_differences": n_exempt_diff, "mismatches": n_bad}


def cpu_baseline(x, seconds, gpu_out=None):
    """The oracle as it stands, on this host's cores, repeated for about
    `seconds`. With the GPU's outputs on the same inputs, one further oracle
    run with diagnostics (outside the timed loop) counts the decisions and
    the low-margin ones, and checks the GPU's outputs against it."""
    import oracle
    cores = oracle.n_cores()
    w = x.w
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle_sample(x, w.B, cores)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    res = {"value": reps * w.B / dt, "unit": UNIT, "cores": min(cores, w.B), "kind": "oracle",
           "sample": "full workload (%d requests) x %d repetitions, %.1f s; fp64 C oracle, pthreads over requests"
                     % (w.B, reps, dt)}
    margins = None
    if gpu_out is not None:
        ref = oracle_sample(x, w.B, cores, diag=True)
        margins = margin_report(gpu_out[0], gpu_out[1], ref, ref.get("verify_len"))
        margins["source"] = "oracle with diagnostics on input set 0, against the GPU's outputs on it"
    return res, margins


def run_reference(args, rank, world):
    """The oracle as the reference arm: same workload, metric and unit, on the
    host cores. Each step verifies a bounded sample of the workload (whole
    requests when K + W steps fit ~3 minutes, else fewer tested positions of
    one request); the value counts request-block equivalents (tested rows of
    the sample / tested rows of one full request-block)."""
    if rank != 0:
        return 0
    from speculative_decoding_block_spec_b200 import synth
    import oracle
    x = synth.workload_inputs(args.workload)
    w = x.w
    cores = oracle.n_cores()
    req = int(max(1, min(w.B, cores)))  # requests run in parallel, one thread each
    oracle_sample(x, req, cores)
    t0 = time.perf_counter()
    oracle_sample(x, req, cores)
    t1 = time.perf_counter() - t0  # one full step of `req` requests on all cores
    budget = 150.0 / max(1, args.steps + args.warmup)
    ell = w.L if t1 <= budget or w.L == 0 else int(max(1, min(w.L, w.L * budget / t1)))
    frac = ell / w.L if w.L else 1.0

    def one_step():
        if ell == w.L:
            oracle_sample(x, req, cores)
        else:
            sl = slice(0, req)
            oracle.verify(x.target[sl], x.draft[sl], x.tokens[sl], x.u[sl], x.g[sl], w.T,
                          mix_w=None if x.mix_w is None else x.mix_w[sl],
                          verify_len=np.full(req, ell, np.int32), n_threads=cores)

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = time.perf_counter() - t0
    value = args.steps * req * frac / dt
    sample = ("%d of %d requests per step" % (req, w.B)) if ell == w.L else \
        ("%d requests with %d of %d positions tested per step (%.3f request-blocks each)" % (req, ell, w.L, frac))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": config_of(w, args.sets, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(cores, req), "kind": "oracle",
                             "sample": sample + " (%s); fp64 C oracle on the host cores" % w.name},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ traffic

def stats_kernel_name(w, sms):
    """The statistics kernel the library picks for this workload: the
    one-block-per-SM balanced kernel for 16-byte rows, windows of at most
    256 MB, at least 4096 units (2 KB slices for 32 warps) per SM and at most
    32 rows per SM share; otherwise the even-split kernel. The window bound
    is the dense one, B (K+1) L rows."""
    esz = 2 if w.dtype == "bf16" else 4
    if (w.V * esz) % 16:
        return "k_row_stats"
    vu = w.V * esz // 16
    units = w.B * (w.K + 1) * w.L * vu
    share = -(-units // sms)
    if units * 16 <= (256 << 20) and share >= 32 * 128 and -(-share // vu) + 1 <= 32:
        return "k_row_stats_dyn"
    return "k_row_stats"


def committed_traffic(kernel, workload_name):
    """Per-launch DRAM bytes from a committed ncu summary, if it was taken on
    the current kernel source (sha256 of the csrc files it names)."""
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(path).read()
        m = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
        k = re.search(r"kernel:\s*(\S+)", text)
        wl = re.search(r"workload:\s*(.+)", text)
        h = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
        files = re.search(r"source_files:\s*(.+)", text)
        if not (m and k and h and files and wl) or k.group(1) != kernel or wl.group(1).strip() != workload_name:
            continue
        d = hashlib.sha256()
        for f in files.group(1).split():
            with open(os.path.join(ROOT, f), "rb") as fh:
                d.update(fh.read())
        if d.hexdigest() == h.group(1):
            return int(m.group(1)), os.path.relpath(path, ROOT)
    return None, None


# -------------------------------------------------------------- specv leg

class Runner:
    """Device-side state of one workload: its rotating input sets, the step
    through the public API, and the CUDA graphs that replay it."""

    def __init__(self, w, x, dev, stream, nsets, top_p=1.0):
        import torch
        import speculative_decoding_block_spec_b200 as specv
        self.torch, self.specv = torch, specv
        self.w, self.x, self.dev, self.stream = w, x, dev, stream
        self.top_p = top_p

        def logits(a):
            if a.dtype == np.uint16:
                return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
            return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

        self.sets = []
        with torch.cuda.stream(stream):
            for _ in range(nsets):
                d = dict(target=logits(x.target), draft=logits(x.draft), tokens=torch.from_numpy(x.tokens).to(dev),
                         u=torch.from_numpy(x.u).to(dev), g=torch.from_numpy(x.g).to(dev))
                if x.mix_w is not None:
                    d["mix_w"] = torch.from_numpy(x.mix_w).to(dev)
                if x.scores is not None:
                    d["scores"] = torch.from_numpy(x.scores).to(dev)
                    d["packed"] = torch.zeros((w.budget, w.V), dtype=d["target"].dtype, device=dev)
                    d["dvl_ws"] = specv.Workspace(specv.dvl_workspace_size(w.B), dev)
                    d["dvl_out"] = (torch.empty(w.B, dtype=torch.int32, device=dev),
                                    torch.empty(w.B + 1, dtype=torch.int32, device=dev),
                                    torch.empty(w.budget, dtype=torch.int32, device=dev))
                d["ws"] = specv.Workspace(specv.verify_top_p_workspace_size(w.B, w.L, w.K, w.V) if top_p < 1 else
                                          specv.verify_workspace_size(w.B, w.L, w.K, w.V), dev)
                d["out"] = (torch.empty(w.B, dtype=torch.int32, device=dev),
                            torch.empty((w.B, w.L + 1), dtype=torch.int32, device=dev))
                self.sets.append(d)
            stream.synchronize()
        self.launches_per_step = (2 if w.L > 0 else 1) + (1 if w.budget is not None else 0)
        self.graphs = {}

    def prepack(self, d):
        """DVL allocation plus the copy of the selected dense target rows into
        the fixed-address packed buffer. In deployment the target model writes
        its logits straight into the packed slots, so the copy is not part of
        the verify step: it runs once per input set here and is timed apart."""
        self.specv.dvl_allocate_pack(d["scores"], self.w.budget, dense_target=d["target"],
                                     packed_target=d["packed"], workspace=d["dvl_ws"], out=d["dvl_out"])

    def step(self, d):
        """One verify step through the public API (the launches a user makes):
        with a DVL budget, the allocation over the survival scores, then
        verification of the packed rows at the allocated offsets; with top-p,
        the filtered verification."""
        w, specv = self.w, self.specv
        vl = off = None
        target = d["target"]
        if w.budget is not None:
            vl, off, _ = specv.dvl_allocate_pack(d["scores"], w.budget, workspace=d["dvl_ws"], out=d["dvl_out"])
            off = off[:w.B]
            target = d["packed"]
        if self.top_p < 1:
            if w.K == 1:
                return specv.spec_verify_block_top_p(target, d["draft"], d["tokens"], d["u"], d["g"], w.T,
                                                     self.top_p, verify_len=vl, target_row_off=off,
                                                     workspace=d["ws"], out=d["out"])
            return specv.spec_verify_mixture_top_p(target, d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], w.T,
                                                   self.top_p, verify_len=vl, target_row_off=off, workspace=d["ws"],
                                                   out=d["out"])
        if w.K == 1:
            return specv.spec_verify_block(target, d["draft"], d["tokens"], d["u"], d["g"], w.T, verify_len=vl,
                                           target_row_off=off, workspace=d["ws"], out=d["out"])
        return specv.spec_verify_mixture(target, d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], w.T,
                                         verify_len=vl, target_row_off=off, workspace=d["ws"], out=d["out"])

    def _window(self, d):
        if self.w.budget is not None:
            return d["dvl_out"][0], d["dvl_out"][1][:self.w.B], d["packed"]
        return None, None, d["target"]

    def verify_only(self, d):
        """The verify call alone (the DVL outputs of the last step stay fixed)."""
        w, specv = self.w, self.specv
        vl, off, target = self._window(d)
        if w.K == 1:
            specv.spec_verify_block(target, d["draft"], d["tokens"], d["u"], d["g"], w.T, verify_len=vl,
                                    target_row_off=off, workspace=d["ws"], out=d["out"])
        else:
            specv.spec_verify_mixture(target, d["draft"], d["mix_w"], d["tokens"], d["u"], d["g"], w.T,
                                      verify_len=vl, target_row_off=off, workspace=d["ws"], out=d["out"])

    def stats_only(self, d):
        """Stage 1 alone: the statistics kernel, the dominant launch."""
        vl, off, target = self._window(d)
        self.specv.spec_verify_window_stats(target, d["draft"], d["tokens"], self.w.T, d["ws"], verify_len=vl,
                                            target_row_off=off)

    def capture(self, name, fn):
        torch = self.torch
        gs = []
        with torch.cuda.stream(self.stream):
            for d in self.sets:
                fn(d)  # warm the library's per-device caches and the kernels before capture
            self.stream.synchronize()
            for d in self.sets:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=self.stream):
                    fn(d)
                gs.append(g)
            self.stream.synchronize()
        self.graphs[name] = gs
        return gs

    def capture_all(self, name, fn):
        """One graph that calls fn once per input set, back to back."""
        torch = self.torch
        with torch.cuda.stream(self.stream):
            for d in self.sets:
                fn(d)
            self.stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                for d in self.sets:
                    fn(d)
            self.stream.synchronize()
        self.graphs[name] = [g]
        return g

    def release(self):
        self.graphs.clear()
        self.sets.clear()


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    from speculative_decoding_block_spec_b200 import synth
    from speculative_decoding_block_spec_b200.dist import max_over_ranks as _max_over_ranks

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    stream = torch.cuda.Stream(dev)
    peak, peak_src = measured_peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(ms):
        """The slowest rank's time (the value itself on one GPU)."""
        return _max_over_ranks(ms, dev)

    def timed_total(fn, n=None):
        """W untimed calls, then K (or n) calls between one pair of events: ms per call (max over ranks)."""
        n = args.steps if n is None else n
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                fn(i)
            barrier()
            k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            k0.record(stream)
            for i in range(n):
                fn(i)
            k1.record(stream)
            k1.synchronize()
            barrier()
        return max_over_ranks(k0.elapsed_time(k1)) / n

    def timed_each(fn):
        """W untimed calls, then K calls with one event pair each: their spread
        (each statistic the max over ranks)."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                fn(i)
            barrier()
            for i in range(args.steps):
                ev[i][0].record(stream)
                fn(i)
                ev[i][1].record(stream)
            stream.synchronize()
            barrier()
        s = spread([a.elapsed_time(b) for a, b in ev])
        for k in ("median_ms", "p10_ms", "p90_ms", "min_ms", "max_ms"):
            s[k] = max_over_ranks(s[k])
        return s

    def measure(cid, headline, top_p=1.0):
        w = synth.WORKLOADS[cid]
        x = synth.make_inputs(w, seed=rank)  # weak scaling: every rank verifies its own batch
        r = Runner(w, x, dev, stream, args.sets, top_p)
        if top_p < 1:  # the filtered step alone: statistics with bonus rows, nuclei, accept / sample
            graphs = r.capture("step", r.step)
            ns = len(r.sets)
            res = {"w": w, "x": None, "top_p": top_p}
            res["ms_step"] = timed_total(lambda i: graphs[i % ns].replay())
            res["graph_replay"] = timed_each(lambda i: graphs[i % ns].replay())
            acc = r.sets[0]["out"][0].cpu().numpy()
            res["flagged_requests"] = int((acc < 0).sum())
            vl_np = np.full(w.B, w.L)
            res["step_bytes"] = step_bytes(w, vl_np, acc) + w.B * w.V * (2 if w.dtype == "bf16" else 4)
            r.release()
            torch.cuda.empty_cache()
            return res
        ns = len(r.sets)
        if w.budget is not None:
            r.capture("pack", r.prepack)
        graphs = r.capture("step", r.step)
        res = {"w": w, "x": x}
        # the statistics kernel alone, as a burst, before the long loops below warm the GPU up to its power cap
        # (against the burst copy peak); the same graph is timed again for K replays after them
        tg = r.capture_all("stats", r.stats_only)  # ns launches per replay: no graph-launch gap between them
        time.sleep(STATS_BURST_PAUSE_S)  # an idle moment first, as the burst copy peak was taken on an idle GPU
        res["ms_stats"] = timed_total(lambda i: tg.replay(), STATS_BURST_REPLAYS) / ns
        sampler = ClockSampler(local) if headline else None
        wall = {}
        with torch.cuda.stream(stream):
            t_w = time.time()
            for i in range(args.warmup):
                graphs[i % ns].replay()
            barrier()
            wall["warmup_s"] = time.time() - t_w
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            r0 = time.time()
            e0.record(stream)
            for i in range(args.steps):
                graphs[i % ns].replay()
            e1.record(stream)
            e1.synchronize()
            r1 = time.time()
            wall["timed_s"] = r1 - r0
            barrier()
        if sampler is not None:
            sampler.region = (r0, r1)
            sampler.stop()
            res["clocks"] = sampler.report()
        res["wall"] = wall
        ms_step = max_over_ranks(e0.elapsed_time(e1)) / args.steps
        res["ms_step"] = ms_step

        # the outputs of the last replay of set 0 give the bytes actually needed
        d0 = r.sets[0]
        acc = d0["out"][0].cpu().numpy()
        outt = d0["out"][1].cpu().numpy()
        vl_np = d0["dvl_out"][0].cpu().numpy() if w.budget is not None else np.full(w.B, w.L)
        res["gpu_out"] = (acc, outt)
        res["step_bytes"] = step_bytes(w, vl_np, acc)

        # replay by replay: the captured step, and the same step as plain launches
        res["graph_replay"] = timed_each(lambda i: graphs[i % ns].replay())
        res["plain_launch"] = timed_each(lambda i: r.step(r.sets[i % ns]))

        # the verify call alone, and the statistics kernel alone (the roofline's kernel)
        vg = r.capture("verify", r.verify_only)
        res["ms_verify"] = timed_total(lambda i: vg[i % ns].replay())
        # the statistics graph again, K replays in a row after the step loops: the clocks the power cap
        # settles at (reported beside it)
        ssamp = ClockSampler(local) if headline else None
        s0 = time.time()
        res["ms_stats_sustained"] = timed_total(lambda i: tg.replay()) / ns
        s1 = time.time()
        if ssamp is not None:
            ssamp.region = (s0, s1)
            ssamp.stop()
            res["stats_clocks"] = ssamp.report()
        res["window_bytes"] = window_bytes(w, vl_np)
        res["stats_kernel"] = stats_kernel_name(w, sms)
        res["ms_pack"] = None
        if w.budget is not None:  # allocation + pack copy, timed apart from the step
            pg = r.graphs["pack"]
            res["ms_pack"] = timed_total(lambda i: pg[i % ns].replay())

        if headline and not args.no_e2e:
            res["e2e"] = e2e_leg(r)
        if not headline:
            res["x"] = None  # only the headline's inputs feed the CPU baseline
        r.release()
        torch.cuda.empty_cache()
        return res

    def e2e_leg(r):
        """End to end: pinned host inputs -> device -> verify through the public
        API -> results to host, every step inside the timed region."""
        w, x = r.w, r.x
        # with a DVL budget the target arrives as the packed rows the model produced
        tgt = ("packed", r.sets[0]["packed"].cpu().pin_memory()) if w.budget is not None else \
            ("target", torch.from_numpy(np.ascontiguousarray(x.target).view(
                np.int16 if x.target.dtype == np.uint16 else np.float32)).pin_memory())
        host = dict([tgt],
                    draft=torch.from_numpy(np.ascontiguousarray(x.draft).view(
                        np.int16 if x.draft.dtype == np.uint16 else np.float32)).pin_memory(),
                    tokens=torch.from_numpy(x.tokens).pin_memory(), u=torch.from_numpy(x.u).pin_memory(),
                    g=torch.from_numpy(x.g).pin_memory())
        if x.mix_w is not None:
            host["mix_w"] = torch.from_numpy(x.mix_w).pin_memory()
        if x.scores is not None:
            host["scores"] = torch.from_numpy(x.scores).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        res_acc = torch.empty(w.B, dtype=torch.int32).pin_memory()
        res_out = torch.empty((w.B, w.L + 1), dtype=torch.int32).pin_memory()
        d2h = res_acc.numel() * 4 + res_out.numel() * 4
        n_e2e = min(args.steps, 20)
        ns = len(r.sets)

        def e2e_step(d):
            for k, t in host.items():
                dst = d[k]
                (dst.view(t.dtype) if dst.dtype != t.dtype else dst).copy_(t, non_blocking=True)
            a, o = r.step(d)
            res_acc.copy_(a, non_blocking=True)
            res_out.copy_(o, non_blocking=True)

        with torch.cuda.stream(stream):
            for i in range(3):
                e2e_step(r.sets[i % ns])
            barrier()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for i in range(n_e2e):
                e2e_step(r.sets[i % ns])
            t1.record(stream)
            t1.synchronize()
            barrier()
        ms_e2e = max_over_ranks(t0.elapsed_time(t1)) / n_e2e
        return {"value": world * w.B / (ms_e2e * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n_e2e,
                "note": "pinned host inputs copied to HBM, verify through the public API, results read back"}

    def summary(res):
        w = res["w"]
        achieved = res["window_bytes"] / (res["ms_stats"] * 1e-3) / 1e9
        sustained = res["window_bytes"] / (res["ms_stats_sustained"] * 1e-3) / 1e9
        gbs = res["step_bytes"] / (res["ms_step"] * 1e-3) / 1e9
        traffic, traffic_src = committed_traffic(res["stats_kernel"], w.name)
        return {
            "value": world * w.B / (res["ms_step"] * 1e-3), "ms_per_step": res["ms_step"],
            "hbm_gbs": gbs, "hbm_frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS, "hbm_frac_of_measured_copy": gbs / peak,
            "algorithmic_bytes_per_step": res["step_bytes"],
            "roofline": {"bound": "hbm", "kernel": res["stats_kernel"], "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic, "traffic_source": traffic_src,
                         "algorithmic_bytes_per_launch": res["window_bytes"], "launch_ms": res["ms_stats"],
                         "peak_source": peak_src, "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                         "timed": "spec_verify_window_stats alone: one CUDA graph of %d launches (one per input "
                                  "set, back to back), %d replays after the warm-up (a burst, before the step's timed "
                                  "loops); time per launch"
                                  % (args.sets, STATS_BURST_REPLAYS),
                         "sustained": {"launch_ms": res["ms_stats_sustained"], "achieved": sustained,
                                       "frac": sustained / peak, "replays": args.steps,
                                       "clocks": res.get("stats_clocks"),
                                       "note": "the same graph for K replays in a row"}},
            "verify_ms": res["ms_verify"], "dvl_allocate_pack_ms": res["ms_pack"],
            "per_replay": {"graph_replay": res["graph_replay"], "plain_launch": res["plain_launch"],
                           "launch_gap_saving_us": (res["plain_launch"]["median_ms"] -
                                                    res["graph_replay"]["median_ms"]) * 1e3,
                           "note": "one event pair per step; plain = the same step as stream launches "
                                   "through the Python binding"},
        }

    head = measure(args.workload, headline=True)
    extras = [measure(c, headline=False) for c in args.extra_ids]
    filtered = [measure(c, headline=False, top_p=args.top_p) for c in args.top_p_ids]

    cpu = margins = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, margins = cpu_baseline(head["x"], args.cpu_seconds, head["gpu_out"])

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    w = head["w"]
    s = summary(head)
    line = {
        "metric": METRIC, "value": s["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": s["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded per rank; Qwen3-size vocabulary, block 16)",
        "config": config_of(w, args.sets, world),
        "launch": "CUDA graph replay, %d launches per step" % ((2 if w.L > 0 else 1) + (w.budget is not None)),
    }
    line.update({k: v for k, v in s.items() if k not in ("value", "ms_per_step")})
    line.update({
        "low_margin_decisions": margins, "cpu_baseline": cpu, "e2e": head.get("e2e"),
        "gpu_launches": ((2 if w.L > 0 else 1) + (w.budget is not None)) * args.steps,
        "clocks": head["clocks"], "host_wall_s": head["wall"],
        "workloads": {e["w"].name: dict(summary(e), config=config_of(e["w"], args.sets, world)) for e in extras},
        "top_p_workloads": {"%s top_p %g" % (f["w"].name, f["top_p"]): {
            "value": world * f["w"].B / (f["ms_step"] * 1e-3), "unit": UNIT, "ms_per_step": f["ms_step"],
            "top_p": f["top_p"], "graph_replay": f["graph_replay"], "flagged_requests": f["flagged_requests"],
            "algorithmic_bytes_per_step": f["step_bytes"],
            "hbm_gbs_algorithmic": f["step_bytes"] / (f["ms_step"] * 1e-3) / 1e9,
            "note": "spec_verify_*_top_p (statistics with bonus rows, nucleus kernel, accept / sample); "
                    "drafted tokens from the seeded generator, i.e. from the unfiltered draft rows; algorithmic "
                    "bytes count each filtered row once, as the unfiltered step does, plus the bonus rows"}
            for f in filtered},
    })
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
