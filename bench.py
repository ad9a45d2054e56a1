"""Benchmark of the canvas denoise-sampling stage on B200.

Workload (the single-step microbenchmark): one 256-position canvas, vocabulary
V = 262144, hidden d = 2816, tied bf16 head/embedding W = E ~ N(0, 0.02), hidden
states N(0, 1) / sqrt(d) * 8, step 1 (T = 0.8), entropy bound 0.1.  A timed step
is one dg_denoise_step: the fused logits / softmax / entropy / argmax /
self-conditioning kernel, the split-vocabulary combine, accept / re-noise and the
stop reduction.  Inputs are larger than L2 (W streams 1.48 GB per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  With --gpus N > 1 (under torchrun) every rank
runs an independent replica (canvases shard across GPUs with no data-path
collective); the value is all ranks' positions over the slowest rank's time.
With --split vocab the ranks instead share one canvas and split the head by
vocabulary rows (an all-gather of the shards' partials each step).
"""

import argparse
import hashlib
import json
import math
import re
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

V, D, N_POS, STEP, BOUND = 262144, 2816, 256, 1, 0.1
ACCEPT_MODE = 0            # 0: accepted positions keep the argmax; 1: a Gumbel-max sample (--accept sample)
ACCEPT_RULE = 0            # 0: accept every position with H <= bound; 1: by groups (--rule group)
CANVASES, UNTIED = 1, False  # per rank; other values are context measurements (--canvases, --untied)
LOGITS_FP8 = False         # --logits e4m3: the head as E4M3 codes for the logits GEMM (its own bench line)
METRIC = "canvas positions/s per denoise step (V=262144,d=2816); % of roofline"
WORKLOAD = ("single-step microbenchmark: 1 canvas of 256 positions, V=262144, d=2816, tied bf16 E=W ~N(0,0.02), "
            "hidden bf16 N(0,1)/sqrt(d)*8, step 1 (T=0.8), bound 0.1; outputs tokens/H/argmax/accept/self-cond fp32")
FLOPS_PER_STEP = 2 * (2.0 * N_POS * V * D)          # two contractions: logits and self-conditioning
WE_BYTES_PER_STEP = 2.0 * V * D                     # tied bf16 W = E streamed once
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "dg_fused_kernel_single_step_v262144_d2816.md")
PROFILE_SUMMARY_FP8 = os.path.join(ROOT, "profiles", "dg_fused_fp8_kernel_single_step_v262144_d2816.md")
CSRC = os.path.join(ROOT, "discrete_diffusion_decoding_b200", "csrc")


def _code_only(text):
    """C/C++ source without comments and with whitespace collapsed (comment edits do not change code)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash():
    """sha256 over the code (comments stripped) of every CUDA source and header of the library, in name order."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            h.update(name.encode())
            with open(os.path.join(CSRC, name), encoding="utf-8") as f:
                h.update(_code_only(f.read()).encode())
    return h.hexdigest()


def _set_vocab(vocab):
    """Reduced-vocabulary variant of the workload (profiler captures only)."""
    global V, FLOPS_PER_STEP, WE_BYTES_PER_STEP, WORKLOAD
    V = int(vocab)
    FLOPS_PER_STEP = 2 * (2.0 * N_POS * V * D)
    WE_BYTES_PER_STEP = 2.0 * V * D
    WORKLOAD = WORKLOAD.replace("V=262144", f"V={V} (reduced, profiling only)")


# ----------------------------------------------------------------------------- helpers
def dist_env():
    """(rank, world_size, local_rank) from the torchrun environment (1-process defaults)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_canvases(n_canvas_total, rank, world):
    """Contiguous canvas range of one rank (replicas: every rank gets its own canvases)."""
    lo = (n_canvas_total * rank) // world
    hi = (n_canvas_total * (rank + 1)) // world
    return lo, hi


def max_over_ranks(value, backend_device=None):
    """Maximum of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=backend_device or "cpu")
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(path=None):
    """DRAM bytes per fused launch from the committed ncu summary, if it was taken on this kernel source."""
    try:
        text = open(path or PROFILE_SUMMARY).read()
        src_hash = kernel_source_hash()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_source_sha256") != src_hash:
        return None
    try:
        return float(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled through NVML every 2 ms on a
    background thread; summary() keeps the samples whose timestamps fall inside the timed region
    (the sampler is started before the warm-up so that its start-up does not eat into the region).
    A 20-step region of ~13 ms still gets several samples."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device_index, period_s=0.002):
        self.dev, self.period, self.rows, self.err = device_index, period_s, [], None
        self._stop = None
        self._thread = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.dev)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def __enter__(self):
        import threading
        try:
            nv, h = self._handle()
        except Exception as e:           # no NVML: the line says so
            self.err = f"nvml unavailable: {e}"
            return self
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        self._stop = threading.Event()

        def read():
            self.rows.append((time.time(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                              nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(get_reasons(h))))
        self._read = read

        def loop():
            while not self._stop.is_set():
                try:
                    read()
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(self.period)
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def sample_now(self, n=3, gap_s=0.002):
        """A few samples from the calling thread (while the GPU works through an enqueued region,
        so that a short region is sampled even when the background thread does not get to run)."""
        read = getattr(self, "_read", None)
        if read is None:
            return
        for _ in range(n):
            try:
                read()
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(gap_s)

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self, t0=None, t1=None):
        """Median SM clock, max clock, median power and the reasons active in any sample of [t0, t1]."""
        if self.err and not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err], "samples": 0}
        rows = [r for r in self.rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        reasons = sorted({name for _, _, _, bits in rows for name, bit in self.REASONS if bits & bit})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": self.max_mhz,
                "power_w": round(statistics.median(r[2] for r in rows), 1), "reasons": reasons,
                "samples": len(rows), "source": "nvml, 2 ms"}


def choose_peak(peaks, region_s, clocks):
    """The bf16 peak that matches the regime the fused kernel was timed in: the sustained figure
    (a seconds-long GEMM loop under the power cap) when the timed region lasted at least a second
    and the power cap was active in it; the burst figure otherwise.  Returns (peak, name)."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    if region_s >= 1.0 and capped:
        return sustained, "sustained"
    return burst, "burst"


# ----------------------------------------------------------------------------- CPU oracle leg
def _set_shape(canvases, untied):
    """--canvases C / --untied: context measurements of the batched and untied workloads (not bench lines)."""
    global CANVASES, UNTIED, N_POS, FLOPS_PER_STEP, WE_BYTES_PER_STEP, WORKLOAD
    CANVASES, UNTIED = int(canvases), bool(untied)
    N_POS = 256 * CANVASES
    FLOPS_PER_STEP = 2 * (2.0 * N_POS * V * D)
    WE_BYTES_PER_STEP = (2.0 if UNTIED else 1.0) * 2.0 * V * D
    if CANVASES != 1:
        WORKLOAD = WORKLOAD.replace("1 canvas of 256 positions", f"{CANVASES} canvases of 256 positions in one launch "
                                    "(context measurement)")
    if UNTIED:
        WORKLOAD = WORKLOAD.replace("tied bf16 E=W ~N(0,0.02)", "untied bf16 W, E ~N(0,0.02) (context measurement)")


def _set_logits(fp8):
    """--logits e4m3: E4M3 logits operands, bf16 self-conditioning (the low-precision head option)."""
    global LOGITS_FP8, WORKLOAD
    LOGITS_FP8 = bool(fp8)
    if LOGITS_FP8:
        WORKLOAD = WORKLOAD.replace("tied bf16 E=W ~N(0,0.02)", "head ~N(0,0.02) as E4M3 codes with one power-of-two "
                                    "scale for the logits GEMM, its exact bf16 decoding as E")


def _set_accept(mode, rule=0):
    """--accept sample / --rule group: time the sampled-acceptance kernel or the group rule."""
    global ACCEPT_MODE, ACCEPT_RULE, WORKLOAD
    ACCEPT_MODE, ACCEPT_RULE = mode, rule
    if mode == 1:
        WORKLOAD = WORKLOAD.replace("bound 0.1", "bound 0.1, accepted tokens drawn by Gumbel-max sampling")
    if rule == 1:
        WORKLOAD = WORKLOAD.replace("bound 0.1", "bound 0.1 on the cumulative entropy of each canvas's accepted group")


def oracle_sample_rate(W64, h_bits, n_rows, T):
    """Time the float64 oracle on n_rows positions of the workload; returns (positions/s, seconds, threads).

    W64 is the head widened to float64 once, outside the timed call.
    """
    from oracle import stage
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    r = stage.step_rows(h_bits[:n_rows], W64, W64, T, BOUND, 0, STEP, 0, list(range(n_rows)), V,
                        accept_mode=ACCEPT_MODE)
    if ACCEPT_RULE == 1:
        # the group rule needs every position of the canvas; a partial sample ranks what it has
        kept = r["sample"] if ACCEPT_MODE == 1 else r["argmax"]
        stage.group_accept(r["H"], kept, BOUND, r["tokens"])
    dt = time.perf_counter() - t0
    return n_rows / dt, dt, threads


def run_reference(args):
    """--impl reference: the float64 CPU oracle as it stands, timed on the host cores.

    Every timed step is a whole 256-position step when K of them fit in about two minutes
    (the driver's short runs); otherwise each step is a bounded sample of positions and the
    line says so (ms_per_step is then scaled to a whole step and marked as such).
    """
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import synth
    from oracle import stage
    W = synth.weights(V, D, seed=1234)
    h = synth.gaussian_hidden(N_POS, D, seed=42)
    W64, hb = stage.bf16_to_f64(synth.bf16_bits(W)), synth.bf16_bits(h)
    del W
    if LOGITS_FP8:
        # the E4M3 workload: the oracle decodes the quantised head and hidden states exactly
        from oracle import fp8
        codes, e = fp8.quantize_tensor(W64)
        W64 = fp8.dequantize_tensor(codes, e)
        del codes
        hq, eh = fp8.quantize_rows(stage.bf16_to_f64(hb))
        hb = stage.f64_to_bf16(fp8.dequantize_rows(hq, eh))
    T = stage.temperature(STEP, 48)
    _, probe_dt, _ = oracle_sample_rate(W64, hb, 8, T)
    full_est = probe_dt * N_POS / 8
    n_rows = N_POS if args.steps * full_est <= 120.0 else int(max(1, min(N_POS, 120.0 / args.steps / probe_dt * 8)))
    for _ in range(args.warmup):
        oracle_sample_rate(W64, hb, 1, T)          # untimed warm-up: one position per step
    times, threads = [], 1
    for _ in range(args.steps):
        _, dt, threads = oracle_sample_rate(W64, hb, n_rows, T)
        times.append(dt)
    measured_ms = statistics.mean(times) * 1e3
    ms = measured_ms * (N_POS / n_rows)
    value = N_POS / (ms * 1e-3)
    whole = n_rows == N_POS
    sample = ("every timed step is a whole 256-position step" if whole else
              f"{n_rows} of 256 positions per timed step ({measured_ms:.0f} ms), scaled to a whole step")
    line = {"metric": METRIC, "value": value, "unit": "positions/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms,
            "ms_per_step_kind": "measured whole steps" if whole else f"scaled from {n_rows} of 256 positions",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "n_canvas": 1, "positions": N_POS, "vocab": V, "hidden": D},
            "cpu_baseline": {"value": value, "unit": "positions/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "positions/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_cpu_configs(args):
    """--cpu-configs: the float64 oracle on the host cores for the other workloads (context lines,
    one per workload): the small decode timed in full (all 16 steps of its schedule, its stub
    included), and one step of the block decode, the 16-canvas batch and the 4-canvas untied
    adversarial batch at their sizes, multiplied by the steps of a 48-step schedule and marked
    "extrapolated"."""
    import numpy as np
    import synth
    from oracle import decode, stage
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count() or 1

    def emit(workload, positions, seconds, kind, extra):
        rate = positions / seconds
        print(json.dumps({"metric": METRIC, "impl": "reference", "kind": "context (not a bench line)",
                          "config": {"workload": workload},
                          "cpu_baseline": {"value": rate, "unit": "positions/s", "cores": threads,
                                           "kind": "oracle", "sample": kind, **extra}}), flush=True)

    # small decode: V=4096, d=128, 1 canvas, literal stub, 16 steps, timed in full
    Ws = synth.bf16_bits(synth.weights(4096, 128))
    seeds = synth.canvas_seeds(1)
    t0 = time.perf_counter()
    r = decode.decode_batch(Ws, Ws, seeds, decode.stub_hidden_fn(Ws, seeds, 16, 1.0, 0.1), 4096, max_steps=16)
    dt = time.perf_counter() - t0
    emit("small decode: 1 canvas, V=4096, d=128, stub gain 1, 16-step schedule", 256 * int(r["stop_step"][0]), dt,
         f"timed in full: {int(r['stop_step'][0])} steps in {dt:.2f} s", {"steps": int(r["stop_step"][0])})
    # full-size workloads: one step each, extrapolated to the 48-step schedule
    W = synth.weights(V, D, seed=1234)
    W64 = stage.bf16_to_f64(synth.bf16_bits(W))
    T = stage.temperature(1, 48)
    for name, C, untied in (("block decode: 8 canvases of 256 one after another", 1, False),
                            ("16 canvases in one launch (N=4096)", 16, False),
                            ("4 canvases (N=1024), untied W and E", 4, True)):
        E64 = stage.bf16_to_f64(synth.bf16_bits(synth.weights(V, D, seed=1235))) if untied else W64
        h = synth.bf16_bits(synth.gaussian_hidden(C * 256, D, seed=42))
        t0 = time.perf_counter()
        for c in range(C):
            stage.step_rows(h[c * 256:(c + 1) * 256], W64, E64, T, BOUND, c, 1, c, np.arange(256), V)
        dt = time.perf_counter() - t0
        total_steps = 48 * (8 if C == 1 else 1)
        emit(name + ", V=262144, d=2816, 48-step schedule", C * 256, dt,
             f"extrapolated: one step of {C * 256} positions took {dt:.1f} s; a 48-step decode of the "
             f"workload would take about {dt * total_steps / 60:.0f} min", {"one_step_s": dt})
        del E64
    return 0


# ----------------------------------------------------------------------------- GPU leg
def run_gpu(args):
    import torch
    import torch.distributed as tdist

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    import synth
    from discrete_diffusion_decoding_b200 import build
    build.build()
    import discrete_diffusion_decoding_b200 as dg
    from discrete_diffusion_decoding_b200 import vocab_parallel as vp

    split = args.split == "vocab" and world > 1
    # inputs first, each rank with its share of the host's cores, so that the ranks reach the
    # process group (and its short timeout) together
    if world > 1:
        torch.set_num_threads(max(1, (os.cpu_count() or 1) // world))
    W_host = synth.weights(V, D, seed=1234)
    if split:
        v0, v1 = vp.shard_bounds(V, world, rank)
        W = W_host[v0:v1].contiguous().to(dev)
        E = synth.weights(V, D, seed=1235)[v0:v1].contiguous().to(dev) if UNTIED else W
    else:
        v0, v1 = 0, V
        W = W_host.to(dev)
        E = synth.weights(V, D, seed=1235).to(dev) if UNTIED else W
    del W_host
    w_exp = 0
    if LOGITS_FP8:
        # one-time head preparation: E4M3 codes on the GPU, and their exact bf16 decoding as E
        W, w_exp = dg.quantize_head_e4m3(W)
        E = (W.view(torch.float8_e4m3fn).to(torch.float32) * (2.0 ** w_exp)).to(torch.bfloat16)
    head_layout = 0
    if not LOGITS_FP8:
        # one-time weight preparation, outside every timed region: the bf16 head (and a separate
        # embedding) re-ordered tile-major, so each operand box of the fused pass is one
        # contiguous block (bit-identical results; ~1 % faster, measured)
        W_t = dg.tile_head(W)
        E = W_t if E is W else dg.tile_head(E)
        W = W_t
        head_layout = 1
        torch.cuda.synchronize()
    h_host = synth.gaussian_hidden(N_POS, D, seed=42)
    if world > 1:
        tdist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))

    # replicas: every rank owns CANVASES canvases of its own (seed = the global canvas index);
    # vocabulary split: every rank works on the same canvases over its rows of the head
    c0 = 0 if split else shard_canvases(world * CANVASES, rank, world)[0]
    p = dg.params(CANVASES, V, D, accept_mode=ACCEPT_MODE, accept_rule=ACCEPT_RULE,
                  tied=0 if (UNTIED or LOGITS_FP8) else 1, logits_format=1 if LOGITS_FP8 else 0, w_scale_exp=w_exp,
                  head_layout=head_layout)
    bufs = dg.StepBuffers(p, dev)
    seeds = torch.arange(c0, c0 + CANVASES, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()
    if split:
        stepper = vp.SplitStep(p, W, E, v0, v1)
        ws = stepper.ws
        stepper.init(seeds, bufs.tokens)
    else:
        ws = dg.Workspace(p, dev)
        dg.dg_canvas_init(p, seeds, bufs.tokens, ws)
    bufs.h.copy_(h_host.to(dev))

    def step(h=None, sc=None):
        h = bufs.h if h is None else h
        if split:
            stepper(STEP, h, seeds, bufs, stream, selfcond=sc)
        else:
            dg.dg_denoise_step(p, STEP, h, W, E, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                               bufs.lse, bufs.selfcond if sc is None else sc, ws, stream)

    clk = ClockSampler(local).__enter__()          # started early: its start-up is not in the region
    try:
        for _ in range(args.warmup):
            step()
        _, _, _ = dg.dg_stop_check(p, ws)
        step()
        launches_per_step = 4 if split else dg.last_launch_count()   # split: partial (2) + merge (2)

        # ---- device-timed region: K steps, inputs resident, W (1.48 GB) larger than L2
        if world > 1:
            tdist.barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dg.profile_enable(args.steps)
        t_region0 = time.time()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        clk.sample_now()                 # the GPU is still working through the enqueued steps
        torch.cuda.synchronize()
        t_region1 = time.time()
    finally:
        clk.__exit__(None, None, None)
    clocks = clk.summary(t_region0, t_region1)
    # the clock the last timed fused pass issued its tensor-core work at, from its own cycle
    # counter over the global timer: under the power limit it sits below what NVML reports
    clocks["kernel_sm_mhz"] = round(dg.dg_last_sm_clock(p, ws), 1)
    n_k1, k1_ms, _ = dg.profile_collect()
    if world > 1:
        tdist.barrier()
    elapsed_ms = ev0.elapsed_time(ev1)
    flags, _, _ = dg.dg_stop_check(p, ws)             # also surfaces an in-kernel timeout
    elapsed_max = max_over_ranks(elapsed_ms, dev if world > 1 else None)
    k1_max = max_over_ranks(k1_ms, dev if world > 1 else None)
    ms_per_step = elapsed_max / args.steps

    # ---- end to end through the public API: pinned host h in, results out, every step.
    # Pipelined as a caller would: h and the self-conditioning vectors are double-buffered
    # and move on a copy stream, so step i+1's upload and step i's download overlap the
    # neighbouring steps' compute; the small per-position results (which the next step
    # overwrites) are read back on the compute stream before it continues.
    h_pin = h_host.pin_memory()
    # entropy, tokens, argmax and accept flags in one pinned buffer (StepBuffers.packed)
    out_small = torch.empty(bufs.packed.numel(), dtype=torch.uint8).pin_memory()
    out_sc = [torch.empty((N_POS, D), dtype=torch.float32).pin_memory() for _ in range(2)]
    e2e_steps = args.steps            # as long as the device-timed loop: the same clock regime
    copy_stream = torch.cuda.Stream(device=dev)
    h_dev = [bufs.h, torch.empty_like(bufs.h)]
    sc_dev = [bufs.selfcond, torch.empty_like(bufs.selfcond)]

    def e2e_run(n):
        """n pipelined steps; returns with both streams' work enqueued (the compute stream waits for all)."""
        h_ready = [torch.cuda.Event(), torch.cuda.Event()]
        done = [torch.cuda.Event(), torch.cuda.Event()]
        copy_stream.wait_stream(stream)
        with torch.cuda.stream(copy_stream):
            h_dev[0].copy_(h_pin, non_blocking=True)
        h_ready[0].record(copy_stream)
        for i in range(n):
            b = i % 2
            stream.wait_event(h_ready[b])
            step(h_dev[b], sc_dev[b])
            with torch.cuda.stream(stream):
                out_small.copy_(bufs.packed, non_blocking=True)      # one copy for the per-position results
            done[b].record(stream)
            with torch.cuda.stream(copy_stream):
                if i + 1 < n:
                    if i >= 1:
                        copy_stream.wait_event(done[1 - b])        # step i-1 no longer reads h_dev[1-b]
                    h_dev[1 - b].copy_(h_pin, non_blocking=True)
                    h_ready[1 - b].record(copy_stream)
                copy_stream.wait_event(done[b])
                out_sc[b].copy_(sc_dev[b], non_blocking=True)
        stream.wait_stream(copy_stream)

    e2e_run(3)
    if world > 1:
        tdist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev if world > 1 else None) / e2e_steps
    h2d = h_pin.numel() * h_pin.element_size()
    d2h = sum(t.numel() * t.element_size() for t in (out_small, out_sc[0]))

    line = None
    if rank == 0:
        peaks, peaks_src = load_peaks()
        peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        region_s = elapsed_max * 1e-3
        peak_tf, regime = choose_peak(peaks, region_s, clocks)
        rows_per_rank = v1 - v0
        flops_launch = 2 * (2.0 * N_POS * rows_per_rank * D)
        achieved = flops_launch / (k1_max * 1e-3) / 1e12
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])) * 1e9
        bytes_launch = (2.0 if UNTIED else 1.0) * 2.0 * rows_per_rank * D
        if LOGITS_FP8:
            # half the FLOPs at the E4M3 rate (twice bf16, the nominal ratio), half at the bf16 rate:
            # the launch's peak is 4 / (1/2 + 1) / 2 = 4/3 of the bf16 figure; bytes: 1-byte codes + bf16 E
            fp8_gain = 4.0 / 3.0
            peak_tf, peak_burst, peak_sus = peak_tf * fp8_gain, peak_burst * fp8_gain, peak_sus * fp8_gain
            bytes_launch = 3.0 * rows_per_rank * D
        roof_ms = max(flops_launch / (peak_tf * 1e12), bytes_launch / hbm) * 1e3
        # the committed DRAM capture is of the default kernel on the one-canvas tied workload
        traffic = (profiled_traffic(PROFILE_SUMMARY_FP8 if LOGITS_FP8 else PROFILE_SUMMARY)
                   if (ACCEPT_MODE == 0 and CANVASES == 1 and not UNTIED and not split) else None)
        positions = (1 if split else world) * N_POS
        value = positions / (ms_per_step * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": "positions/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if split else "weak",
            "vs_baseline": None, "dtype": "e4m3 logits + bf16 self-conditioning" if LOGITS_FP8 else "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "n_canvas": (1 if split else world) * CANVASES, "positions": positions,
                       "vocab": V, "hidden": D,
                       "parallelism": (f"vocabulary split x{world} (all-gather of shard partials)" if split else
                                       f"replicas x{world}" if world > 1 else "single GPU"),
                       "l2": "inputs larger than L2 (W/E 1.48 GB streamed per step)",
                       "head_layout": "tile-major" if head_layout else "row-major",
                       "group": dg.plan(p)["group"], "n_groups": dg.plan(p)["n_groups"]},
            "steps_per_s": 1e3 / ms_per_step,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": achieved / peak_tf, "traffic": traffic,
                         "kernel": ("dg_fused_fp8" if LOGITS_FP8 else "dg_fused") + ("_sample_kernel" if ACCEPT_MODE
                                                                                       else "_kernel"),
                         "kernel_ms": k1_max, "launches_timed": n_k1, "flops_per_launch": flops_launch,
                         "peak_regime": regime,
                         "peak_source": (f"{peaks_src} bf16 {regime}: " +
                                         ("a seconds-long GEMM loop under the power cap; the timed region lasted "
                                          f"{region_s:.2f} s with sw_power_cap active" if regime == "sustained" else
                                          f"a short GEMM burst; the timed region lasted {region_s:.3f} s")),
                         "frac_of_burst": achieved / peak_burst, "frac_of_sustained": achieved / peak_sus,
                         "burst_peak": peak_burst, "sustained_peak": peak_sus,
                         "step_frac": roof_ms / ms_per_step, "roofline_step_ms": roof_ms},
            "e2e": {"value": positions / (e2e_ms * 1e-3), "unit": "positions/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "stop_flags_after": flags,
        }
        if split:
            line["multi_gpu_note"] = "vocabulary split: NCCL all-gather of each rank's partial, merge on every rank"
        if LOGITS_FP8:
            line["roofline"]["peak_source"] += (" x 4/3: the logits GEMM runs on E4M3 operands at twice the bf16 "
                                                "rate (nominal ratio), the self-conditioning GEMM at the bf16 rate")
        if world == 1 and not args.no_cpu_baseline and CANVASES == 1 and not UNTIED and not LOGITS_FP8:
            # bounded sample of the same workload through the float64 oracle on the host cores
            from oracle import stage
            W64 = stage.bf16_to_f64(synth.bf16_bits(W.cpu()))
            hb = synth.bf16_bits(h_host)
            rate, dt, threads = oracle_sample_rate(W64, hb, args.cpu_rows, stage.temperature(STEP, 48))
            del W64
            line["cpu_baseline"] = {"value": rate, "unit": "positions/s", "cores": threads, "kind": "oracle",
                                    "sample": f"{args.cpu_rows} of 256 positions of one step ({dt:.1f} s)"}
    if world > 1:
        tdist.barrier()
        tdist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=256, help="positions in the oracle's bounded CPU sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-configs", action="store_true",
                    help="time the float64 oracle on the other workloads (context lines) and exit")
    ap.add_argument("--accept", choices=["argmax", "sample"], default="argmax",
                    help="token kept at accepted positions (sample: Gumbel-max draw from softmax(z/T))")
    ap.add_argument("--rule", choices=["position", "group"], default="position",
                    help="accepted positions: H <= bound each, or the canvas's entropy-ordered group within the bound")
    ap.add_argument("--canvases", type=int, default=1,
                    help="canvases per rank in one launch; values other than 1 are context measurements, not bench lines")
    ap.add_argument("--untied", action="store_true", help="separate W and E (context measurement, not a bench line)")
    ap.add_argument("--logits", choices=["bf16", "e4m3"], default="bf16",
                    help="number format of the logits GEMM operands (e4m3: the head as 8-bit codes; its own bench line)")
    ap.add_argument("--split", choices=["replicas", "vocab"], default="replicas",
                    help="with --gpus N > 1: independent replicas (weak scaling, default) or one head split by "
                         "vocabulary rows over the ranks (strong scaling)")
    ap.add_argument("--vocab", type=int, default=262144,
                    help="vocabulary size; smaller values are for profiler captures only, not bench lines")
    args = ap.parse_args(argv)
    if args.vocab != V:
        _set_vocab(args.vocab)
    _set_accept(1 if args.accept == "sample" else 0, 1 if args.rule == "group" else 0)
    _set_shape(args.canvases, args.untied)
    _set_logits(args.logits == "e4m3")
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.cpu_configs:
        return run_cpu_configs(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
