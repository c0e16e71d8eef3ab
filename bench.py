#!/usr/bin/env python
"""Benchmark of the chunkwise (TFLA) mLSTM forward + backward on B200.

One step = one mlstm_fwd plus one mlstm_bwd over one batch (every kernel of
the path) at B8 H32 T4096 d128, chunk 128, mLSTMexp, bf16 I/O.  Prints one
JSON line (rank 0).  Multi-GPU runs (torchrun) are independent replicas: each
rank processes its own batch, no collective touches the data path; the step
time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (heads are independent), on the host cores.
"""

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mLSTM chunkwise fwd/bwd TFLOP/s & tokens/s (B8 H32 d128 T4k-16k), % bf16 peak"
UNIT = "TFLOP/s"
WORKLOAD = "exp_b8h32_t4096_d128_c128"
# CUDA-core fp32 FMA peak: 148 SMs x 128 lanes x 2 flops x 1.965 GHz max SM clock
FP32_CORE_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
KERNEL_SOURCES = {
    "gate_prep": "gates.cu", "bwd_token_prep": "gates.cu", "gate_grad": "gates.cu",
    "state_fwd_simt": "simt_fwd.cu", "output_fwd_simt": "simt_fwd.cu",
    "state_bwd_simt": "simt_bwd.cu", "dq_simt": "simt_bwd.cu", "dk_simt": "simt_bwd.cu",
    "dv_simt": "simt_bwd.cu", "output_fwd_tc": "tc_fwd.cu", "dq_tc": "tc_bwd.cu",
    "dk_tc": "tc_bwd.cu", "dv_tc": "tc_bwd.cu", "state_fwd_tc": "tc_state.cu",
    "output_fwd_xl": "tc_fwd_xl.cu", "bwd_xl_table": "tc_bwd_xl.cu", "dq_xl": "tc_bwd_xl.cu",
    "dk_xl": "tc_bwd_xl.cu", "dv_xl": "tc_bwd_xl.cu", "state_fwd_fix": "tc_state.cu",
    "state_bwd_fix": "tc_state.cu", "gate_grad_sums": "gates.cu",
    "state_bwd_tc": "tc_state.cu", "dkv_walk_tc": "tc_bwd_walk.cu", "fwd_walk_tc": "tc_fwd_walk.cu",
}


# ---------------------------------------------------------------------------
# algorithmic FLOP and byte counts (per (b, h) head)
# ---------------------------------------------------------------------------

def flops_fwd(T, dqk, dhv, L):
    """States 2 T dqk dhv + inter term 2 T dqk dhv + causal intra T L (dqk + dhv)."""
    return 4 * T * dqk * dhv + T * L * (dqk + dhv)


def flops_bwd(T, dqk, dhv, L):
    """Four T dqk dhv contractions x2 + causal intra dS K, dS^T Q, S, dP, A^T dH."""
    return 8 * T * dqk * dhv + T * L * (3 * dqk + 2 * dhv)


def kernel_costs(T, dqk, dhv, L, exp_variant, io_bytes):
    """(flops, bytes) per head for every kernel of the path, algorithmic counts.

    Bytes count each tensor once per kernel that must touch it: inputs read,
    outputs written, chunk states (two bf16 planes = 4 B per element on the
    bf16 path, the tensor-core forward reads only the hi plane) and the fp32
    per-token gate arrays.
    """
    NC = -(-T // L)
    g = 3 if exp_variant else 2  # per-token gate floats (b, log i [, m])
    st_full = NC * dqk * dhv * 4            # hi + lo planes (or one fp32 plane)
    st_hi = NC * dqk * dhv * io_bytes       # hi plane only
    stn = NC * dqk * 4 if exp_variant else 0
    tdd = 2 * T * dqk * dhv
    tok_f = T * 4
    c = {
        "gate_prep": (0, T * 2 * io_bytes + g * tok_f),
        "state_fwd": (tdd, T * (dqk + dhv) * io_bytes + g * tok_f + st_full + stn),
        "output_fwd": (tdd + T * L * (dqk + dhv),
                       T * (2 * dqk + 2 * dhv) * io_bytes + g * tok_f + st_hi + stn
                       + (tok_f if exp_variant else 0)),
        "bwd_token_prep": (0, (T * 2 * dhv * io_bytes + 2 * tok_f + 4 * tok_f) if exp_variant
                           else 3 * tok_f),
        "state_bwd": (tdd, T * (dqk + dhv) * io_bytes + 4 * tok_f + st_full + stn),
        "dq": (tdd + T * L * (dhv + dqk), T * (3 * dqk + 2 * dhv) * io_bytes + 6 * tok_f + st_full + stn),
        "dk": (tdd + T * L * dqk, T * (3 * dqk + 2 * dhv) * io_bytes + 6 * tok_f + st_full + stn),
        "dv": (tdd + T * L * (dqk + dhv), T * (2 * dqk + 2 * dhv) * io_bytes + 4 * tok_f + st_full),
        "gate_grad": (0, T * 4 * io_bytes + 2 * tok_f),
        # the large-chunk backward's gate table: five per-token arrays in, seven out
        "bwd_xl_table": (0, 12 * tok_f),
        # completion of a segmented state walk: every state read and written once
        "state_fwd_fix": (0, 2 * st_full + (2 * stn if exp_variant else 0)),
        "state_bwd_fix": (0, 2 * st_full + (2 * stn if exp_variant else 0)),
        # segment totals of q.dq - k.dk (few heads): pq and pk read once
        "gate_grad_sums": (0, 2 * tok_f),
        # state gradients, dk and dv in one pass: the state-gradient recurrence and the
        # dk, dv contractions; q, k, v, dh read once, dk, dv and k.dk written, the state
        # gradients never leave the chip
        # the states and the outputs in one pass: q, k, v read once, h, the states (both
        # planes, the backward reads them) and the normaliser written
        "fwd_walk": (2 * tdd + T * L * (dqk + dhv),
                     T * (2 * dqk + 2 * dhv) * io_bytes + g * tok_f + st_full + stn
                     + (tok_f if exp_variant else 0)),
        "dkv_walk": (3 * tdd + T * L * (2 * dqk + dhv),
                     T * (3 * dqk + 3 * dhv) * io_bytes
                     + (g + (2 if exp_variant else 0) + 1) * tok_f),
    }
    out = {}
    for role, v in c.items():
        out[role] = v
        for impl in ("_simt", "_tc", "_xl"):
            out[role + impl] = v
    return out


def kernel_bound(name):
    """Which roofline bounds a kernel of this implementation."""
    if name.endswith("_simt"):
        return "alu"
    if name.endswith("_tc") or name.endswith("_xl"):
        return "tensor"
    return "hbm"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def source_sha(kernel):
    src = KERNEL_SOURCES.get(kernel)
    if src is None:
        return None
    path = os.path.join(ROOT, "mlstm_chunkwise_attention_b200", "csrc", src)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def reduce_max(v, world, device):
    """The largest of every rank's v (one all-reduce; v itself when world == 1)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def committed_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kernel)
    if not e or e.get("workload") != workload or e.get("source_sha") != source_sha(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons during the timed region.

    Read in-process through NVML every 5 ms by a background thread (a region of a few tens
    of milliseconds still gets several samples); nvidia-smi polling at 200 ms when NVML
    cannot be loaded.  Reading clocks changes nothing on the GPU."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h): the slowdowns that reject a number, and the cap
    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
                   ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, gpu_index, period_s=0.005):
        self.gpu_index = gpu_index
        self.period_s = period_s
        self.proc = None
        self.out = None
        self.thread = None
        self.rows = []

    def start(self):
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByIndex(self.gpu_index)
            max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
            self.stop_event = threading.Event()

            def loop():
                while True:
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                        bits = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle))
                    except Exception:  # noqa: BLE001
                        break
                    self.rows.append({"sm": sm, "max": max_mhz, "bits": bits})
                    if self.stop_event.wait(self.period_s):
                        break

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:  # noqa: BLE001
            self.thread = None
        try:
            self.out = open(os.path.join("/tmp", f"mlstm_clocks_{os.getpid()}.csv"), "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu_index)], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def _summary(self, rows, reasons):
        if not rows:
            return None
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows)}

    def stop(self):
        if self.thread is not None:
            self.stop_event.set()
            self.thread.join(timeout=5)
            try:  # release NVML before the per-kernel timing that follows
                import pynvml
                pynvml.nvmlShutdown()
            except Exception:  # noqa: BLE001
                pass
            reasons = {name for r in self.rows for name, bit in self.REASON_BITS if r["bits"] & bit}
            return self._summary(self.rows, reasons)
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append({"sm": float(parts[1]), "max": float(parts[2]), "active": parts[4],
                                 "hw": parts[5], "hwt": parts[6], "swt": parts[7], "pcap": parts[8]})
                except ValueError:
                    continue
        os.unlink(self.out.name)
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return self._summary(rows, reasons)


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------

def oracle_sample(spec, heads, budget_s=20.0, tokens=None):
    """Time the fp64 oracle (chunkwise forward + parallel-form backward) on whole heads, or on
    heads of `tokens` tokens (a multiple of the chunk) when given."""
    import numpy as np
    import oracle
    from mlstm_chunkwise_attention_b200.synthetic import make_inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        cores = 1
    T, dqk, dhv, L, var = spec["T"], spec["d_qk"], spec["d_hv"], spec["chunk"], spec["variant"]
    T_all = T
    if tokens is not None:
        T = tokens
    done, elapsed = [], 0.0
    for (b, hh) in heads:
        x = make_inputs(1, 1, T, dqk, dhv, seed=spec["seed"] * 1000 + b * 64 + hh,
                        igate_mean=spec["igate_mean"], fgate_mean=spec["fgate_mean"], with_dh=True)
        x = {k: v[0, 0].double().numpy() for k, v in x.items()}
        t0 = time.perf_counter()
        li, lf = oracle.gate_logs(x["igate"], x["fgate"], var)
        oracle.chunkwise_forward(x["q"], x["k"], x["v"], li, lf, var, L)
        g = oracle.parallel_backward(x["q"], x["k"], x["v"], li, lf, var, x["dh"])
        oracle.preact_grads(g["dlog_i"], g["dlog_f"], x["igate"], x["fgate"], var)
        elapsed += time.perf_counter() - t0
        done.append((b, hh))
        if elapsed >= budget_s:
            break
    flops = len(done) * (flops_fwd(T, dqk, dhv, L) + flops_bwd(T, dqk, dhv, L))
    return {"value": flops / elapsed / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "seconds": elapsed, "heads": len(done),
            "tokens": T,
            "sample": f"{len(done)} of {spec['B'] * spec['NH']} heads of the workload "
                      f"(T={T_all}, d={dqk}/{dhv}, chunk {L})"
                      + (f", each on {T} of its {T_all} tokens" if T != T_all else "")
                      + ": fp64 chunkwise forward + parallel-form backward in numpy; throughput "
                        "scaled by the algorithmic FLOPs of the tokens run"}


def run_reference(args, spec):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import math
    from mlstm_chunkwise_attention_b200.synthetic import sample_heads
    heads = sample_heads(spec["B"], spec["NH"], args.warmup + args.steps, 4242)
    T, dqk, dhv, L = spec["T"], spec["d_qk"], spec["d_hv"], spec["chunk"]
    # Each step is one head; when --steps --warmup heads of the whole sequence would take more
    # than about 150 s, each step runs a head on its first Ts tokens instead, Ts sized from one
    # untimed calibration head (the parallel-form backward grows as tokens squared).
    per_step = 150.0 / (args.warmup + args.steps)
    Tc = min(T, 8 * L)
    t_c = max(oracle_sample(spec, [heads[0]], budget_s=0.0, tokens=Tc)["seconds"], 1e-6)
    Ts = T if t_c * (T / Tc) ** 2 <= per_step else int(Tc * math.sqrt(per_step / t_c)) // L * L
    Ts = min(T, max(L, Ts))
    times = []
    info = None
    for i, hd in enumerate(heads):
        info = oracle_sample(spec, [hd], budget_s=0.0, tokens=Ts)
        if i >= args.warmup:
            times.append(info["seconds"])
    per_head = flops_fwd(Ts, dqk, dhv, L) + flops_bwd(Ts, dqk, dhv, L)
    total_s = sum(times)
    value = per_head * len(times) / total_s / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(spec, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": info["cores"], "kind": "oracle",
                         "sample": "each step: one head of the workload"
                                   + (f" on its first {Ts} of {T} tokens" if Ts != T else "")
                                   + ", fp64 chunkwise forward + parallel-form backward (numpy)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """Forward chunk-size / sequence-length sweep at B8 H32 d128 (one JSON line per point).

    Each point times mlstm_fwd with CUDA events over `--steps` calls (after
    `--warmup`), per kernel through the library's timing hook; reports
    forward TFLOP/s, tokens/s, and the output kernel's TFLOP/s as a share of
    the measured dense bf16 peak.
    """
    import torch
    from mlstm_chunkwise_attention_b200 import binding
    from mlstm_chunkwise_attention_b200.synthetic import SWEEP_CHUNK, SWEEP_SEED, SWEEP_T, make_inputs
    peaks = load_peaks()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    B, NH, d = args.sweep_batch, 32, 128
    Ts = [int(t) for t in args.sweep_t.split(",")] if args.sweep_t else list(SWEEP_T)
    Ls = [int(c) for c in args.sweep_chunk.split(",")] if args.sweep_chunk else list(SWEEP_CHUNK)
    cells = ((0, 0.0, "sig"), (1, 0.0, "exp"), (1, -10.0, "exp_igate_bias_m10"))
    if args.sweep_cells:
        keep = args.sweep_cells.split(",")
        cells = tuple(c for c in cells if c[2] in keep)
    for T in Ts:
        for (var, igm, label) in cells:
            cpu = make_inputs(B, NH, T, d, d, seed=SWEEP_SEED, igate_mean=igm, fgate_mean=3.0,
                              dtype=torch.bfloat16)
            x = {k: v.to(dev) for k, v in cpu.items()}
            del cpu
            h = torch.empty_like(x["v"])
            for L in Ls:
                sizes = binding.problem_sizes(x["q"], x["v"], L, var)
                saved = torch.empty(binding.mlstm_saved_size(*sizes), dtype=torch.uint8, device=dev)
                nf = binding.mlstm_fwd_launch_count(*sizes)
                names = [binding.mlstm_launch_name(0, i, *sizes) for i in range(nf)]
                evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nf)] for _ in range(args.steps)]
                for row in evs:
                    for e in row:
                        e.record(stream)
                torch.cuda.synchronize(dev)
                arrs = [(ctypes.c_void_p * (2 * nf))(*[e.cuda_event for e in row]) for row in evs]

                def call(ev=None):
                    if ev is not None:
                        binding.mlstm_set_timing_events(ev, 2 * nf)
                    st = binding.mlstm_fwd(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
                                           x["igate"].data_ptr(), x["fgate"].data_ptr(), h.data_ptr(),
                                           saved.data_ptr(), None, 0, *sizes, sh)
                    binding.mlstm_set_timing_events(None, 0)
                    if st != 0:
                        raise binding.MLSTMError(st, "mlstm_fwd")

                for _ in range(args.warmup):
                    call()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize(dev)
                e0.record(stream)
                for i in range(args.steps):
                    call(arrs[i])
                e1.record(stream)
                torch.cuda.synchronize(dev)
                binding.check_device()
                ms = e0.elapsed_time(e1) / args.steps
                kms = {n: sum(row[2 * i].elapsed_time(row[2 * i + 1]) for row in evs) / args.steps
                       for i, n in enumerate(names)}
                flops = B * NH * flops_fwd(T, d, d, L)
                # the output kernel, or the forward walker (states and outputs in one pass,
                # counted with the state products)
                out_name = [n for n in names if n.startswith(("output_fwd", "fwd_walk"))][0]
                role = "fwd_walk" if out_name.startswith("fwd_walk") else "output_fwd"
                out_fl = B * NH * kernel_costs(T, d, d, L, var == 1, 2)[role][0]
                line = {
                    "sweep": f"fwd_b{B}h32_d128", "cell": label, "T": T, "chunk": L,
                    "ms": ms, "tflops": flops / ms / 1e9, "tokens_per_s": B * T / ms * 1e3,
                    "kernel_ms": kms, "output_kernel": out_name,
                    "output_tflops": out_fl / kms[out_name] / 1e9,
                    "output_pct_bf16_peak": 100 * out_fl / kms[out_name] / 1e9 / peaks["bf16_tflops"],
                }
                if args.sweep_bwd:
                    line.update(sweep_bwd_point(args, binding, x, h, saved, sizes, sh, stream, dev,
                                                B, NH, T, d, L, var, peaks))
                print(json.dumps(line), flush=True)
                del saved
            del x, h
            torch.cuda.empty_cache()
    return 0


# RetNet chunk_fwd / chunk_fwdbwd times (ms) on one A100 80GB at B8, 32 heads,
# head dim 128 (flash-linear-attention README, RetNet vs FlashAttention-2
# timing table; units not printed, read as ms).  Context only: other hardware.
RETNET_A100_MS = {128: (0.185344, 1.591296), 256: (0.219136, 1.596928), 512: (0.397312, 1.603584),
                  1024: (0.747520, 3.089408), 2048: (1.403904, 6.059008), 4096: (2.755072, 11.938816),
                  8192: (5.491712, 23.952385), 16384: (10.870784, 48.745472)}


def run_retnet(args):
    """Retention (RetNet decays gamma_h = 1 - 2^(-5-h)) through the SIG kernels.

    B8 H32 d128 bf16 at the sequence lengths of the pages' A100 table; per T the
    forward and forward+backward are timed (CUDA events, mean of --steps after
    --warmup) at every chunk in 128..1024 not above T, and the fastest chunk of
    each pass is reported.  One JSON line per T.
    """
    import torch
    from mlstm_chunkwise_attention_b200 import binding
    from mlstm_chunkwise_attention_b200.synthetic import make_inputs, retention_gates, retnet_decays
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    B, NH, d = 8, 32, 128
    gamma = retnet_decays(NH)
    Ts = [int(t) for t in args.sweep_t.split(",")] if args.sweep_t else sorted(RETNET_A100_MS)
    for T in Ts:
        cpu = make_inputs(B, NH, T, d, d, seed=11, igate_mean=0.0, fgate_mean=3.0,
                          dtype=torch.bfloat16, with_dh=True)
        x = {k: v.to(dev) for k, v in cpu.items()}
        del cpu
        ig, fg = retention_gates(gamma, B, T, torch.bfloat16, dev)
        best = {}
        for L in [c for c in (128, 256, 512, 1024) if c <= max(T, 128)]:
            def fwd():
                return binding.forward(x["q"], x["k"], x["v"], ig, fg, L, binding.SIG,
                                       keep_saved=True)

            def fwdbwd():
                h, saved = fwd()
                binding.backward(x["q"], x["k"], x["v"], ig, fg, h, x["dh"], saved, L, binding.SIG)

            for name, fn in (("fwd", fwd), ("fwdbwd", fwdbwd)):
                for _ in range(args.warmup):
                    fn()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize(dev)
                e0.record(stream)
                for _ in range(args.steps):
                    fn()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                binding.check_device()
                ms = e0.elapsed_time(e1) / args.steps
                if name not in best or ms < best[name][0]:
                    best[name] = (ms, L)
        ref = RETNET_A100_MS.get(T)
        print(json.dumps({
            "retnet": "b8h32_d128_bf16", "T": T,
            "fwd_ms": best["fwd"][0], "fwd_chunk": best["fwd"][1],
            "fwd_tflops": B * NH * flops_fwd(T, d, d, best["fwd"][1]) / best["fwd"][0] / 1e9,
            "fwdbwd_ms": best["fwdbwd"][0], "fwdbwd_chunk": best["fwdbwd"][1],
            "tokens_per_s_fwdbwd": B * T / best["fwdbwd"][0] * 1e3,
            "a100_chunk_fwd_ms": ref[0] if ref else None,
            "a100_chunk_fwdbwd_ms": ref[1] if ref else None,
        }), flush=True)
        del x
        torch.cuda.empty_cache()
    return 0


def run_decode(args):
    """One-token steps (generation) at B8 H32 d128 bf16, both cells.

    Times --steps replays of a CUDA graph of 100 consecutive mlstm_step calls
    (state ping-pong, CUDA events), and reports tokens/s and the step kernel's
    HBM roofline: every step reads and writes the fp32 state (C, and n for
    EXP) once and touches q, k, v, h and the gates.  Also times the hand-off
    from a T = 4096 chunk-128 forward (mlstm_final_state).
    """
    import torch
    from mlstm_chunkwise_attention_b200 import binding
    from mlstm_chunkwise_attention_b200.synthetic import make_inputs
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    B, NH, d, T, L = 8, 32, 128, 4096, 128
    for var, label in ((0, "sig"), (1, "exp")):
        cpu = make_inputs(B, NH, T, d, d, seed=13, igate_mean=-2.0, fgate_mean=3.0,
                          dtype=torch.bfloat16, with_dh=False)
        x = {k: v.to(dev) for k, v in cpu.items()}
        _, saved = binding.forward(x["q"], x["k"], x["v"], x["igate"], x["fgate"], L, var)
        state = binding.final_state(x["k"], x["v"], saved, L, var)
        other = torch.empty_like(state)
        tok = {k: v[:, :, -1].contiguous() for k, v in x.items()}
        h = torch.empty((B, NH, d), dtype=torch.bfloat16, device=dev)

        def steps(n):
            nonlocal state, other
            for _ in range(n):
                binding.step(tok["q"], tok["k"], tok["v"], tok["igate"], tok["fgate"], state, other,
                             var, h=h)
                state, other = other, state

        steps(100 * args.warmup)
        torch.cuda.synchronize(dev)
        # 100 steps captured once in a CUDA graph (an even count: the state
        # buffers end where they started), so the device time is measured
        # without the host's per-call overhead
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            steps(100)
        for _ in range(args.warmup):
            graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        binding.check_device()
        ms = e0.elapsed_time(e1) / (100 * args.steps)
        del graph
        st_bytes = B * NH * (d * d * 4 + (d * 4 if var == 1 else 0))
        step_bytes = 2 * st_bytes + B * NH * (4 * d * 2 + 2 * 2) + (B * NH * 4 * 2 if var == 1 else 0)
        # hand-off from the prefill: mlstm_final_state
        for _ in range(args.warmup):
            binding.final_state(x["k"], x["v"], saved, L, var, state=other)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            binding.final_state(x["k"], x["v"], saved, L, var, state=other)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        achieved = step_bytes / ms / 1e6
        print(json.dumps({
            "decode": "b8h32_d128_bf16", "cell": label, "ms_per_step": ms,
            "tokens_per_s": B / ms * 1e3,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "bytes_per_step": step_bytes},
            "final_state_ms": f0.elapsed_time(f1) / args.steps,
        }), flush=True)
        del x, saved, state, other
        torch.cuda.empty_cache()
    return 0


def sweep_bwd_point(args, binding, x, h, saved, sizes, sh, stream, dev, B, NH, T, d, L, var, peaks):
    """Backward at one sweep point: mlstm_bwd timed like the forward, per kernel.

    Reports backward TFLOP/s (algorithmic count 8 T d^2 + T L 5 d per head) and
    the intra-chunk kernels' (dq, dk, dv; at chunk 128 with d 128 dq and the walker,
    whose count includes the state-gradient products) combined TFLOP/s against the
    dense bf16 peak.  Inputs: the point's forward outputs and an upstream dh ~ N(0,1).
    """
    import torch
    g = torch.Generator(device="cpu").manual_seed(7)
    dh = torch.randn(x["v"].shape, generator=g).to(device=dev, dtype=x["v"].dtype)
    dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
    dig, dfg = torch.empty_like(x["igate"]), torch.empty_like(x["fgate"])
    ws = torch.empty(binding.mlstm_bwd_workspace_size(*sizes), dtype=torch.uint8, device=dev)
    nb = binding.mlstm_bwd_launch_count(*sizes)
    names = [binding.mlstm_launch_name(1, i, *sizes) for i in range(nb)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nb)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize(dev)
    arrs = [(ctypes.c_void_p * (2 * nb))(*[e.cuda_event for e in row]) for row in evs]

    def call(ev=None):
        if ev is not None:
            binding.mlstm_set_timing_events(ev, 2 * nb)
        st = binding.mlstm_bwd(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
                               x["igate"].data_ptr(), x["fgate"].data_ptr(), h.data_ptr(),
                               dh.data_ptr(), saved.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), dig.data_ptr(), dfg.data_ptr(), ws.data_ptr(),
                               ws.numel(), *sizes, sh)
        binding.mlstm_set_timing_events(None, 0)
        if st != 0:
            raise binding.MLSTMError(st, "mlstm_bwd")

    for _ in range(args.warmup):
        call()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for i in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    # per-kernel times: the same calls with every kernel on the caller's stream, each alone
    binding.mlstm_set_serial_launches(True)
    for i in range(args.steps):
        call(arrs[i])
    binding.mlstm_set_serial_launches(False)
    torch.cuda.synchronize(dev)
    binding.check_device()
    ms = e0.elapsed_time(e1) / args.steps
    kms = {n: sum(row[2 * i].elapsed_time(row[2 * i + 1]) for row in evs) / args.steps
           for i, n in enumerate(names)}
    costs = kernel_costs(T, d, d, L, var == 1, 2)
    intra = [n for n in names if n.split("_")[0] in ("dq", "dk", "dv", "dkv")]
    intra_fl = B * NH * sum(costs[n][0] for n in intra)
    intra_ms = sum(kms[n] for n in intra)
    return {"bwd_ms": ms, "bwd_tflops": B * NH * flops_bwd(T, d, d, L) / ms / 1e9,
            "bwd_kernel_ms": kms, "bwd_intra_tflops": intra_fl / intra_ms / 1e9,
            "bwd_intra_pct_bf16_peak": 100 * intra_fl / intra_ms / 1e9 / peaks["bf16_tflops"]}


def workload_config(spec, n):
    return {"workload": WORKLOAD, "cell": "mLSTMexp" if spec["variant"] == 1 else "mLSTMsig",
            "B": spec["B"], "NH": spec["NH"], "T": spec["T"], "d_qk": spec["d_qk"],
            "d_hv": spec["d_hv"], "chunk": spec["chunk"], "pass": "fwd+bwd",
            "global_batch": spec["B"] * n, "seq_len": spec["T"],
            "parallelism": f"replicas{n}" if n > 1 else "single",
            "l2": "no flush: q, k, v, dh are %d MB each, larger than the 126 MB L2"
                  % (spec["B"] * spec["NH"] * spec["T"] * spec["d_qk"] * 2 >> 20)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def main():
    global WORKLOAD
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="forward chunk/sequence sweep at B8 H32 d128 instead of the headline step")
    ap.add_argument("--sweep-t", default=None, help="comma list of T for --sweep")
    ap.add_argument("--sweep-chunk", default=None, help="comma list of chunk sizes for --sweep")
    ap.add_argument("--sweep-batch", type=int, default=8,
                    help="B for --sweep (smaller for ncu captures; the sweep workload is B8)")
    ap.add_argument("--sweep-cells", default=None,
                    help="comma subset of sig,exp,exp_igate_bias_m10 for --sweep")
    ap.add_argument("--sweep-bwd", action="store_true",
                    help="also time the backward at every --sweep point")
    ap.add_argument("--retnet", action="store_true",
                    help="retention (RetNet decays) through the SIG kernels at B8 H32 d128, "
                         "T from --sweep-t or the 128..16384 list")
    ap.add_argument("--decode", action="store_true",
                    help="one-token steps (generation) at B8 H32 d128, and the prefill hand-off")
    ap.add_argument("--batch", type=int, default=None,
                    help="override B (smaller captures for ncu; the default is the workload's B)")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["exp_b8h32_t4096_d128_c128", "train_b4h16_t8192_d256_c256",
                             "sig_long_b1h8_t65536_c1024"],
                    help="bf16 workload of the fwd+bwd step (default: the headline)")
    ap.add_argument("--variant", choices=["sig", "exp"], default=None,
                    help="override the workload's cell variant")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from mlstm_chunkwise_attention_b200.synthetic import WORKLOADS
    WORKLOAD = args.workload
    spec = dict(WORKLOADS[WORKLOAD])
    if args.batch is not None:
        spec["B"] = args.batch
    if args.variant is not None:
        spec["variant"] = 0 if args.variant == "sig" else 1

    if args.impl == "reference":
        return run_reference(args, spec)
    if args.sweep:
        return run_sweep(args)
    if args.retnet:
        return run_retnet(args)
    if args.decode:
        return run_decode(args)

    import torch
    import torch.distributed as dist
    from mlstm_chunkwise_attention_b200 import binding
    from mlstm_chunkwise_attention_b200.synthetic import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    B, NH, T, dqk, dhv, L, var = (spec[k] for k in ("B", "NH", "T", "d_qk", "d_hv", "chunk", "variant"))
    dtype = torch.bfloat16
    cpu = make_inputs(B, NH, T, dqk, dhv, seed=spec["seed"] + 1000 * rank,
                      igate_mean=spec["igate_mean"], fgate_mean=spec["fgate_mean"], dtype=dtype,
                      with_dh=True)
    x = {k: v.to(dev) for k, v in cpu.items()}
    sizes = binding.problem_sizes(x["q"], x["v"], L, var)
    saved = torch.empty(binding.mlstm_saved_size(*sizes), dtype=torch.uint8, device=dev)
    wsb = binding.mlstm_bwd_workspace_size(*sizes)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    h = torch.empty_like(x["v"])
    grads = {"dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]),
             "dv": torch.empty_like(x["v"]), "dig": torch.empty_like(x["igate"]),
             "dfg": torch.empty_like(x["fgate"])}
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    nf = binding.mlstm_fwd_launch_count(*sizes)
    nb = binding.mlstm_bwd_launch_count(*sizes)
    names = ([binding.mlstm_launch_name(0, i, *sizes) for i in range(nf)]
             + [binding.mlstm_launch_name(1, i, *sizes) for i in range(nb)])

    def step(src, fwd_ev=None, bwd_ev=None, out=None):
        o = out if out is not None else {"h": h, **grads}
        if fwd_ev is not None:
            binding.mlstm_set_timing_events(fwd_ev, 2 * nf)
        st = binding.mlstm_fwd(src["q"].data_ptr(), src["k"].data_ptr(), src["v"].data_ptr(),
                               src["igate"].data_ptr(), src["fgate"].data_ptr(), o["h"].data_ptr(),
                               saved.data_ptr(), None, 0, *sizes, sh)
        if st != 0:
            raise binding.MLSTMError(st, "mlstm_fwd")
        if bwd_ev is not None:
            binding.mlstm_set_timing_events(bwd_ev, 2 * nb)
        st = binding.mlstm_bwd(src["q"].data_ptr(), src["k"].data_ptr(), src["v"].data_ptr(),
                               src["igate"].data_ptr(), src["fgate"].data_ptr(), o["h"].data_ptr(),
                               src["dh"].data_ptr(), saved.data_ptr(), o["dq"].data_ptr(),
                               o["dk"].data_ptr(), o["dv"].data_ptr(),
                               o["dig"].data_ptr(), o["dfg"].data_ptr(), ws.data_ptr(),
                               wsb, *sizes, sh)
        binding.mlstm_set_timing_events(None, 0)
        if st != 0:
            raise binding.MLSTMError(st, "mlstm_bwd")

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(v):
        return reduce_max(v, world, dev)

    # ---- device-timed region: inputs resident in HBM
    for _ in range(args.warmup):
        step(x)
    ev_keep = []
    fwd_evs, bwd_evs = [], []
    for _ in range(args.steps):
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(2 * nf)]
        be = [torch.cuda.Event(enable_timing=True) for _ in range(2 * nb)]
        for e in fe + be:  # creates the underlying CUDA event, outside the timed region
            e.record(stream)
        ev_keep.append((fe, be))
    torch.cuda.synchronize(dev)
    for fe, be in ev_keep:
        fwd_evs.append((ctypes.c_void_p * (2 * nf))(*[e.cuda_event for e in fe]))
        bwd_evs.append((ctypes.c_void_p * (2 * nb))(*[e.cuda_event for e in be]))
        assert all(p_ for p_ in fwd_evs[-1]) and all(p_ for p_ in bwd_evs[-1])
    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    start.record(stream)
    for i in range(args.steps):
        step(x)
    end.record(stream)
    barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    ms_max = max_over_ranks(ms)
    # per-kernel times: the same steps once more with every kernel on the caller's stream
    # (the timed steps overlap dq with the backward walker), each kernel bracketed alone
    binding.mlstm_set_serial_launches(True)
    for i in range(args.steps):
        step(x, fwd_evs[i], bwd_evs[i])
    binding.mlstm_set_serial_launches(False)
    barrier()
    per_kernel = {n: 0.0 for n in names}
    for fe, be in ev_keep:
        for i in range(nf):
            per_kernel[names[i]] += fe[2 * i].elapsed_time(fe[2 * i + 1])
        for i in range(nb):
            per_kernel[names[nf + i]] += be[2 * i].elapsed_time(be[2 * i + 1])
    per_kernel = {n: v / args.steps for n, v in per_kernel.items()}  # ms per launch

    heads = B * NH
    step_flops = heads * (flops_fwd(T, dqk, dhv, L) + flops_bwd(T, dqk, dhv, L))
    tflops = step_flops * args.steps * world / (ms_max * 1e-3) / 1e12
    tokens_s = B * T * args.steps * world / (ms_max * 1e-3)
    peaks = load_peaks()

    # ---- roofline of the dominant kernel
    costs = kernel_costs(T, dqk, dhv, L, var == 1, 2)
    dom = max(per_kernel, key=per_kernel.get)
    fl, by = costs[dom]
    dur_s = per_kernel[dom] * 1e-3
    bound = kernel_bound(dom)
    if bound == "hbm" or (bound != "alu" and by / peaks["hbm_gbs"] > fl / (peaks["bf16_tflops"] * 1e3)):
        bound = "hbm"
        achieved, peak, unit = heads * by / dur_s / 1e9, peaks["hbm_gbs"], "GB/s"
        peak_src = peaks["source"]
    elif bound == "tensor":
        achieved, peak, unit = heads * fl / dur_s / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s"
        peak_src = peaks["source"] + " (sustained)"
    else:
        achieved, peak, unit = heads * fl / dur_s / 1e12, FP32_CORE_TFLOPS, "TFLOP/s"
        peak_src = "derived: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz"
    traffic = committed_traffic(dom, WORKLOAD)
    roofline = {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                "algorithmic_per_launch": heads * (by if bound == "hbm" else fl),
                "ms_per_launch": per_kernel[dom]}

    # ---- end to end through the C ABI with pinned host buffers: every step copies its
    # inputs in from pinned host memory and all of its results (h and the five gradients)
    # back out.  Timed twice: one stream (copy in, compute, copy out, step after step), and
    # pipelined as a user streaming batches would run it, with two device buffer sets and one
    # copy stream per direction, so step i+1's inputs cross the host link while step i's
    # results come back (the link is full duplex) and its compute runs in between.
    host_in = {k: v.pin_memory() for k, v in cpu.items()}
    out_keys = ["h"] + list(grads)
    xd = [{k: torch.empty_like(v) for k, v in x.items()} for _ in range(2)]
    od = [{"h": h, **grads}, {k: torch.empty_like(v) for k, v in [("h", h), *grads.items()]}]
    host_out = [{k: torch.empty(od[0][k].shape, dtype=dtype).pin_memory() for k in out_keys}
                for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(host_out[0][k].numel() * host_out[0][k].element_size() for k in out_keys)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_in + ev_comp + ev_out:
        e.record(stream)

    def e2e_serial_step():
        for k_ in xd[0]:
            xd[0][k_].copy_(host_in[k_], non_blocking=True)
        step(xd[0], out=od[0])
        for k_ in out_keys:
            host_out[0][k_].copy_(od[0][k_], non_blocking=True)

    def e2e_pipelined_step(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[b])  # the compute that read this input set is done
            for k_ in xd[b]:
                xd[b][k_].copy_(host_in[k_], non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])  # this output set has been read back
        step(xd[b], out=od[b])
        ev_comp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            for k_ in out_keys:
                host_out[b][k_].copy_(od[b][k_], non_blocking=True)
            ev_out[b].record(s_out)

    def timed(fn, pipelined):
        for i in range(args.warmup):
            fn(i) if pipelined else fn()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(args.steps):
            fn(i) if pipelined else fn()
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        e1.record(stream)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1))

    del x
    e2e_serial_ms = timed(e2e_serial_step, False)
    e2e_ms = timed(e2e_pipelined_step, True)
    e2e_tflops = step_flops * args.steps * world / (e2e_ms * 1e-3) / 1e12

    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from mlstm_chunkwise_attention_b200.synthetic import sample_heads
        cpu_base = oracle_sample(spec, sample_heads(B, NH, 8, 99), budget_s=15.0)
        cpu_base.pop("seconds", None)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": tflops, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(spec, world),
        "tokens_per_s": tokens_s, "pct_bf16_peak": 100.0 * tflops / (world * peaks["bf16_tflops"]),
        "kernel_ms": per_kernel,
        "kernel_ms_mode": "each kernel alone (mlstm_set_serial_launches); the timed steps run "
                          "dq alongside the backward walker where the plan has one",
        "roofline": roofline,
        "cpu_baseline": cpu_base,
        "e2e": {"value": e2e_tflops, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
                "mode": "pipelined: two device buffer sets, one copy stream per direction; "
                        "step i+1's input copies overlap step i's result copies",
                "serial_ms_per_step": e2e_serial_ms / args.steps},
        "gpu_launches": args.steps * (nf + nb),
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
