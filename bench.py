#!/usr/bin/env python
"""Throughput of the Cosmos 3 MoT layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload t2v480] [--impl native|reference]

A step is one pass of the whole hot path over one synthetic batch: the layout
and mRoPE-table build, then one MoT layer forward with the Euler step
(cosmot_layer_forward: routed norms, QKV + mRoPE, attention, O + residual,
gate/up + SiLU, down + residual, final norm, velocity + Euler).  Inputs live
in HBM when the timed region starts; L2 is flushed (256 MiB write) between
steps outside the timed events.  Rank 0 prints one JSON line.

With N > 1 (torchrun) every rank runs its own sequence: independent replicas,
no collective on the data path ("scaling": "weak"); the step time is the max
over ranks.  `--impl reference` times the fp64 CPU oracle instead (rank 0
only) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "MoT layer tokens/s and attention+GEMM TFLOP/s (% of B200 bf16 peak), 1 GPU"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by stage, with the
# sha256 of the kernel source it was taken on (comments excluded); reported
# only while that code is unchanged.
NCU_TRAFFIC = {
    # one attention launch at the 480p shape (18,978 rows x 32 heads):
    # dram__bytes_read.sum 475,295,232 + dram__bytes_write.sum 135,822,848
    "t2v480:attention": {"bytes_per_launch": 611118080, "src_sha": "5ebc251138102a27"},
}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default="t2v480", choices=sorted(synth.PRESETS))
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--micro", choices=["attention", "gemm", "mrope", "euler", "rmsnorm", "epilogues"],
                   help="time one kernel alone on the workload's widths (prints its own JSON line); "
                        "'epilogues' times the QKV and velocity GEMMs with their fused mRoPE and Euler "
                        "epilogues against the same GEMMs with a plain epilogue")
    p.add_argument("--tokens", type=int, default=0, help="rows for --micro (default: the workload's N)")
    return p.parse_args()


# ---------------------------------------------------------------- algorithmic work

class Counts:
    """Token counts of one packed sequence plus its chunk ids (host copy)."""

    def __init__(self, n_ar, n_clean, n_noisy, chunk=None):
        self.n_ar, self.n_clean, self.n_noisy = n_ar, n_clean, n_noisy
        self.n_tokens = n_ar + n_clean + n_noisy
        self.chunk = chunk


def attention_pairs(lay, mode: str) -> int:
    """Visible (query, key) pairs of one sequence under the MoT mask: causal
    pairs inside AR, every AR key for each DM row, and every DM key (full) or
    the DM keys of the same or earlier chunks (block-causal)."""
    n_ar, n = lay.n_ar, lay.n_tokens
    n_dm = n - n_ar
    pairs = n_ar * (n_ar + 1) // 2 + n_dm * n_ar
    if mode == "full":
        pairs += n_dm * n_dm
    else:
        ch = np.asarray(lay.chunk[n_ar:], dtype=np.int64)
        pairs += int(np.searchsorted(np.sort(ch), ch, side="right").sum())
    return int(pairs)


def stage_work(dims, R, nz, pairs):
    """(flops, bytes) per stage of one layer call, algorithmic (operands counted
    once, only visible attention pairs): R rows computed, nz noisy rows."""
    dd, F, hd = dims.d_model, dims.ffn, dims.head_dim
    qc, qkvc = dims.q_cols, dims.qkv_cols
    w_set = 2  # bytes per bf16
    # h1 (the residual stream between the two halves) is float32: written by the
    # O projection, read by the pre-FFN norm and by the down projection
    return {
        "norm1": (0, R * dd * 4),
        "qkv_mrope": (2 * R * dd * qkvc, (R * dd + 2 * qkvc * dd + R * qkvc) * w_set),
        "attention": (4 * pairs * dims.n_heads * hd, (R * qkvc + R * qc) * w_set),
        "oproj_residual": (2 * R * qc * dd, (R * qc + 2 * dd * qc + R * dd) * w_set + R * dd * 4),
        "norm2": (0, R * dd * 4 + R * dd * 2),
        "gateup_silu": (2 * R * dd * 2 * F, (R * dd + 4 * F * dd + R * F) * w_set),
        "down_residual": (2 * R * F * dd, (R * F + 2 * dd * F + R * dd) * w_set + R * dd * 4),
        "norm_final": (0, nz * dd * 4),
        "velocity_euler": (2 * nz * dd * dd, (nz * dd * 3 + dd * dd) * w_set),
    }


def resolve_schedule(wl, use_oracle: bool):
    """A workload with its sampler noise levels filled in: the flow-shift
    schedule comes from the library's host function (native arm) or the
    oracle (reference arm); tests check that the two agree bit for bit."""
    if wl.sigmas or wl.shift <= 0:
        return wl
    import dataclasses
    if use_oracle:
        from oracle import layer as olayer
        sig = olayer.shift_sigmas(wl.n_sampler_steps, wl.shift)
    else:
        from flow_matching_dit_cosmot_b200 import _lib as L
        sig = L.cosmot_flow_shift_sigmas(wl.n_sampler_steps, wl.shift)
    return dataclasses.replace(wl, sigmas=tuple(float(x) for x in sig))


def workload_kind(wl) -> str:
    if wl.stream is not None:
        return "stream"
    return "sampler" if len(wl.sigmas) > 2 else "layer"


def stream_layout_spec(wl, block: int):
    """One streaming step as a packed sequence: AR rows, the cached history
    blocks as clean latent steps, the block being generated as the noisy step."""
    v = wl.layout.video
    return dict(n_text=wl.layout.n_text, video=(v.views, v.grid_h, v.grid_w, v.fps, wl.stream.cached_blocks, 1),
                tau_offset=block)


def reduce_max(value: float, device=None) -> float:
    """Max of `value` over all ranks (the job's time is its slowest rank's);
    the value itself on a single process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank_step * steps / (max_ms / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = self._match(uuid)
        self.proc = None
        self.out = os.path.join("/tmp", f"cosmot_clocks_{os.getpid()}.csv")

    @staticmethod
    def _match(uuid):
        """nvidia-smi's UUID ("GPU-...") of the torch device, or None."""
        if uuid is None:
            return None
        want = str(uuid).lower().replace("gpu-", "")
        try:
            out = subprocess.run(["nvidia-smi", "--query-gpu=uuid", "--format=csv,noheader"], capture_output=True,
                                 text=True, timeout=30).stdout
        except (OSError, subprocess.SubprocessError):
            return None
        for line in out.split():
            if line.strip().lower().replace("gpu-", "") == want:
                return line.strip()
        return None

    # NVML clock-event reason bits (nvml.h: clocksEventReason*); read only
    _NVML_REASONS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
                     ("hw_thermal_slowdown", 0x40))

    def _nvml_start(self):
        """Samples SM clock and clock-event reasons every 10 ms through NVML in a
        thread (nvidia-smi's 200 ms loop gives a timed region of a few hundred
        ms only two or three samples).  Returns False if NVML is unavailable."""
        try:
            import pynvml
            pynvml.nvmlInit()
        except Exception:
            return False
        handle = None
        try:
            count = pynvml.nvmlDeviceGetCount()
            if self.uuid is None and count != 1:
                return False  # NVML indices ignore CUDA_VISIBLE_DEVICES: match by UUID or not at all
            for i in range(count):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if self.uuid is None or u.lower() == self.uuid.lower():
                    handle = h
                    break
        except Exception:
            handle = None
        if handle is None:
            return False
        import threading
        self._nvml, self._h, self._samples, self._stop = pynvml, handle, [], threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    sm = self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM)
                    smax = self._nvml.nvmlDeviceGetMaxClockInfo(self._h, self._nvml.NVML_CLOCK_SM)
                    get = getattr(self._nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                        self._nvml.nvmlDeviceGetCurrentClocksThrottleReasons
                    rs = get(self._h)
                    self._samples.append((sm, smax, rs))
                except Exception:
                    pass
                self._stop.wait(0.01)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return True

    def _nvml_stop(self):
        self._stop.set()
        self._thread.join(timeout=5)
        try:
            self._nvml.nvmlShutdown()
        except Exception:
            pass
        sm = [x[0] for x in self._samples]
        smax = [x[1] for x in self._samples]
        reasons = {nm for _, _, rs in self._samples for nm, bit in self._NVML_REASONS if rs & bit}
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "NVML, every 10 ms"}

    def start(self):
        self.nvml = self._nvml_start()
        if self.nvml:
            return
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.f = open(self.out, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if getattr(self, "nvml", False):
            return self._nvml_stop()
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.out):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.out)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- reference arm (fp64 CPU oracle)

_ORACLE = {}


def oracle_setup(wl):
    """Oracle inputs of the workload (same seeded generators as the GPU arm)."""
    if wl.name not in _ORACLE:
        from oracle import layer as olayer
        from oracle import layout as olayout
        W = olayer.weights_from_bits(wl.dims, synth.make_weights(wl.dims, wl.weight_seed))
        if workload_kind(wl) == "stream":
            lay = olayout.build_layout(synth.LayoutSpec(n_text=wl.layout.n_text, video=wl.layout.video))
            h_ar = synth.bf16_to_f64(synth.make_activations(lay.n_ar, wl.dims.d_model, wl.act_seed(0)))
            hist = [synth.bf16_to_f64(synth.make_activations(lay.n_noisy, wl.dims.d_model, 4000 + k))
                    for k in range(wl.stream.cached_blocks)]
            st = olayer.StreamState(slots=wl.stream.cached_blocks)
            spec_blk = synth.LayoutSpec(n_text=wl.layout.n_text, video=wl.layout.video)
            for k, x in enumerate(hist):  # prefill, not timed
                olayer.stream_commit(wl.dims, W, st, x, olayout.build_layout(spec_blk, tau_offset=k))
            _ORACLE[wl.name] = (lay, W, (h_ar, hist, st))
        else:
            lay = olayout.build_layout(wl.layout)
            h64 = synth.bf16_to_f64(synth.make_activations(lay.n_tokens, wl.dims.d_model, wl.act_seed(0)))
            _ORACLE[wl.name] = (lay, W, h64)
    return _ORACLE[wl.name]


def oracle_sample(wl, quick: bool = False):
    """Times the fp64 oracle on a bounded sample of one step of the workload.

    Returns (seconds for one whole step, seconds spent, description).
      layer:   two row samples (256 and 512 noisy query rows, fewer for small
               layouts; K and V formed for every row each time), extrapolated
               linearly to all rows and the batch;
      sampler: the whole 10-step sampling of one sequence, times the batch;
      stream:  one denoising step on 256 and 512 of the block's rows against
               a cache of 8 prefilled history blocks (prefill not timed),
               extrapolated to the block and its 4 steps, plus the K/V commit.
    """
    from oracle import layer as olayer
    from oracle import layout as olayout
    kind = workload_kind(wl)
    lay, W, data = oracle_setup(wl)
    # Row samples large enough that the per-row work (FFN, attention rows)
    # is measured at full-size memory behaviour, not from cache.
    big = 16 if quick else 256
    rows_lo = min(big, max(lay.n_noisy // 4, 1))
    rows_hi = min(2 * big, max(lay.n_noisy // 2, 2))
    if kind == "layer":
        dm0 = lay.n_ar + lay.n_clean
        t = []
        for r in (rows_lo, rows_hi):
            rows = np.arange(dm0, min(lay.n_tokens, dm0 + r))
            t0 = time.perf_counter()
            olayer.layer_forward(wl.dims, W, data, lay.region, lay.pos, lay.chunk, wl.sigmas[0], wl.sigmas[1],
                                 wl.mask_mode, rows=rows)
            t.append(time.perf_counter() - t0)
        per_row = max(t[1] - t[0], 0.0) / (rows_hi - rows_lo)
        fixed = max(t[0] - rows_lo * per_row, 0.0)
        return ((fixed + per_row * lay.n_tokens) * wl.batch, sum(t),
                f"oracle layer forward on {rows_lo} and {rows_hi} noisy query rows (K/V of all {lay.n_tokens} "
                f"rows each), extrapolated linearly to all rows and the batch"
                + (" (both passes of each guided pair; the guided combine is not timed)" if wl.guidance else ""))
    if kind == "sampler":
        # The oracle recomputes every row at every step, so its steps cost the
        # same: time one and scale by the step count.
        t0 = time.perf_counter()
        olayer.layer_forward(wl.dims, W, data, lay.region, lay.pos, lay.chunk, wl.sigmas[0], wl.sigmas[1],
                             wl.mask_mode)
        t = time.perf_counter() - t0
        n = len(wl.sigmas) - 1
        return (t * n * wl.batch * wl.n_layers, t,
                f"one oracle layer forward of a {lay.n_tokens}-token sequence (all rows), times {n} sampler steps, "
                f"the batch of {wl.batch}" + (f" and the {wl.n_layers} layers" if wl.n_layers > 1 else ""))
    h_ar, hist, st = data
    lb = olayout.build_layout(synth.LayoutSpec(n_text=wl.layout.n_text, video=wl.layout.video),
                              tau_offset=len(hist))
    x0 = synth.bf16_to_f64(synth.make_activations(lay.n_noisy, wl.dims.d_model, 5000))
    t = []
    for r in (rows_lo, rows_hi):
        t0 = time.perf_counter()
        olayer.stream_block(wl.dims, W, st, h_ar, x0, lb, wl.sigmas, rows=np.arange(r))
        t.append(time.perf_counter() - t0)
    per_row = max(t[1] - t[0], 0.0) / (rows_hi - rows_lo)
    fixed = max(t[0] - rows_lo * per_row, 0.0)
    t0 = time.perf_counter()
    k, v = olayer.project_kv(wl.dims, W, x0, lb.region[lb.n_ar:], lb.pos[lb.n_ar:])  # the commit's work
    t_commit = time.perf_counter() - t0
    n = len(wl.sigmas) - 1
    return (n * (fixed + per_row * lay.n_noisy) + t_commit, sum(t) + t_commit,
            f"one oracle denoising step on {rows_lo} and {rows_hi} of the {lay.n_noisy} block rows against "
            f"{len(hist)} cached blocks, extrapolated to the block, times {n} steps, plus the timed K/V commit")


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 0) for i in threadpool_info()), default=0)
        if n:
            return n
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    kind = workload_kind(wl)
    lay = oracle_setup(wl)[0]
    if kind == "stream":
        tokens = lay.n_noisy * (len(wl.sigmas) - 1)
        seq_len = lay.n_ar + wl.stream.cached_blocks * lay.n_noisy + lay.n_noisy
    else:
        tokens = wl.batch * lay.n_tokens * (len(wl.sigmas) - 1 if kind == "sampler" else 1)
        seq_len = lay.n_tokens
    for _ in range(args.warmup):
        oracle_sample(wl, quick=True)  # warm-up: the smallest sample
    t_full, t_spent, sample = [], 0.0, ""
    for _ in range(args.steps):
        tf, ts, sample = oracle_sample(wl)
        t_full.append(tf)
        t_spent += ts
    value = tokens * len(t_full) / sum(t_full)
    cores = cpu_threads()
    cfg = config_block(wl, lay, args.gpus)
    cfg["seq_len"] = seq_len
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(t_full),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Philox: activations N(0,1), weights N(0,0.02), gains 1+N(0,0.02))",
        "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s_sampled": t_spent,
    }
    print(json.dumps(line), flush=True)


def config_block(wl, lay, n_gpus):
    return {"workload": f"{wl.name}: {wl.description}", "global_batch": wl.batch * n_gpus,
            "seq_len": lay.n_tokens, "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU",
            "d_model": wl.dims.d_model, "heads": wl.dims.n_heads, "head_dim": wl.dims.head_dim,
            "ffn": wl.dims.ffn, "n_ar": lay.n_ar, "n_clean": lay.n_clean, "n_noisy": lay.n_noisy,
            "mask": wl.mask_mode, "sigma": [wl.sigmas[0], wl.sigmas[1]],
            **({"guidance": wl.guidance, "prompt_pairs": wl.batch // 2} if wl.guidance is not None else {}),
            **({"layers": wl.n_layers, "distinct_layer_weight_draws": wl.weight_draws or wl.n_layers}
               if wl.n_layers > 1 else {}),
            **({"shift": wl.shift, "sigmas": list(wl.sigmas)} if wl.shift > 0 else {}),
            **({"action_dim": wl.action_dim, "action_rows": wl.layout.action_clean + wl.layout.action_noisy}
               if wl.action_dim else {}),
            "l2": "flushed between steps (256 MiB write, outside the timed events)"}


# ---------------------------------------------------------------- native arm

def code_sha(text):
    """sha256 of source text with its // comments and blank lines removed, so
    that a comment edit keeps the counters taken on the same code."""
    code = []
    for line in text.splitlines():
        cut = line.find("//")
        line = (line if cut < 0 else line[:cut]).rstrip()
        if line:
            code.append(line)
    return hashlib.sha256("\n".join(code).encode()).hexdigest()[:16]


def src_sha(name):
    p = os.path.join(ROOT, "flow_matching_dit_cosmot_b200", "csrc", name)
    return code_sha(open(p, encoding="utf-8").read()) if os.path.exists(p) else None


def stage_spans(n_layers, n_stage):
    """(stage, k) pairs: that stage of one layer call runs from event k to event k + 1.

    The event layout of the stage-timed entry points: one layer has an event
    before each of its n_stage stages and one after the last; a stack of
    n_layers records 8 l + i before stage i (< 7) of layer l, 8 l + 7 after
    that layer's last one (where the final-norm stage starts), 8 n_layers
    before the velocity stage and 8 n_layers + 1 after it.
    """
    if n_layers > 1:
        return [(j, 8 * lyr + j) for lyr in range(n_layers) for j in range(7)] + [(7, 8 * n_layers - 1),
                                                                                  (8, 8 * n_layers)]
    return [(j, j) for j in range(n_stage)]


def dominant_marks(n_layers, n_stage, dom):
    """Event indices a timed step records: the two boundaries of stage `dom` in every layer."""
    return {k + e for j, k in stage_spans(n_layers, n_stage) if j == dom for e in (0, 1)}


def stage_times(per_step_evs, n_layers, n_stage, steps):
    """Mean device ms per step of every stage, from the events recorded at its two
    boundaries (None: that boundary was not recorded)."""
    import numpy as np
    out = np.zeros(n_stage)
    spans = stage_spans(n_layers, n_stage)
    for per_call in per_step_evs:
        for evs in per_call:
            for j, k in spans:
                if evs[k] is not None and evs[k + 1] is not None:
                    out[j] += evs[k].elapsed_time(evs[k + 1])
    return out / steps


def run_native(args, wl):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))

    from flow_matching_dit_cosmot_b200 import _lib as L
    from flow_matching_dit_cosmot_b200 import api as A

    kind = workload_kind(wl)
    dims_s = wl.dims
    dev = torch.device("cuda", local)
    sh = torch.cuda.current_stream().cuda_stream
    stream = torch.cuda.current_stream()
    n_stage = L.COSMOT_LAYER_STAGES
    mode = L.COSMOT_MASK_FULL if wl.mask_mode == "full" else L.COSMOT_MASK_BLOCK_CAUSAL

    def spec_for(step_idx):
        if kind == "stream":
            return A.layout_spec(**stream_layout_spec(wl, step_idx % 16))
        v = wl.layout.video
        return A.layout_spec(wl.layout.n_text,
                             None if v is None else (v.views, v.grid_h, v.grid_w, v.fps, v.clean_steps, v.noisy_steps),
                             wl.layout.audio_clean, wl.layout.audio_noisy, wl.layout.audio_rate,
                             wl.layout.action_clean, wl.layout.action_noisy, wl.layout.action_hz, wl.layout.proprio)

    dl = A.build_layout(spec_for(0), dev)
    lay = Counts(dl.n_ar, dl.n_clean, dl.n_noisy, dl.chunk.cpu().numpy())
    B, N, d = wl.batch, lay.n_tokens, dims_s.d_model

    def to_dev(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).to(dev)

    n_layers = wl.n_layers
    if n_layers > 1:  # a stack: distinct draws go to the device once, layers share them
        draws = synth.make_stack_weights(dims_s, wl.weight_seed, n_layers, distinct=wl.weight_draws)
        dev_draws = {}
        for dw in draws:
            if id(dw) not in dev_draws:
                dev_draws[id(dw)] = {k: to_dev(v) for k, v in dw.items()}
        stack_w = [dev_draws[id(dw)] for dw in draws]
        w = stack_w[-1]
    else:
        w = {k: to_dev(v) for k, v in synth.make_weights(dims_s, wl.weight_seed).items()}
    h_host = np.stack([synth.make_activations(N, d, wl.act_seed(rank * B + b)) for b in range(B)])
    guided = wl.guidance is not None
    if guided:  # each (cond, base) pair shares its DM rows; the prompts (AR rows) differ
        h_host[1::2, lay.n_ar:] = h_host[0::2, lay.n_ar:]
    h = to_dev(h_host)
    h_out = torch.empty_like(h)
    pos = torch.empty((N, 3), dtype=torch.float32, device=dev)
    chunk = torch.empty((N,), dtype=torch.int32, device=dev)
    cs = torch.empty((N, dims_s.head_dim // 2, 2), dtype=torch.float32, device=dev)
    dims = A.make_dims(dims_s.d_model, dims_s.n_heads, dims_s.n_kv_heads, dims_s.head_dim, dims_s.ffn,
                       dims_s.rope_sections, dims_s.rope_base, dims_s.eps)
    layer = A.MoTLayer(dims, w)
    stack = A.MoTStack(dims, stack_w) if n_layers > 1 else None
    ca = wl.action_dim
    if ca:  # domain action heads; the action state of each (cond, base) pair is shared
        a_clean, a_noisy = wl.layout.action_clean, wl.layout.action_noisy
        na = a_clean + a_noisy
        v = wl.layout.video
        clean_row = lay.n_ar + (v.views * v.grid_h * v.grid_w * v.clean_steps if v else 0) + wl.layout.audio_clean
        wi_h, wo_h = synth.make_action_weights(d, ca, wl.weight_seed + 500)
        w_in, w_out = to_dev(wi_h), to_dev(wo_h)
        xa_host = np.concatenate([synth.make_actions(na, ca, wl.act_seed(rank * B + b)) for b in range(B)])
        if guided:
            for pr in range(B // 2):
                xa_host[(2 * pr + 1) * na:(2 * pr + 2) * na] = xa_host[2 * pr * na:(2 * pr + 1) * na]
        xa = to_dev(xa_host)
        xa_src = xa.clone()

        def act_desc(s0, s1):  # the actions follow the same schedule as the video
            return L.ActionDesc(ca, a_clean, a_noisy, clean_row, w_in.data_ptr(), w_out.data_ptr(), xa.data_ptr(),
                                ca, s0, s1)
    z0 = lay.n_ar + lay.n_clean  # first noisy row of a sequence

    def seq(n_cached):
        return layer.seq_desc(lay.n_ar, lay.n_clean, lay.n_noisy, B, cs, chunk, mode, n_cached=n_cached)

    ws = stack.workspace(seq(0), dev) if stack is not None else layer.workspace(seq(0), dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    # ---- the plan of one step: (n_cached, sigma, sigma_next) per layer call
    sig = wl.sigmas
    if kind == "layer":
        calls = [(0, sig[0], sig[1])]
    elif kind == "sampler":
        calls = [(0, sig[0], sig[1])] + [(lay.n_ar, a, b) for a, b in zip(sig[1:-1], sig[2:])]
    else:
        calls = [(z0, a, b) for a, b in zip(sig[:-1], sig[1:])]
    seqs = {c: seq(c) for c in {c for c, _, _ in calls}}
    # samplers keep the state of the noisy rows in float32 between steps
    # (cosmot_layer_forward_io / cosmot_stack_forward_io); the first call of a
    # sampling or of a streaming block takes it from the bf16 rows of h
    x_state = None
    step_ios = [None] * len(calls)
    if kind in ("sampler", "stream") and not guided and not ca:
        x_state = torch.empty((B, lay.n_noisy, d), dtype=torch.float32, device=dev)
        step_ios = [L.step_io(x_state.data_ptr(), d, 0, 0, i == 0) for i in range(len(calls))]
    if kind == "stream":
        noise = [to_dev(synth.make_activations(lay.n_noisy, d, 5000 + k)) for k in range(4)]
        # prefill the cache: AR rows and the 8 seeded history blocks, K/V in place
        L.cosmot_build_layout(spec_for(0), pos.data_ptr(), chunk.data_ptr(), 0, sh)
        L.cosmot_mrope_table(pos.data_ptr(), N, dims_s.head_dim, dims_s.rope_sections, dims_s.rope_base,
                             cs.data_ptr(), sh)
        L.cosmot_layer_commit_kv(dims, layer.cw, seq(0), h.data_ptr(), 0, ws.data_ptr(), ws.numel(), sh)
        commit_seq = seq(z0)

    def layer_pairs(n_cached):
        """Visible attention pairs of one call (queries = rows >= n_cached)."""
        if n_cached == 0:
            return attention_pairs(lay, wl.mask_mode)
        # DM queries only; every key is visible to them here (full mask, or a
        # block-causal cache that holds only earlier chunks)
        return (N - n_cached) * N

    work = [stage_work(dims_s, B * (N - c), B * lay.n_noisy, B * layer_pairs(c)) for c, _, _ in calls]
    if n_layers > 1:  # every layer runs the body stages; the head runs once
        work = [{nm: ((f * n_layers, b * n_layers) if i < 7 else (f, b)) for i, (nm, (f, b)) in enumerate(wk.items())}
                for wk in work]
    commit_flops = 2 * lay.n_noisy * d * dims_s.qkv_cols if kind == "stream" else 0
    tokens_per_step = {"layer": B * N, "sampler": B * N * len(calls), "stream": B * lay.n_noisy * len(calls)}[kind]

    step_no = [0]
    hcur = [h]  # the input buffer a step runs on (the pipelined end-to-end loop alternates two)

    def handles(evs):
        return [e.cuda_event if e is not None else None for e in evs]

    def step(stage_evs=None, commit_evs=None):
        b = step_no[0]
        step_no[0] += 1
        hp = hcur[0].data_ptr()
        L.cosmot_build_layout(spec_for(b), pos.data_ptr(), chunk.data_ptr(), 0, sh)
        L.cosmot_mrope_table(pos.data_ptr(), N, dims_s.head_dim, dims_s.rope_sections, dims_s.rope_base,
                             cs.data_ptr(), sh)
        for i, (c, s0, s1) in enumerate(calls):
            if ca:
                L.cosmot_policy_step(dims, stack.cw, seqs[c], act_desc(s0, s1), hp, h_out.data_ptr(), s0,
                                     s1, wl.guidance, ws.data_ptr(), ws.numel(), sh,
                                     handles(stage_evs[i]) if stage_evs is not None else None)
            elif stack is not None:
                if stage_evs is not None:
                    L.cosmot_stack_forward_timed(dims, stack.cw, seqs[c], hp, h_out.data_ptr(), s0, s1,
                                                 ws.data_ptr(), ws.numel(), sh, handles(stage_evs[i]),
                                                 step_ios[i])
                else:
                    L.cosmot_stack_forward_io(dims, stack.cw, seqs[c], hp, h_out.data_ptr(), s0, s1,
                                              step_ios[i], ws.data_ptr(), ws.numel(), sh)
            elif stage_evs is not None:
                L.cosmot_layer_forward_timed(dims, layer.cw, seqs[c], hp, h_out.data_ptr(), s0, s1,
                                             ws.data_ptr(), ws.numel(), sh, handles(stage_evs[i]),
                                             wl.guidance, step_ios[i])
            elif guided:
                L.cosmot_layer_forward_cfg(dims, layer.cw, seqs[c], hp, h_out.data_ptr(), s0, s1,
                                           wl.guidance, ws.data_ptr(), ws.numel(), sh)
            else:
                L.cosmot_layer_forward_io(dims, layer.cw, seqs[c], hp, h_out.data_ptr(), s0, s1,
                                          step_ios[i], ws.data_ptr(), ws.numel(), sh)
        if kind == "stream":
            if commit_evs is not None:
                commit_evs[0].record(stream)
            slot = b % wl.stream.cached_blocks
            L.cosmot_layer_commit_kv(dims, layer.cw, commit_seq, hp,
                                     lay.n_ar + slot * lay.n_noisy, ws.data_ptr(), ws.numel(), sh)
            if commit_evs is not None:
                commit_evs[1].record(stream)

    def pre_step():
        flush.zero_()
        if kind == "stream":  # the new block starts from fresh noise
            h[0, z0:].copy_(noise[step_no[0] % len(noise)])
        elif kind == "sampler":  # a new sampling starts from the same seeded noise
            h.copy_(h_src)
            if ca:
                xa.copy_(xa_src)

    h_src = h.clone() if kind == "sampler" else None
    launches_per_step = 2 + n_stage * len(calls) + (2 if kind == "stream" else 0)
    if kind == "stream" and n_layers == 1:  # a key-split attention adds its merge kernel to every call
        sd = L.AttnDesc(n_q=lay.n_noisy, q_key_offset=N - lay.n_noisy, n_keys=N, n_ar=lay.n_ar, n_heads=dims_s.n_heads,
                        n_kv_heads=dims_s.n_kv_heads, head_dim=dims_s.head_dim, mask_mode=mode, batch=B,
                        flags=L.COSMOT_ATTN_NO_TILE_SKIP)
        if L.cosmot_attention_kv_split(sd) > 1:
            launches_per_step += len(calls)
    if n_layers > 1:  # 7 kernels per layer body, 2 for the head (the AR K/V copies are memcpys)
        launches_per_step = 2 + (7 * n_layers + 2) * len(calls)
        if ca:  # the action embedding and the action head; the guided head adds one kernel per pair
            launches_per_step += (2 + (B // 2 if guided else 0)) * len(calls)
    n_ev = 8 * n_layers + 2 if n_layers > 1 else n_stage + 1

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)  # creates the underlying cudaEvent_t
        return evs

    for _ in range(args.warmup):
        pre_step()
        step()
    torch.cuda.synchronize()
    st, where = L.cosmot_get_device_status(sh)
    if st:
        raise RuntimeError(f"device status {L.status_string(st)} at {where}")

    # Instrumented steps, outside the timed region: an event at every stage
    # boundary gives the stage table and picks the dominant stage.  Each event
    # between two kernels also ends their overlapped launch, so these steps run
    # a little slower than the timed ones.
    stage_evs = [[new_events(n_ev) for _ in calls] for _ in range(args.steps)]
    commit_evs = [new_events(2) for _ in range(args.steps)]
    prof_starts, prof_ends = new_events(args.steps), new_events(args.steps)
    for i in range(args.steps):
        pre_step()
        prof_starts[i].record(stream)
        step(stage_evs[i], commit_evs[i])
        prof_ends[i].record(stream)
    torch.cuda.synchronize()
    stage_ms = stage_times(stage_evs, n_layers, n_stage, args.steps)
    prof_ms_step = sum(prof_starts[i].elapsed_time(prof_ends[i]) for i in range(args.steps)) / args.steps
    commit_ms = (sum(e[0].elapsed_time(e[1]) for e in commit_evs) / args.steps) if kind == "stream" else 0.0
    dom = max(range(n_stage), key=lambda j: stage_ms[j])
    dom_keep = dominant_marks(n_layers, n_stage, dom)

    def dom_events():
        """A timed step's events: only the two around the dominant stage (in every layer)."""
        made = iter(new_events(len(dom_keep)))
        return [next(made) if k in dom_keep else None for k in range(n_ev)]

    # The timed steps record events only around the dominant stage, for its
    # roofline; every other kernel boundary keeps its overlapped launch.
    starts, ends = new_events(args.steps), new_events(args.steps)
    dom_evs = [[dom_events() for _ in calls] for _ in range(args.steps)]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(getattr(torch.cuda.get_device_properties(dev), "uuid", None))
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        pre_step()
        starts[i].record(stream)
        step(dom_evs[i])
        ends[i].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    st, where = L.cosmot_get_device_status(sh)
    if st:
        raise RuntimeError(f"device status {L.status_string(st)} at {where}")

    # `value` is throughput over the K timed steps (their summed device time);
    # the median step is reported beside it
    step_ms = [starts[i].elapsed_time(ends[i]) for i in range(args.steps)]
    total_ms = sum(step_ms)
    median_ms = statistics.median(step_ms)
    dom_ms = stage_times(dom_evs, n_layers, n_stage, args.steps)[dom]  # the dominant stage inside the timed steps

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        if kind == "stream":
            in_pin = noise[0].cpu().pin_memory()
            ins = [(h[0, z0:], in_pin)]
            outs = [(torch.empty_like(in_pin).pin_memory(), h[0, z0:])]
        else:
            ins = [(h, torch.from_numpy(h_host.view(np.int16)).view(torch.bfloat16).pin_memory())]
            outs = [(torch.empty((B, lay.n_noisy, d), dtype=torch.bfloat16).pin_memory(), h[:, z0:])]
        if ca:  # a policy reads the action state in and the actions out
            ins.append((xa, torch.from_numpy(xa_host.view(np.int16)).view(torch.bfloat16).pin_memory()))
            outs = [(torch.empty_like(xa, device="cpu").pin_memory(), xa)]

        def e2e_step():
            for dst, src in ins:
                dst.copy_(src, non_blocking=True)
            step()
            for dst, src in outs:
                dst.copy_(src, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        # (a) serial: each step copies in, computes, copies out on one stream
        e_s, e_e = new_events(args.steps), new_events(args.steps)
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            e_s[i].record(stream)
            e2e_step()
            e_e[i].record(stream)
        torch.cuda.synchronize()
        serial_ms = reduce_max(sum(e_s[i].elapsed_time(e_e[i]) for i in range(args.steps)), dev)

        # (b) pipelined, as a serving loop runs it: a copy stream uploads step
        # i+1's inputs and downloads step i-1's result while step i computes;
        # every step's copies are inside the timed region (one event pair
        # around all K steps, L2 flushed before each step's compute).  Without
        # an action state the step's own input buffer alternates between two
        # (the uploads land in it and the result is read from it: no device
        # copy on the compute stream); a policy step stages its inputs.
        cstream = torch.cuda.Stream(dev)
        direct = not ca
        h_alt = h.clone() if direct else None

        def same_view(v, base):  # view v of h, taken of the other buffer
            return base.as_strided(v.size(), v.stride(), v.storage_offset())
        if direct:
            st_in = [[dst for dst, _ in ins], [same_view(dst, h_alt) for dst, _ in ins]]
            st_out = [[src for _, src in outs], [same_view(src, h_alt) for _, src in outs]]
        else:
            st_in = [[torch.empty_like(dst) for dst, _ in ins] for _ in range(2)]
            st_out = [[torch.empty_like(src) for _, src in outs] for _ in range(2)]
        h_out_pin = [[torch.empty_like(dst).pin_memory() for dst, _ in outs] for _ in range(2)]
        K = args.steps
        ev = {k: [torch.cuda.Event() for _ in range(K)] for k in ("in", "used", "out", "down")}
        p_s, p_e = new_events(1)[0], new_events(1)[0]
        torch.cuda.synchronize()
        p_s.record(stream)

        def upload(i):
            with torch.cuda.stream(cstream):
                if i >= 2:  # the slot's previous contents consumed (and, direct, its result downloaded)
                    cstream.wait_event(ev["down" if direct else "used"][i - 2])
                for stg, (_, src) in zip(st_in[i % 2], ins):
                    stg.copy_(src, non_blocking=True)
                ev["in"][i].record(cstream)

        cstream.wait_event(p_s)
        upload(0)
        for i in range(K):
            if i + 1 < K:
                upload(i + 1)
            stream.wait_event(ev["in"][i])
            flush.zero_()
            if direct:
                hcur[0] = h if i % 2 == 0 else h_alt
            else:
                for stg, (dst, _) in zip(st_in[i % 2], ins):
                    dst.copy_(stg, non_blocking=True)
            ev["used"][i].record(stream)
            step()
            if not direct:
                if i >= 2:
                    stream.wait_event(ev["down"][i - 2])  # the output slot's previous download done
                for stg, (_, src) in zip(st_out[i % 2], outs):
                    stg.copy_(src, non_blocking=True)
            ev["out"][i].record(stream)
            with torch.cuda.stream(cstream):
                cstream.wait_event(ev["out"][i])
                for hp, stg in zip(h_out_pin[i % 2], st_out[i % 2]):
                    hp.copy_(stg, non_blocking=True)
                ev["down"][i].record(cstream)
        stream.wait_event(ev["down"][K - 1])
        p_e.record(stream)
        torch.cuda.synchronize()
        hcur[0] = h
        e2e_ms = reduce_max(p_s.elapsed_time(p_e), dev)
        e2e = {"value": job_throughput(tokens_per_step, args.steps, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(sum(src.numel() * 2 for _, src in ins)),
               "d2h_bytes_per_step": int(sum(dst.numel() * 2 for dst, _ in outs)),
               "ms_per_step": e2e_ms / args.steps,
               "mode": "pipelined: a second stream uploads step i+1 and downloads step i-1 while step i computes"
                       + ("; the step's input buffer alternates between two" if direct else "; inputs staged"),
               "serial": {"value": job_throughput(tokens_per_step, args.steps, world, serial_ms),
                          "ms_per_step": serial_ms / args.steps},
               "path": "cosmot_build_layout + cosmot_mrope_table + "
                       + ("cosmot_policy_step" if ca else
                          ("cosmot_stack_forward" if n_layers > 1 else "cosmot_layer_forward_cfg" if guided else
                           "cosmot_layer_forward") + ("_io (float32 state)" if x_state is not None else ""))
                       + (" + cosmot_layer_commit_kv" if kind == "stream" else "")
                       + (", pinned host inputs (h, action state) in, actions out" if ca else
                          ", pinned host input in, x' (noisy rows) out")}

    total_ms = reduce_max(total_ms, dev)

    if rank == 0:
        names = L.STAGE_NAMES
        wsum = {nm: (sum(wk[nm][0] for wk in work), sum(wk[nm][1] for wk in work)) for nm in names}
        flops_total = sum(f for f, _ in wsum.values()) + commit_flops
        peaks, peak_src = load_peaks()
        peak_tf = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        peak_tf_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        peak_bw = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        ms_step = total_ms / args.steps
        stages = {}
        for j, nm in enumerate(names):
            f, b = wsum[nm]
            t_s = stage_ms[j] / 1e3
            ent = {"ms": round(float(stage_ms[j]), 4), "share": round(float(stage_ms[j] / prof_ms_step), 4)}
            if f:
                ent["tflops"] = round(f / t_s / 1e12, 1) if t_s > 0 else None
                ent["frac_of_peak"] = round(f / t_s / 1e12 / peak_tf, 3) if t_s > 0 else None
            else:
                ent["gbs"] = round(b / t_s / 1e9, 1) if t_s > 0 else None
                ent["frac_of_hbm"] = round(b / t_s / 1e9 / peak_bw, 3) if t_s > 0 else None
            stages[nm] = ent
        if kind == "stream":
            stages["kv_commit"] = {"ms": round(commit_ms, 4), "share": round(commit_ms / prof_ms_step, 4),
                                   "tflops": round(commit_flops / (commit_ms / 1e3) / 1e12, 1) if commit_ms else None}
        dname = names[dom]
        f, b = wsum[dname]
        t_dom = dom_ms / 1e3  # per timed step; one launch per layer call
        per_launch = len(calls) * (n_layers if dom < 7 else 1)  # launches of the dominant kernel per step
        src = "attention.cu" if dname == "attention" else ("gemm.cu" if f else "elementwise.cu")
        traffic = None
        rec = NCU_TRAFFIC.get(f"{wl.name}:{dname}")
        if rec and rec.get("src_sha") == src_sha(src):
            traffic = rec["bytes_per_launch"]
        if f:
            achieved = f / t_dom / 1e12
            roof = {"bound": "tensor", "kernel": dname, "achieved": round(achieved, 1), "peak": peak_tf,
                    "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 3), "traffic": traffic,
                    "algorithmic_flops_per_launch": f // per_launch, "launches_per_step": per_launch,
                    "peak_source": f"{peak_src} bf16_tflops_sustained"}
        else:
            achieved = b / t_dom / 1e9
            roof = {"bound": "hbm", "kernel": dname, "achieved": round(achieved, 1), "peak": peak_bw,
                    "unit": "GB/s", "frac": round(achieved / peak_bw, 3), "traffic": traffic,
                    "algorithmic_bytes_per_launch": b // per_launch, "launches_per_step": per_launch,
                    "peak_source": f"{peak_src} hbm_gbs"}
        value = job_throughput(tokens_per_step, args.steps, world, total_ms)
        layer_tflops = flops_total / (ms_step / 1e3) / 1e12
        cfg = config_block(wl, lay, world)
        cfg["step"] = {"layer": ("one guided layer step: both passes of each prompt pair, the guided velocity "
                                  "and one Euler step" if guided else "one layer forward + Euler step"),
                       "sampler": ("policy inference with W_in / W_out action heads, " if ca else "")
                                  + (f"guided (cond, base) pairs, w {wl.guidance}, " if guided else "")
                                  + (f"{n_layers}-layer stack, " if n_layers > 1 else "")
                                  + f"one {len(calls)}-step Euler sampling (step 1 all rows, then DM rows with the "
                                  f"AR K/V kept in the workspace)",
                       "stream": f"one streaming block: {len(calls)} denoising steps of {lay.n_noisy} tokens "
                                 f"against {N - lay.n_noisy} cached key rows, then the block's K/V commit"}[kind]
        cfg["tokens_per_step"] = tokens_per_step
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "median_ms_per_step": round(median_ms, 4),
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Philox: activations N(0,1), weights N(0,0.02), gains 1+N(0,0.02))",
            "config": cfg,
            "tflops": round(layer_tflops, 1),
            "tflops_frac_of_peak": round(layer_tflops / peak_tf, 3),
            "tflops_frac_of_burst_peak": round(layer_tflops / peak_tf_burst, 3),
            "flops_per_step": flops_total,
            "clocks": clk, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "roofline": roof, "stages": stages,
            "stages_from": (f"{args.steps} separate steps with an event at every stage boundary, "
                            f"{prof_ms_step:.4f} ms per step; the timed steps record events around the "
                            f"dominant stage only"),
        }
        if world == 1 and not args.no_cpu_baseline:
            t_full, t_spent, sample = oracle_sample(wl)
            line["cpu_baseline"] = {"value": tokens_per_step / t_full, "unit": UNIT, "cores": cpu_threads(),
                                    "kind": "oracle", "sample": f"{sample}; {t_spent:.1f} s of CPU wall time"}
        print(json.dumps(line), flush=True)

    if world > 1:
        dist.destroy_process_group()


def run_micro(args, wl):
    """One kernel alone, `--steps` timed launches after `--warmup`, L2 flushed
    between launches (outside the events).  Burst peaks apply (kernel timed
    alone)."""
    import torch

    from flow_matching_dit_cosmot_b200 import _lib as L
    from flow_matching_dit_cosmot_b200 import api as A

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dm = wl.dims
    d, hd, H, Hkv = dm.d_model, dm.head_dim, dm.n_heads, dm.n_kv_heads
    T = args.tokens or synth.preset(args.workload).layout.n_ar + synth.preset(args.workload).layout.n_dm
    n_ar = min(wl.layout.n_ar, T)
    g = torch.Generator(device=dev)
    g.manual_seed(3000 + wl.config_id)

    def rnd(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    sh = torch.cuda.current_stream().cuda_stream
    peaks, peak_src = load_peaks()
    qkvc = dm.qkv_cols
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def time_launch(launch):
        for _ in range(args.warmup):
            flush.zero_()
            launch()
        torch.cuda.synchronize()
        st_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        en_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            st_ev[i].record()
            launch()
            en_ev[i].record()
        torch.cuda.synchronize()
        st, where = L.cosmot_get_device_status(sh)
        if st:
            raise RuntimeError(f"device status {L.status_string(st)} at {where}")
        t = [st_ev[i].elapsed_time(en_ev[i]) for i in range(args.steps)]
        return statistics.mean(t), statistics.median(t)

    if args.micro == "epilogues":
        # the QKV projection (mRoPE on its Q and K heads) and the velocity head
        # (Euler step into the state), each against the same GEMM with a plain
        # epilogue: the fused epilogue's cost is the extra time
        a = rnd(T, d)
        w = rnd(qkvc, d, std=0.02)
        out = torch.empty((T, qkvc), dtype=torch.bfloat16, device=dev)
        segs = [(0, n_ar, 0, 0), (n_ar, T, n_ar, 1)]
        pos = torch.empty((T, 3), dtype=torch.float32, device=dev)
        pos[:, 0] = torch.arange(T, device=dev, dtype=torch.float32)
        pos[:, 1:] = (torch.arange(T, device=dev, dtype=torch.float32) % 26)[:, None]
        cs = A.mrope_table(pos, hd, dm.rope_sections, dm.rope_base)
        e_rope = L.Epilogue(kind=L.COSMOT_EPI_MROPE, head_dim=hd, rope_cols=(H + Hkv) * hd, rope_cs=cs.data_ptr(),
                            rope_period=0)
        nz = T - n_ar
        wv = rnd(d, d, std=0.02)
        x = rnd(nz, d)
        xo = torch.empty_like(x)
        vsegs = [(0, nz, 0, 1)]
        e_euler = L.Epilogue(kind=L.COSMOT_EPI_EULER, x=x.data_ptr(), ld_x=d, dsigma=-0.03)
        cases = {
            "qkv_plain": lambda: L.cosmot_routed_linear(a.data_ptr(), d, d, segs, w.data_ptr(), w.data_ptr(), qkvc,
                                                        out.data_ptr(), qkvc, stream=sh),
            "qkv_mrope": lambda: L.cosmot_routed_linear(a.data_ptr(), d, d, segs, w.data_ptr(), w.data_ptr(), qkvc,
                                                        out.data_ptr(), qkvc, e_rope, stream=sh),
            "velocity_plain": lambda: L.cosmot_routed_linear(a.data_ptr(), d, d, vsegs, wv.data_ptr(), wv.data_ptr(),
                                                             d, xo.data_ptr(), d, stream=sh),
            "velocity_euler": lambda: L.cosmot_routed_linear(a.data_ptr(), d, d, vsegs, wv.data_ptr(), wv.data_ptr(),
                                                             d, xo.data_ptr(), d, e_euler, stream=sh),
        }
        res = {k: time_launch(f) for k, f in cases.items()}
        f_qkv, f_vel = 2 * T * d * qkvc, 2 * nz * d * d
        burst = float(peaks["bf16_tflops"])
        line = {"micro": "epilogues", "workload": wl.name, "tokens": T, "steps": args.steps, "warmup": args.warmup,
                "peak_tflops": burst, "peak_source": f"{peak_src} burst"}
        for k, (mean_ms, med_ms) in res.items():
            fl = f_qkv if k.startswith("qkv") else f_vel
            line[k] = {"ms": round(mean_ms, 4), "median_ms": round(med_ms, 4),
                       "tflops": round(fl / (mean_ms / 1e3) / 1e12, 1),
                       "frac": round(fl / (mean_ms / 1e3) / 1e12 / burst, 3)}
        line["mrope_extra_ms"] = round(res["qkv_mrope"][0] - res["qkv_plain"][0], 4)
        line["euler_extra_ms"] = round(res["velocity_euler"][0] - res["velocity_plain"][0], 4)
        # what the same work would cost as a standalone HBM pass at the measured bandwidth
        hbm = float(peaks["hbm_gbs"]) * 1e9
        line["mrope_standalone_floor_ms"] = round((4 * T * (H + Hkv) * hd + T * (hd // 2) * 8) / hbm * 1e3, 4)
        line["euler_standalone_floor_ms"] = round(6 * nz * d / hbm * 1e3, 4)
        print(json.dumps(line), flush=True)
        return
    kv_split = 1
    if args.micro == "attention":
        n_q, q_off = T, 0
        if wl.stream is not None and not args.tokens:
            # a streaming step: the newest block's rows are the queries; every
            # key (AR, the cached blocks, the block itself) is visible to them
            n_q = wl.layout.n_noisy
            T = wl.layout.n_ar + (wl.stream.cached_blocks + 1) * n_q
            q_off = T - n_q
        qkv = rnd(T, qkvc)
        o = torch.empty((n_q, H * hd), dtype=torch.bfloat16, device=dev)
        desc = L.AttnDesc(n_q=n_q, q_key_offset=q_off, n_keys=T, n_ar=n_ar, n_heads=H, n_kv_heads=Hkv, head_dim=hd,
                          mask_mode=L.COSMOT_MASK_FULL, batch=1)
        base = qkv.data_ptr()
        # the key split the layer would take for this shape (1 = none)
        kv_split = L.cosmot_attention_kv_split(desc) if q_off else 1
        split_ws = torch.empty((max(1, L.cosmot_attention_split_workspace(desc, kv_split)),), dtype=torch.uint8,
                               device=dev)

        def launch_plain():
            L.cosmot_mot_attention(desc, base + q_off * qkvc * 2, qkvc, base + 2 * H * hd, base + 2 * (H + Hkv) * hd,
                                   qkvc, o.data_ptr(), H * hd, sh)

        def launch():
            if kv_split == 1:
                return launch_plain()
            L.cosmot_mot_attention_split(desc, base + q_off * qkvc * 2, qkvc, base + 2 * H * hd,
                                         base + 2 * (H + Hkv) * hd, qkvc, o.data_ptr(), H * hd, kv_split,
                                         split_ws.data_ptr(), split_ws.numel(), sh)
        pairs = (n_ar * (n_ar + 1) // 2 + (T - n_ar) * T) if q_off == 0 else n_q * T
        work, unit, peak = 4 * pairs * H * hd, "TFLOP/s", float(peaks["bf16_tflops"])
    elif args.micro == "gemm":
        a = rnd(T, d)
        w = rnd(qkvc, d, std=0.02)
        out = torch.empty((T, qkvc), dtype=torch.bfloat16, device=dev)
        segs = [(0, n_ar, 0, 0), (n_ar, T, n_ar, 1)]

        def launch():
            L.cosmot_routed_linear(a.data_ptr(), d, d, segs, w.data_ptr(), w.data_ptr(), qkvc, out.data_ptr(), qkvc,
                                   stream=sh)
        work, unit, peak = 2 * T * d * qkvc, "TFLOP/s", float(peaks["bf16_tflops"])
    elif args.micro == "mrope":
        qkv = rnd(T, qkvc)
        cs = torch.rand((T, hd // 2, 2), generator=g, device=dev, dtype=torch.float32)
        base = qkv.data_ptr()

        def launch():
            L.cosmot_mrope_apply(base, qkvc, H, base + 2 * H * hd, qkvc, Hkv, T, hd, cs.data_ptr(), sh)
        work, unit, peak = 4 * T * (H + Hkv) * hd + T * (hd // 2) * 8, "GB/s", float(peaks["hbm_gbs"])
    elif args.micro == "euler":
        x = rnd(T, d)
        v = rnd(T, d)

        def launch():
            L.cosmot_flow_euler_step(x.data_ptr(), d, v.data_ptr(), d, 0, T, d, 1.0, 0.97, sh)
        work, unit, peak = 6 * T * d, "GB/s", float(peaks["hbm_gbs"])
    else:
        h = rnd(T, d)
        gg = rnd(d, std=0.02) + 1
        out = torch.empty_like(h)
        segs = [(0, n_ar, 0, 0), (n_ar, T, n_ar, 1)]

        def launch():
            L.cosmot_rmsnorm_routed(h.data_ptr(), d, segs, gg.data_ptr(), gg.data_ptr(), d, 1e-6, out.data_ptr(), d,
                                    sh)
        work, unit, peak = 4 * T * d, "GB/s", float(peaks["hbm_gbs"])

    ms, med = time_launch(launch)
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    achieved = work / (ms / 1e3) / scale
    extra = {}
    if args.micro == "attention" and kv_split > 1:
        ms_plain, _ = time_launch(launch_plain)
        extra = {"kv_split": kv_split, "ms_unsplit": ms_plain,
                 "achieved_unsplit": round(work / (ms_plain / 1e3) / scale, 1)}
    print(json.dumps({"micro": args.micro, "workload": wl.name, "tokens": T, "ms": ms, "median_ms": med,
                      "achieved": round(achieved, 1),
                      "unit": unit, "peak": peak, "frac": round(achieved / peak, 3),
                      "peak_source": f"{peak_src} burst", "algorithmic_per_launch": work,
                      "steps": args.steps, "warmup": args.warmup, **extra}), flush=True)


def main():
    args = parse_args()
    wl = synth.preset(args.workload)
    if args.micro:
        run_micro(args, wl)
        return
    if args.impl == "reference":
        run_reference(args, resolve_schedule(wl, use_oracle=True))
    else:
        run_native(args, resolve_schedule(wl, use_oracle=False))


if __name__ == "__main__":
    main()
