"""Benchmark of the VideoMLA latent-attention layer step on B200.

One step = one streaming chunk of one Wan-1.3B-shaped layer through the whole path:
compress + 3D-RoPE + ring append (4680 tokens), absorbed query, latent attention of 4680 x 12 query
rows against the full 21-frame window (32760 cached tokens), and the value up-projection.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B] [--impl reference]

Prints one JSON line (rank 0).  ``value`` is latent-attention TFLOP/s: 2*B*H*Nq*Nk*(2*d_c + d_rope)
algorithmic flops per step, the whole step timed on the device with CUDA events, summed over ranks
(each rank runs its own batch: weak scaling).  No step finds the previous one's data in L2:
- by default consecutive steps cycle over 10 layer caches and 4 input sets, 262 MB at B = 1, more
  than the 126 MB L2, as consecutive layers of a rollout do;
- with ``--l2 flush`` one cache is used, with a 512 MB write between steps.
``--impl reference`` times the float64 CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

from rank_latent_kv_vmla_b200.config import WAN

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
N_INPUT_SETS = 4          # distinct x / q sets cycled through the steps (all resident in HBM)
E2E_LAYERS = 10          # layer caches the end-to-end run cycles over
FLUSH_BYTES = 512 << 20   # > 126 MB L2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--batch", type=int, default=1, help="sequences per GPU")
    ap.add_argument("--impl", default="vmla", choices=["vmla", "reference"])
    ap.add_argument("--no-dense", action="store_true", help="skip the dense MHA comparison arm")
    ap.add_argument("--parallel", default="batch", choices=["batch", "query"],
                    help="batch: each rank runs its own sequences (weak scaling, no collective); query: one "
                         "batch whose chunk query rows are sharded over the ranks, each holding a replica of "
                         "the latent cache that every rank's compress kernel writes (strong scaling)")
    ap.add_argument("--nvtx", action="store_true",
                    help="mark every timed step and each of its calls with an NVTX range (for Nsight Systems)")
    ap.add_argument("--l2", default="rotate", choices=["rotate", "flush"],
                    help="rotate: consecutive steps use different layer caches (10 x 14.7 MB at B = 1) and input "
                         "sets, more than L2, as consecutive layers of a rollout do; flush: one cache, and a "
                         "512 MB write between steps")
    ap.add_argument("--path", default="fused", choices=["fused", "three"],
                    help="fused: compress + one fused attention launch per step; three: compress + "
                         "absorb + attention + value-up launches (the other path is timed beside it)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sustained-seconds", type=float, default=1.2,
                    help="length of the sustained leg (the step back to back; 0 leaves it out)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--workload", default="layer", choices=["layer", "batch8", "dc_sweep", "rollout", "fewstep",
                                                            "capacity"],
                    help="layer: the headline line; the others print a measurement line of their own")
    return ap.parse_args()


# ------------------------------------------------------------------------------------------------
# Workload arithmetic
# ------------------------------------------------------------------------------------------------
def attention_flops(cfg, batch) -> float:
    """Algorithmic flops of one latent-attention call: 2*B*H*Nq*Nk*(2*d_c + d_rope)."""
    return 2.0 * batch * cfg.n_heads * cfg.chunk_tokens * cfg.window_tokens * (2 * cfg.d_c + cfg.d_rope)


def dense_attention_flops(cfg, batch) -> float:
    return 2.0 * batch * cfg.n_heads * cfg.chunk_tokens * cfg.window_tokens * (cfg.d_h + cfg.d_v)


def kernel_bytes(cfg, batch):
    """Algorithmic HBM bytes per launch of the HBM-bound steps (bf16)."""
    e = 2
    nq, H = cfg.chunk_tokens, cfg.n_heads
    return {
        "compress_append": batch * nq * (cfg.dim + cfg.d_c + cfg.d_rope) * e + (cfg.d_c + cfg.d_rope) * cfg.dim * e,
        "absorb_q": batch * nq * H * (cfg.d_nope + cfg.d_rope + cfg.d_qk) * e + H * cfg.d_nope * cfg.d_c * e,
        "value_up": batch * nq * H * (cfg.d_c + cfg.d_v) * e + H * cfg.d_v * cfg.d_c * e,
    }


def projection_flops(cfg, batch) -> float:
    """Flops of the two per-head projections the fused kernel also performs:
    2*B*Nq*H*(d_nope*d_c + d_c*d_v)."""
    return 2.0 * batch * cfg.chunk_tokens * cfg.n_heads * (cfg.d_nope * cfg.d_c + cfg.d_c * cfg.d_v)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def traffic_for(kernel: str, source_hash: str):
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        ent = t.get(kernel)
        if ent and ent.get("source_hash") == source_hash:
            return ent.get("bytes_per_launch")
    except Exception:
        pass
    return None


def source_hash(names):
    """Hash of the kernel sources' code: comments and blank space removed, so that only a change of
    the code itself marks a recorded ncu traffic figure as stale."""
    import hashlib
    import re
    h = hashlib.sha256()
    for n in names:
        p = os.path.join(ROOT, "rank_latent_kv_vmla_b200", "csrc", n)
        if os.path.exists(p):
            text = open(p, encoding="utf-8").read()
            text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)      # block comments
            text = re.sub(r"//[^\n]*", " ", text)                     # line comments
            h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ------------------------------------------------------------------------------------------------
_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def gpu_bus_id(cuda_index: int):
    """PCI bus id of a CUDA device, as NVML and nvidia-smi name it (CUDA and NVML may order devices
    differently); None if torch does not report it."""
    try:
        pr = torch.cuda.get_device_properties(cuda_index)
        return "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi every 100 ms in a child process: the clocks line of the whole measured run (timed
    region, interleaved path comparison, end-to-end leg, sustained leg)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_bus_id(gpu_index) or str(gpu_index)
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    @staticmethod
    def _parse(lines):
        sm, smax, reasons = [], None, set()
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(_REASONS, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return sm, smax, reasons

    def snapshot(self):
        """One blocking nvidia-smi sample (parsed), or None."""
        try:
            r = subprocess.run(["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                                "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=20)
            sm, smax, reasons = self._parse(r.stdout.splitlines())
            return {"sm_mhz": sm[0], "sm_max_mhz": smax, "reasons": sorted(reasons)} if sm else None
        except Exception:
            return None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = self._parse(open(self.path))
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi every 100 ms"}


class NvmlSampler:
    """SM clock and clock-event reasons read through NVML every ``period_s`` by a host thread, so that
    even a timed region of a few tens of milliseconds holds samples.  mark() opens a named window;
    window(name) summarises the samples taken in it."""
    _BITS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
             "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, cuda_index: int, period_s: float = 0.002):
        import threading
        self.period = period_s
        self.samples = []             # (t, sm_mhz, reasons bitmask)
        self.marks = {}
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            bus = gpu_bus_id(cuda_index)
            self.h = (pynvml.nvmlDeviceGetHandleByPciBusId(bus) if bus
                      else pynvml.nvmlDeviceGetHandleByIndex(cuda_index))
            self.nv = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.nv = None

    def start(self):
        if self.nv is None:
            return
        import threading

        def loop():
            nv, h = self.nv, self.h
            while not self._stop.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((time.perf_counter(), float(mhz), int(rs)))
                except Exception:
                    pass
                time.sleep(self.period)
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def mark(self, name: str, end: bool = False):
        self.marks.setdefault(name, [None, None])[1 if end else 0] = time.perf_counter()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def window(self, name: str):
        t0, t1 = self.marks.get(name, (None, None))
        if t0 is None or t1 is None:
            return None
        got = [(mhz, rs) for t, mhz, rs in self.samples if t0 <= t <= t1]
        if not got:
            return None
        reasons = sorted(n for n, bit in self._BITS.items() if any(rs & bit for _, rs in got))
        return {"sm_mhz": statistics.median(m for m, _ in got), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(got), "source": "NVML every %g ms" % (1e3 * self.period)}


# ------------------------------------------------------------------------------------------------
# Distributed plumbing (one process per GPU; timing collective only)
# ------------------------------------------------------------------------------------------------
def dist_setup(backend: str = "nccl"):
    """One process per GPU (torchrun env).  Returns (rank, world, local_rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ["RANK"])
        local = int(os.environ.get("LOCAL_RANK", rank))
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return rank, world, local
    return 0, 1, 0


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """Largest value over all ranks (the timing collective: every rank calls it once per region)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of a rank's inputs: the headline layer's seed for rank 0, distinct per rank."""
    return 1234 + 1 + 1000 * rank


def whole_job_rate(work_per_step: float, steps: int, world: int, max_total_ms: float) -> float:
    """Work of all ranks (each rank runs its own batch) per second of the slowest rank."""
    return world * work_per_step * steps / (max_total_ms * 1e-3)


# ------------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and --impl reference)
# ------------------------------------------------------------------------------------------------
class OracleStep:
    """The float64 oracle on a bounded sample of one layer step: a full 21-frame window is built once
    (untimed); a timed step compresses ``n_rows`` tokens of the new chunk, absorbs their queries and
    runs latent attention (the plain definition, all heads) and the value up-projection for them."""

    def __init__(self, cfg, seed):
        from oracle import vmla_oracle as O
        import synthetic
        self.O, self.cfg = O, cfg
        n_chunks = cfg.window_frames // cfg.chunk_frames
        inp = synthetic.draw_layer(cfg, batch=1, seed=seed, n_chunks=n_chunks)
        self.pairs = (cfg.rope_pairs_t, cfg.rope_pairs_h, cfg.rope_pairs_w)
        self.w = inp.w_dkv_kr.double().numpy()
        self.w_uk, self.w_uv = inp.w_uk.double().numpy(), inp.w_uv.double().numpy()
        self.x_new = inp.x_chunks[-1][0].double().numpy()
        self.qn, self.qr = inp.q_nope[0].double().numpy(), inp.q_rope[0].double().numpy()
        kw = dict(d_c=cfg.d_c, d_rope=cfg.d_rope, chunk_frames=cfg.chunk_frames, grid_h=cfg.grid_h,
                  grid_w=cfg.grid_w, pairs=self.pairs, theta=cfg.rope_theta)
        hist = O.build_history([x.double().numpy() for x in inp.x_chunks], self.w, 0, **kw)
        self.c, self.k_r, self.frames = hist.c, hist.k_r, hist.frames
        self.f0 = (n_chunks - 1) * cfg.chunk_frames

    def run(self, n_rows: int) -> float:
        """Time the sample; the rows go through the oracle in groups of at most 128 (bounded memory)."""
        rows_all = np.linspace(0, self.cfg.chunk_tokens - 1, n_rows).astype(np.int64)
        return sum(self._run_rows(rows_all[i:i + 128]) for i in range(0, n_rows, 128))

    def _run_rows(self, rows) -> float:
        O, cfg = self.O, self.cfg
        t0 = time.perf_counter()
        pos = O.token_positions(self.f0, cfg.chunk_tokens, cfg.grid_h, cfg.grid_w)[rows]
        O.compress(self.x_new[rows], self.w, cfg.d_c, pos, self.pairs, cfg.rope_theta)
        q_abs = O.absorbed_query(self.qn[rows], O.rotate_query(self.qr[rows], pos, self.pairs, cfg.rope_theta),
                                 self.w_uk)
        hi = O.query_chunk_end(self.f0, cfg.chunk_tokens, cfg.chunk_frames, cfg.tokens_per_frame)[rows]
        mask = O.visible(hi, self.frames, cfg.window_frames)
        o_lat, _ = O.latent_attention(q_abs, self.c, self.k_r, mask, cfg.scale)
        O.value_up(o_lat, self.w_uv)
        return time.perf_counter() - t0

    def size_for(self, seconds: float) -> int:
        """Rows whose step takes about `seconds` (linear fit t = a + b*n from two probes)."""
        n1, n2 = 8, 32
        t1, t2 = self.run(n1), self.run(n2)
        b = max((t2 - t1) / (n2 - n1), 1e-6)
        a = max(t1 - b * n1, 0.0)
        return int(min(self.cfg.chunk_tokens, max(1, (seconds - a) / b)))


def _sample_text(cfg, n_rows, t):
    return (f"float64 NumPy oracle, one Wan-1.3B layer step restricted to {n_rows} of {cfg.chunk_tokens} "
            f"query tokens: their compression, absorbed queries, latent attention over the full "
            f"{cfg.window_tokens}-token window (all {cfg.n_heads} heads) and value up-projection; "
            f"{t:.2f} s; value = those rows' latent-attention flops / time")


def cpu_baseline(cfg, target_s):
    cores = len(os.sched_getaffinity(0))
    st = OracleStep(cfg, 4321)
    n_rows = st.size_for(target_s)
    t = st.run(n_rows)
    flops = attention_flops(cfg, 1) * n_rows / cfg.chunk_tokens
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "query_tokens_per_s": n_rows / t, "sample": _sample_text(cfg, n_rows, t)}


def headline_config(cfg, B, world, args) -> dict:
    """The `config` object of the headline line, computed from the shapes and arguments alone, so that
    the GPU arm and the reference arm print the same one."""
    rotate, fused = args.l2 == "rotate", args.path == "fused"
    cache_mb = E2E_LAYERS * B * cfg.window_tokens * cfg.d_qk * 2 / 1e6
    inputs_mb = N_INPUT_SETS * 2 * B * cfg.chunk_tokens * (cfg.dim + cfg.n_heads * (cfg.d_nope + cfg.d_rope)) / 1e6
    return {"workload": "wan1.3b_layer_stream_step", "batch_per_gpu": B, "global_batch": B * world,
            "query_tokens": cfg.chunk_tokens, "cached_tokens": cfg.window_tokens,
            "heads": cfg.n_heads, "d_c": cfg.d_c, "d_rope": cfg.d_rope, "d_v": cfg.d_v,
            "dim": cfg.dim, "parallelism": f"dp{world} (independent sequences)",
            "l2": ("inputs larger than L2: steps cycle over %d layer caches (%.0f MB) and %d input sets (%.0f MB)"
                   % (E2E_LAYERS, cache_mb, N_INPUT_SETS, inputs_mb) if rotate
                   else "flushed between steps (512 MB write)"),
            "path": ("compress + fused absorb/attention/value-up" if fused
                     else "compress + absorb + attention + value-up")}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = WAN
    cores = len(os.sched_getaffinity(0))
    st = OracleStep(cfg, 4321)
    budget = 150.0                      # seconds for all warm-up + timed steps
    per_step = min(5.0, budget / max(1, args.steps + args.warmup))
    n_rows = st.size_for(per_step)
    for _ in range(args.warmup):
        st.run(n_rows)
    times = [st.run(n_rows) for _ in range(args.steps)]
    t = sum(times)
    flops = attention_flops(cfg, 1) * n_rows / cfg.chunk_tokens * args.steps
    val = flops / t / 1e12
    line = {"metric": "latent-attention TFLOP/s (Wan-1.3B layer step, B200 BF16 TC peak fraction)",
            "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": headline_config(cfg, args.batch, args.gpus, args),
            "impl": "reference",
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": _sample_text(cfg, n_rows, t / args.steps) + " (per step)"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------
def _time(fn, reps, stream):
    """Mean device time (ms) of fn() over reps calls, CUDA events around each, L2 not flushed."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def _time_pair(fa, fb, reps, stream):
    """Median device times (ms) of fa() and fb(), reps calls each, interleaved a, b, b, a, ... so that
    both see the same clock and power state."""
    res = ([], [])
    for i in range(2 * reps):
        k = 0 if (i % 4) in (0, 3) else 1
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        (fa, fb)[k]()
        b.record(stream)
        res[k].append((a, b))
    torch.cuda.synchronize()
    return tuple(statistics.median(a.elapsed_time(b) for a, b in r) for r in res)


def _fewstep_workload(V, synthetic, dev, stream, clocks, batch=1, n_chunks=14, n_denoise=4):
    """One Wan layer streaming n_chunks chunks, each denoised over n_denoise steps: the first step
    appends the chunk, the others rewrite it in place; every step attends with its own queries
    (latent: compress -> fused absorb / attention / value-up; dense: project -> rope -> MHA)."""
    cfg, B = WAN, batch
    sets = [tuple(t.to(dev) for t in synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(11, 0, k)))
            for k in range(n_denoise)]
    wd, wuk, wuv = (t.to(dev) for t in synthetic.draw_weights(cfg, 12))
    w_kv = synthetic.draw_dense_weights(cfg, 13).to(dev)
    o = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)
    dq = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_h), dtype=torch.bfloat16, device=dev)
    res = {}
    clocks.start()
    # the two layers step in lockstep, alternating which goes first, so that both see the same clock
    caches = {"latent": V.LatentCache(cfg, B, device=dev), "dense": V.DenseCache(cfg, B, device=dev)}
    f0 = {"latent": 0, "dense": 0}
    evs = {"latent": [], "dense": []}

    def one(path, k, s):
        x, qn, qr = sets[s]
        cache = caches[path]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if s == 0:
            f0[path] = cache.frames_written
        if path == "latent":
            if s == 0:
                V.compress_append(cfg, x, wd, cache)
            else:
                V.compress_rewrite(cfg, x, wd, cache)
            V.latent_attention_fused(cfg, qn, qr, wuk, wuv, cache, f0[path], out=o)
        else:
            if s == 0:
                V.dense_append(cfg, x, w_kv, cache)
            else:
                V.dense_rewrite(cfg, x, w_kv, cache)
            V.rope_q(cfg, qn, qr, f0[path], out=dq)
            V.dense_mha(cfg, dq, cache, f0[path], out=o)
        b.record(stream)
        evs[path].append((k, a, b))

    for k in range(n_chunks):
        for s in range(n_denoise):
            for path in (("latent", "dense") if (k * n_denoise + s) % 2 == 0 else ("dense", "latent")):
                one(path, k, s)
    torch.cuda.synchronize()
    for path in ("latent", "dense"):
        # steady state: chunks whose window is full (frame f0 + F >= W)
        full = [a.elapsed_time(b) for k, a, b in evs[path] if (k + 1) * cfg.chunk_frames >= cfg.window_frames]
        ms = statistics.mean(full)
        fl = attention_flops(cfg, B) if path == "latent" else dense_attention_flops(cfg, B)
        res[path] = {"ms_per_denoising_step": ms, "attention_tflops_per_step_time": fl / (ms * 1e-3) / 1e12,
                     "steps_timed": len(full), "total_ms_all_steps": sum(a.elapsed_time(b) for _, a, b in evs[path])}
    del caches
    torch.cuda.empty_cache()
    res["step_time_ratio_latent_over_dense"] = res["latent"]["ms_per_denoising_step"] / res["dense"]["ms_per_denoising_step"]
    return {"batch": B, "chunks": n_chunks, "denoising_steps_per_chunk": n_denoise, **res}


def _capacity_workload(V, synthetic, dev, clocks, budget=60 * 10**9, n_layers=30):
    """Largest batch for 30 Wan layers under a 60 GB budget, latent (d_c 64 / 128 / 192) and dense,
    from the planner; for d_c = 192 and dense the planned caches of all layers are then allocated and
    one layer step runs at that batch, with the device's peak allocation recorded."""
    rows = []
    clocks.start()
    for name, cfg, dense in (("latent_dc64", WAN.replace(d_c=64), False),
                             ("latent_dc128", WAN.replace(d_c=128), False),
                             ("latent_dc192", WAN, False), ("dense", WAN, True)):
        # the latent step runs fused where the fused kernel supports the shape
        fused = (not dense) and V.fused_supported(cfg)
        plan = V.plan_capacity(cfg, n_layers, budget, dense=dense, fused=fused)
        row = {"path": name + ("_fused" if fused else ""), **plan}
        if name in ("latent_dc192", "dense"):
            B = plan["max_batch"]
            torch.cuda.empty_cache()
            torch.cuda.reset_peak_memory_stats()
            x, qn, qr = (t.to(dev) for t in synthetic.draw_chunk(cfg, B, 21))
            if dense:
                w_kv = synthetic.draw_dense_weights(cfg, 22).to(dev)
                caches = [V.DenseCache(cfg, B, device=dev) for _ in range(n_layers)]
                ws = [w_kv] * n_layers
            else:
                wd, wuk, wuv = (t.to(dev) for t in synthetic.draw_weights(cfg, 22))
                caches = [V.LatentCache(cfg, B, device=dev) for _ in range(n_layers)]
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record()
            if dense:
                V.dense_append(cfg, x, w_kv, caches[0])
                out = V.dense_mha(cfg, V.rope_q(cfg, qn, qr, 0), caches[0], 0)
            else:
                out = V.layer_step(cfg, x, qn, qr, wd, wuk, wuv, caches[0])
            t1.record()
            torch.cuda.synchronize()
            row.update({"allocated_batch": B, "peak_allocated_bytes": torch.cuda.max_memory_allocated(),
                        "one_layer_step_ms": t0.elapsed_time(t1), "output_finite": bool(torch.isfinite(out).all())})
            del caches, out, x, qn, qr
            torch.cuda.empty_cache()
        rows.append(row)
    by = {r["path"].replace("_fused", ""): r["max_batch"] for r in rows}
    return {"budget_bytes": budget, "n_layers": n_layers, "rows": rows,
            "batch_ratio_dc192_over_dense": by["latent_dc192"] / max(by["dense"], 1),
            "batch_ratio_dc64_over_dense": by["latent_dc64"] / max(by["dense"], 1)}


def run_workload(args):
    """Measurement lines for the larger workloads (not the headline): batch-8 latent vs dense,
    the d_c sweep at batch 16, the 30-layer x 80-chunk streaming rollout at batch 4, few-step
    generation (4 denoising steps per chunk) and the batch capacity at a 60 GB budget."""
    from rank_latent_kv_vmla_b200 import vmla as V
    import synthetic
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    out = {"workload": args.workload, "device": torch.cuda.get_device_name(0)}
    clocks = ClockSampler(0)
    if args.workload in ("batch8", "dc_sweep"):
        B = 8 if args.workload == "batch8" else 16
        dcs = [192] if args.workload == "batch8" else [64, 128, 192]
        rows = []
        clocks.start()
        # the dense MHA layer (per-head K, V: independent of d_c) on the same shapes and batch, timed
        # interleaved with each latent call
        inp_d = synthetic.draw_layer(WAN, batch=B, seed=1234 + 2, n_chunks=7)
        w_kv = synthetic.draw_dense_weights(WAN, 77).to(dev)
        dcache = V.DenseCache(WAN, B, device=dev)
        for x in inp_d.x_chunks:
            fd = dcache.frames_written
            V.dense_append(WAN, x.to(dev), w_kv, dcache)
        q_d = V.rope_q(WAN, inp_d.q_nope.to(dev), inp_d.q_rope.to(dev), fd)
        o_d = torch.empty((B, WAN.chunk_tokens, WAN.n_heads, WAN.d_v), dtype=torch.bfloat16, device=dev)
        dense_call = lambda: V.dense_mha(WAN, q_d, dcache, fd, out=o_d)
        for _ in range(3):
            dense_call()
        del inp_d
        for d_c in dcs:
            cfg = WAN.replace(d_c=d_c)
            inp = synthetic.draw_layer(cfg, batch=B, seed=1234 + 2, n_chunks=7)
            cache = V.LatentCache(cfg, B, device=dev)
            w = inp.w_dkv_kr.to(dev)
            for x in inp.x_chunks:
                f0 = cache.frames_written
                V.compress_append(cfg, x.to(dev), w, cache)
            qn, qr, wuk = inp.q_nope.to(dev), inp.q_rope.to(dev), inp.w_uk.to(dev)
            q_abs = V.absorb_q(cfg, qn, qr, wuk, f0)
            o_lat = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_c), dtype=torch.bfloat16, device=dev)
            lat_call = lambda: V.latent_attention(cfg, q_abs, cache, f0, out=o_lat)
            for _ in range(3):
                lat_call()
            # throughput: the latent calls timed on their own; comparison: each interleaved with the
            # dense call (the dense kernel draws less power, so alternating with it changes the clock)
            ms = _time(lat_call, 20, stream)
            ms_i, dms_a = _time_pair(lat_call, dense_call, 10, stream)
            row = {"d_c": d_c, "batch": B, "latent_attention_ms": ms,
                   "latent_tflops": attention_flops(cfg, B) / (ms * 1e-3) / 1e12,
                   "query_tokens_per_s": B * cfg.chunk_tokens / (ms * 1e-3),
                   "cache_bytes_per_layer": V.latent_cache_bytes(cfg, B),
                   "cache_fraction_of_dense": V.latent_cache_bytes(cfg, B) / V.dense_cache_bytes(cfg, B),
                   "interleaved": {"latent_attention_ms": ms_i, "dense_mha_ms": dms_a},
                   "attention_alone_ratio_latent_over_dense": ms_i / dms_a}
            ms, dms = ms_i, dms_a
            if V.fused_supported(cfg):
                # the fused call: absorb + attention + value-up in one launch (what the layer step runs)
                wuv = inp.w_uv.to(dev)
                o_f = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)
                fused_call = lambda: V.latent_attention_fused(cfg, qn, qr, wuk, wuv, cache, f0, out=o_f)
                for _ in range(3):
                    fused_call()
                fms_alone = _time(fused_call, 20, stream)
                fms, dms = _time_pair(fused_call, dense_call, 10, stream)
                row.update({"fused_ms": fms_alone,
                            "fused_attention_tflops": attention_flops(cfg, B) / (fms_alone * 1e-3) / 1e12})
                row["interleaved"].update({"fused_ms": fms, "dense_mha_ms_with_fused": dms})
                ms = fms
            row.update({"dense_mha_ms": dms, "dense_tflops": dense_attention_flops(cfg, B) / (dms * 1e-3) / 1e12,
                        "attention_time_ratio_latent_over_dense": ms / dms,
                        "ratio_uses": "fused call (absorb + attention + value-up) vs dense MHA, interleaved",
                        "dense_cache_bytes_per_layer": V.dense_cache_bytes(cfg, B)})
            rows.append(row)
            del cache
            torch.cuda.empty_cache()
        del dcache
        torch.cuda.empty_cache()
        out["rows"] = rows
    elif args.workload == "fewstep":
        out.update(_fewstep_workload(V, synthetic, dev, stream, clocks))
    elif args.workload == "capacity":
        out.update(_capacity_workload(V, synthetic, dev, clocks))
    else:
        cfg, B, L, n_chunks = WAN, 4, 30, 80
        n_sets = 3
        sets = [tuple(t.to(dev) for t in synthetic.draw_chunk(cfg, B, synthetic.rollout_seed(9, 0, k))) for k in range(n_sets)]
        weights = [tuple(t.to(dev) for t in synthetic.draw_weights(cfg, synthetic.rollout_seed(9, l, -1))) for l in range(L)]
        dense_w = [synthetic.draw_dense_weights(cfg, 500 + l).to(dev) for l in range(L)]
        res = {}
        clocks.start()
        for path in ("latent", "dense"):
            caches = [V.LatentCache(cfg, B, device=dev) if path == "latent" else V.DenseCache(cfg, B, device=dev)
                      for _ in range(L)]
            bufs = {"q_abs": torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_qk), dtype=torch.bfloat16, device=dev),
                    "o_latent": torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_c), dtype=torch.bfloat16, device=dev),
                    "o": torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)}
            dq = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_h), dtype=torch.bfloat16, device=dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(stream)
            for k in range(n_chunks):
                x, qn, qr = sets[k % n_sets]
                for l in range(L):
                    if path == "latent":
                        wd, wuk, wuv = weights[l]
                        V.layer_step(cfg, x, qn, qr, wd, wuk, wuv, caches[l], bufs)
                    else:
                        f0 = caches[l].frames_written
                        V.dense_append(cfg, x, dense_w[l], caches[l], f0)
                        V.rope_q(cfg, qn, qr, f0, out=dq)
                        V.dense_mha(cfg, dq, caches[l], f0, out=bufs["o"])
            b.record(stream)
            torch.cuda.synchronize()
            res[path] = {"total_s": a.elapsed_time(b) / 1e3,
                         "cache_bytes_all_layers": sum(c.nbytes() for c in caches)}
            del caches
            torch.cuda.empty_cache()
        res["speedup_latent_over_dense"] = res["dense"]["total_s"] / res["latent"]["total_s"]
        res["latent"]["attention_tflops"] = attention_flops(cfg, B) * L * n_chunks / res["latent"]["total_s"] / 1e12
        out.update({"layers": L, "chunks": n_chunks, "batch": B, "frames": n_chunks * cfg.chunk_frames, **res})
    out["clocks"] = clocks.stop()
    assert V.device_status() == 0
    print(json.dumps(out), flush=True)


def run_query_sharded(args):
    """--parallel query: one batch of B sequences; every rank compresses and attends its token range of
    each chunk (rank_latent_kv_vmla_b200.sharding).  value = the whole chunk's latent-attention flops per
    second of the slowest rank (strong scaling: the work does not grow with the ranks)."""
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_setup("nccl")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from rank_latent_kv_vmla_b200 import vmla as V
    from rank_latent_kv_vmla_b200.sharding import ShardedLayer, TorchComm
    import synthetic
    cfg, B = WAN, args.batch
    pk, pk_src = peaks()
    seed = rank_seed(0)                                   # every rank draws the same sequence
    prefill = cfg.window_frames // cfg.chunk_frames - 1
    inp = synthetic.draw_layer(cfg, batch=B, seed=seed, n_chunks=prefill + N_INPUT_SETS)
    extra_q = [synthetic.draw_queries(cfg, B, seed + 7 + i) for i in range(N_INPUT_SETS)]
    w, w_uk, w_uv = inp.w_dkv_kr.to(dev), inp.w_uk.to(dev), inp.w_uv.to(dev)
    comm = TorchComm(device=dev)
    layer = ShardedLayer(cfg, B, comm, device=dev)
    b0, cnt = layer.begin, layer.count
    rows = lambda t: t[:, b0:b0 + cnt].contiguous().to(dev)
    xs = [rows(x) for x in inp.x_chunks]
    qs = [(rows(qn), rows(qr)) for qn, qr in extra_q]
    out = torch.empty((B, max(cnt, 1), cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)[:, :cnt]
    for k in range(prefill):
        layer.step(xs[k], qs[0][0], qs[0][1], w, w_uk, w_uv, out=out if cnt else None)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        j = i % N_INPUT_SETS
        if ev: ev[0].record(stream)
        layer.step(xs[prefill + j], qs[j][0], qs[j][1], w, w_uk, w_uv, out=out if cnt else None)
        if ev: ev[1].record(stream)

    for i in range(args.warmup):
        step(i)
        flush.zero_()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    launches0 = V.launch_count()
    for i in range(args.steps):
        step(args.warmup + i, evs[i])
        flush.zero_()
    torch.cuda.synchronize()
    launches = V.launch_count() - launches0
    clk = clocks.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world)
    assert V.device_status() == 0
    layer.close()
    f_step = attention_flops(cfg, B)
    value = f_step * args.steps / (total_ms * 1e-3) / 1e12
    if rank == 0:
        line = {"metric": "latent-attention TFLOP/s (Wan-1.3B layer step, B200 BF16 TC peak fraction)",
                "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "wan1.3b_layer_stream_step", "batch": B, "query_tokens": cfg.chunk_tokens,
                           "cached_tokens": cfg.window_tokens, "heads": cfg.n_heads, "d_c": cfg.d_c,
                           "parallelism": f"query rows sharded over {world} GPUs, latent cache replicated",
                           "shards": layer.shards, "l2": "flushed between steps (512 MB write)"},
                "query_tokens_per_s": B * cfg.chunk_tokens * args.steps / (total_ms * 1e-3),
                "pct_of_bf16_peak": 100.0 * value / world / pk["bf16_tflops"],
                "gpu_launches": launches, "clocks": clk, "e2e": None, "cpu_baseline": None}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload != "layer":
        return run_workload(args)
    if args.parallel == "query":
        return run_query_sharded(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_setup("nccl")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from rank_latent_kv_vmla_b200 import vmla as V
    import synthetic

    cfg = WAN
    B = args.batch
    pk, pk_src = peaks()
    seed = rank_seed(rank)
    prefill = cfg.window_frames // cfg.chunk_frames - 1          # 6 chunks: frames 0..17
    inp = synthetic.draw_layer(cfg, batch=B, seed=seed, n_chunks=prefill + N_INPUT_SETS)
    extra_q = [synthetic.draw_queries(cfg, B, seed + 7 + i) for i in range(N_INPUT_SETS)]
    w = inp.w_dkv_kr.to(dev)
    w_uk, w_uv = inp.w_uk.to(dev), inp.w_uv.to(dev)
    xs = [x.to(dev) for x in inp.x_chunks[prefill:]]
    qs = [(qn.to(dev), qr.to(dev)) for qn, qr in extra_q]
    # the layer caches the steps cycle over: E2E_LAYERS of them (147 MB at B = 1, with the 115 MB of input
    # sets more than L2, so no step finds the previous step's data in L2), or one with --l2 flush
    rotate = args.l2 == "rotate"
    caches = []
    for _ in range(E2E_LAYERS if rotate else 1):
        c1 = V.LatentCache(cfg, B, device=dev)
        for x in inp.x_chunks[:prefill]:
            V.compress_append(cfg, x.to(dev), w, c1)
        caches.append(c1)
    cache = caches[0]
    bufs = {"q_abs": torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_qk), dtype=torch.bfloat16, device=dev),
            "o_latent": torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_c), dtype=torch.bfloat16, device=dev),
            "o": torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)}
    flush = None if rotate else torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def between_steps():
        if flush is not None:
            flush.zero_()

    fused = args.path == "fused"
    names = (["compress_append", "latent_attention_fused"] if fused else
             ["compress_append", "absorb_q", "latent_attention", "value_up"])
    n_ev = len(names) + 1

    nvtx = torch.cuda.nvtx if args.nvtx else None

    def mark(name):
        if nvtx is not None:
            nvtx.range_pop()
            nvtx.range_push(name)

    def step(i, ev=None, x=None, qn=None, qr=None, use_fused=fused):
        if nvtx is not None:
            nvtx.range_push(f"step {i}")
            nvtx.range_push("compress_append")
        try:
            _step(i, ev, x, qn, qr, use_fused)
        finally:
            if nvtx is not None:
                nvtx.range_pop()
                nvtx.range_pop()

    def _step(i, ev, x, qn, qr, use_fused):
        x = xs[i % N_INPUT_SETS] if x is None else x
        if qn is None:
            qn, qr = qs[i % N_INPUT_SETS]
        cache = caches[i % len(caches)]
        f0 = cache.frames_written
        if ev: ev[0].record(stream)
        V.compress_append(cfg, x, w, cache, f0)
        if ev: ev[1].record(stream)
        if use_fused:
            mark("latent_attention_fused")
            V.latent_attention_fused(cfg, qn, qr, w_uk, w_uv, cache, f0, out=bufs["o"])
            if ev: ev[2].record(stream)
            return
        mark("absorb_q")
        V.absorb_q(cfg, qn, qr, w_uk, f0, out=bufs["q_abs"])
        if ev: ev[2].record(stream)
        mark("latent_attention")
        V.latent_attention(cfg, bufs["q_abs"], cache, f0, out=bufs["o_latent"])
        if ev: ev[3].record(stream)
        mark("value_up")
        V.value_up(cfg, bufs["o_latent"], w_uv, out=bufs["o"])
        if ev: ev[4].record(stream)

    for i in range(args.warmup):
        step(i)
        between_steps()
    torch.cuda.synchronize()
    assert V.device_status() == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    clocks = ClockSampler(local)          # 100 ms samples over the timed region and every leg after it
    nvml = NvmlSampler(local)             # 2 ms samples: the timed region itself may last only ~20 ms
    nvml.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    launches0 = V.launch_count()
    nvml.mark("timed")
    wall0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i, evs[i])
        between_steps()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    nvml.mark("timed", end=True)
    after_timed = clocks.snapshot()       # one blocking sample right after the timed region
    launches = V.launch_count() - launches0
    barrier(world)
    per_kernel = {n: [evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)] for j, n in enumerate(names)}
    step_ms = [evs[i][0].elapsed_time(evs[i][n_ev - 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(sum(step_ms), world)
    assert V.device_status() == 0

    f_step = attention_flops(cfg, B)
    value = whole_job_rate(f_step, args.steps, world, total_ms) / 1e12
    q_tok_s = whole_job_rate(B * cfg.chunk_tokens, args.steps, world, total_ms)
    kb = kernel_bytes(cfg, B)
    k3 = "latent_attention_fused" if fused else "latent_attention"
    k3_ms = statistics.mean(per_kernel[k3])
    # algorithmic flops of the dominant launch: the attention, plus the two projections when fused
    k3_flops = f_step + (projection_flops(cfg, B) if fused else 0.0)
    k3_tflops = k3_flops / (k3_ms * 1e-3) / 1e12
    kernels = {k3: {"ms": k3_ms, "tflops": k3_tflops, "attention_tflops": f_step / (k3_ms * 1e-3) / 1e12}}
    for n in names:
        if n == k3:
            continue
        ms = statistics.mean(per_kernel[n])
        kernels[n] = {"ms": ms, "gbs": kb[n] / (ms * 1e-3) / 1e9, "frac_hbm": kb[n] / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
        if n == "compress_append":
            # 224 flops per byte of x, near the ridge: at the measured peaks the flops alone take 75 % of
            # the HBM time, so the MMAs must overlap the loads to reach the HBM bound
            fl = 2.0 * B * cfg.chunk_tokens * (cfg.d_c + cfg.d_rope) * cfg.dim
            kernels[n]["tflops"] = fl / (ms * 1e-3) / 1e12
    k3_src = source_hash(["tc_attention.cu", "tc_kernels.cuh", "ptx_sm100.cuh"])
    roofline = {"bound": "tensor", "kernel": k3, "achieved": k3_tflops,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": k3_tflops / pk["bf16_tflops"],
                "peak_source": f"{pk_src} bf16 burst (MEASURED_PEAKS.json)" if pk_src == "measured" else "fallback 1.59 PFLOP/s",
                "frac_of_sustained": k3_tflops / pk["bf16_tflops_sustained"],
                "flops_per_launch": k3_flops,
                "traffic": traffic_for("%s_wan_b%d" % (k3, B), k3_src)}

    # ---- both paths on the same cache and inputs, interleaved step by step so that both see the same
    # clock and power state (not part of `value`) ----
    ab_steps = max(10, args.steps // 8)
    ab = {True: [], False: []}
    for i in range(2 * ab_steps):
        use = (i % 4) in (0, 3)                   # fused, three, three, fused, ...
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        between_steps()
        a.record(stream)
        step(args.warmup + args.steps + i, use_fused=use)
        b.record(stream)
        ab[use].append((a, b))
    torch.cuda.synchronize()
    path_ab = {"fused_step_ms": statistics.median(a.elapsed_time(b) for a, b in ab[True]),
               "three_call_step_ms": statistics.median(a.elapsed_time(b) for a, b in ab[False]),
               "steps_each": ab_steps}
    path_ab["fused_over_three"] = path_ab["fused_step_ms"] / path_ab["three_call_step_ms"]

    # ---- end to end through the public API with host buffers (pinned): the streaming executor, which
    # overlaps each step's host -> device and device -> host copies with the neighbouring steps'
    # kernels.  Steps cycle over E2E_LAYERS layer caches (147 MB with the inputs' staging: more than
    # L2, so no flush is needed between steps) ----
    e_caches = list(caches)
    while len(e_caches) < E2E_LAYERS:
        c2 = V.LatentCache(cfg, B, device=dev)
        for x in inp.x_chunks[:prefill]:
            V.compress_append(cfg, x.to(dev), w, c2)
        e_caches.append(c2)
    hx = [x.cpu().pin_memory() for x in xs]
    hq = [(qn.cpu().pin_memory(), qr.cpu().pin_memory()) for qn, qr in qs]
    ho = [torch.empty(bufs["o"].shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = hx[0].numel() * 2 + hq[0][0].numel() * 2 + hq[0][1].numel() * 2
    d2h = ho[0].numel() * 2
    e2e_steps = max(20, args.steps // 4)
    with V.Executor(cfg, B, device=dev) as ex:
        def e2e_run(n):
            for i in range(n):
                j = i % N_INPUT_SETS
                ex.submit(e_caches[i % E2E_LAYERS], w, w_uk, w_uv, hx[j], hq[j][0], hq[j][1], ho[i % 2])
            ex.wait()
        e2e_run(4)
        torch.cuda.synchronize()
        barrier(world)
        t0 = time.perf_counter()
        e2e_run(e2e_steps)
        e2e_ms = (time.perf_counter() - t0) * 1e3
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e = {"value": world * f_step * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": e2e_ms / e2e_steps,
           "how": f"vmla_executor, {e2e_steps} steps over {E2E_LAYERS} layer caches, host wall clock from "
                  "the first submit to the last output in host memory, max over ranks"}
    del e_caches

    # ---- sustained: the same step back to back for at least a second (not part of `value`): a long
    # run settles at the clock the 1 kW power cap allows, below the burst clock of a short one ----
    sus_steps = (int(min(20000, max(200, math.ceil(args.sustained_seconds * 1e3 / statistics.mean(step_ms)))))
                 if args.sustained_seconds > 0 else 0)
    sus_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(sus_steps)]
    torch.cuda.synchronize()
    nvml.mark("sustained")
    for i in range(sus_steps):
        step(args.warmup + args.steps + 2 * ab_steps + i, sus_ev[i])
        between_steps()
    torch.cuda.synchronize()
    nvml.mark("sustained", end=True)
    sus_step = [sus_ev[i][0].elapsed_time(sus_ev[i][n_ev - 1]) for i in range(sus_steps)] or [float("nan")]
    sus_k3 = statistics.mean([sus_ev[i][names.index(k3)].elapsed_time(sus_ev[i][names.index(k3) + 1])
                              for i in range(sus_steps)] or [float("nan")])
    sustained = None if not sus_steps else {"steps": sus_steps, "seconds": sum(sus_step) / 1e3, "ms_per_step": statistics.mean(sus_step),
                 "tflops": f_step / (statistics.mean(sus_step) * 1e-3) / 1e12,
                 "dominant_kernel_ms": sus_k3, "dominant_kernel_tflops": k3_flops / (sus_k3 * 1e-3) / 1e12,
                 "frac_of_burst_peak": k3_flops / (sus_k3 * 1e-3) / 1e12 / pk["bf16_tflops"],
                 "frac_of_sustained_peak": k3_flops / (sus_k3 * 1e-3) / 1e12 / pk["bf16_tflops_sustained"],
                 "clocks": nvml.window("sustained")}
    assert V.device_status() == 0

    # ---- dense per-head MHA comparison on the same shapes (not part of `value`): dense and latent steps
    # interleaved (latent, dense, dense, latent, ...) so that both see the same clock and power state;
    # each arm's median over its steps ----
    comparison = None
    if not args.no_dense:
        w_kv = synthetic.draw_dense_weights(cfg, seed + 3).to(dev)
        dcache = V.DenseCache(cfg, B, device=dev)
        for x in inp.x_chunks[:prefill]:
            V.dense_append(cfg, x.to(dev), w_kv, dcache)
        dq = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_h), dtype=torch.bfloat16, device=dev)
        do = torch.empty((B, cfg.chunk_tokens, cfg.n_heads, cfg.d_v), dtype=torch.bfloat16, device=dev)
        dsteps = max(10, args.steps // 4)

        def dstep(i, ev):
            f0 = dcache.frames_written
            ev[0].record(stream)
            V.dense_append(cfg, xs[i % N_INPUT_SETS], w_kv, dcache, f0)
            ev[1].record(stream)
            V.rope_q(cfg, qs[i % N_INPUT_SETS][0], qs[i % N_INPUT_SETS][1], f0, out=dq)
            ev[2].record(stream)
            V.dense_mha(cfg, dq, dcache, f0, out=do)
            ev[3].record(stream)

        # the dense cache (201 MB per sequence) alone exceeds L2
        warm = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        for i in range(3):
            dstep(i, warm)
            between_steps()
        lat0 = args.warmup + args.steps + 2 * ab_steps + sus_steps
        d_ev, l_ev = [], []
        for i in range(2 * dsteps):
            if (i % 4) in (0, 3):
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
                step(lat0 + i, ev)
                l_ev.append(ev)
            else:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
                dstep(i, ev)
                d_ev.append(ev)
            between_steps()
        torch.cuda.synchronize()
        d_step_ms = statistics.median(ev[0].elapsed_time(ev[3]) for ev in d_ev)
        d_mha_ms = statistics.median(ev[2].elapsed_time(ev[3]) for ev in d_ev)
        l_step_ms = statistics.median(ev[0].elapsed_time(ev[n_ev - 1]) for ev in l_ev)
        k3i = names.index(k3)
        l_k3_ms = statistics.median(ev[k3i].elapsed_time(ev[k3i + 1]) for ev in l_ev)
        comparison = {"dense_step_ms": d_step_ms, "dense_mha_ms": d_mha_ms,
                      "dense_mha_tflops": dense_attention_flops(cfg, B) / (d_mha_ms * 1e-3) / 1e12,
                      "latent_step_ms": l_step_ms, "latent_attention_ms": l_k3_ms,
                      "latent_attention_includes_projections": fused,
                      "step_speedup_vs_dense": d_step_ms / l_step_ms,
                      "attention_speedup_vs_dense": d_mha_ms / l_k3_ms,
                      "how": f"{dsteps} dense and {dsteps} latent steps interleaved, medians",
                      "cache_bytes_latent": V.latent_cache_bytes(cfg, B),
                      "cache_bytes_dense": V.dense_cache_bytes(cfg, B),
                      "cache_bytes_ratio": V.latent_cache_bytes(cfg, B) / V.dense_cache_bytes(cfg, B)}
        assert V.device_status() == 0

    run_clocks = clocks.stop()
    nvml.stop()
    # the clocks line: the 2 ms NVML samples inside the timed region; the 100 ms nvidia-smi samples of
    # the whole run and one blocking sample right after the timed region beside them
    clk = nvml.window("timed") or (dict(after_timed, samples=1, source="nvidia-smi right after the timed region")
                                   if after_timed else run_clocks)
    if clk is not None:
        clk = dict(clk, nvidia_smi_run=run_clocks, nvidia_smi_after_timed=after_timed)
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(cfg, args.cpu_seconds)
        line = {"metric": "latent-attention TFLOP/s (Wan-1.3B layer step, B200 BF16 TC peak fraction)",
                "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": headline_config(cfg, B, world, args),
                "query_tokens_per_s": q_tok_s,
                "pct_of_bf16_peak": 100.0 * value / world / pk["bf16_tflops"],
                "roofline": roofline, "kernels": kernels, "e2e": e2e, "gpu_launches": launches,
                "clocks": clk, "wall_s_timed": wall, "cpu_baseline": cpu, "path_ab": path_ab,
                "sustained": sustained, "comparison": comparison}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
