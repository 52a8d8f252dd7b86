"""Benchmark: exact tiled attention forward + backward on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fattn|reference]
                    [--workload long_causal]

One step = the whole hot path once over one batch: fa_fwd (O, LSE) then fa_bwd
(D preprocess, dK/dV kernel, dQ kernel) on the long-context workload (B=2, H=32,
N=16384, d=128, bf16, causal, seeded N(0,1) inputs).  Throughput is attention TFLOPS
with 4·B·H·N²·d forward FLOPs (halved when causal) and 2.5x that for the backward pass.
Sliding-window workloads (--workload long_local_w4096) call fa_fwd_local / fa_bwd_local
and count 4·d FLOPs per allowed (query, key) pair.  Multi-GPU (torchrun) runs one independent problem per rank (heads /
batches are independent: no collective on the data path, weak scaling); time is the max
over ranks of CUDA-event time.

--impl reference times the CPU fp64 oracle (the only reference this build has) on a
bounded sample of the same workload: the last R query rows of one head against all keys,
which under the bottom-right causal reading is exactly those rows' share of the problem.
"""

from __future__ import annotations

import argparse
import hashlib
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

METRIC = "attention TFLOPS (fwd, fwd+bwd) and % of B200 BF16 tensor peak, N=1K–16K"
UNIT = "TFLOPS"
FALLBACK_PEAK_TFLOPS = 1590.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.txt")
BWD_SOURCES = ["exact_tiled_attention_33_b200/csrc/bwd_fused_kernel.cuh",
               "exact_tiled_attention_33_b200/csrc/sm100.cuh",
               "exact_tiled_attention_33_b200/csrc/fattn_internal.h"]
FP8_SOURCES = ["exact_tiled_attention_33_b200/csrc/fwd_kernel.cuh",
               "exact_tiled_attention_33_b200/csrc/sm100.cuh",
               "exact_tiled_attention_33_b200/csrc/fattn_internal.h"]
BWD_KERNEL_DESC = ("fa_bwd (D preprocess + single-pass dK/dV/dQ kernel + dQ conversion, timed "
                   "as one call)")
FWD_SOURCES = ["exact_tiled_attention_33_b200/csrc/fwd_kernel.cuh",
               "exact_tiled_attention_33_b200/csrc/sm100.cuh",
               "exact_tiled_attention_33_b200/csrc/fattn_internal.h"]


# ------------------------------------------------------------------ helpers (CPU-testable)
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput_tflops(flops_per_step_per_rank: float, steps: int, world: int,
                      max_seconds: float) -> float:
    """Whole-job throughput: all ranks' work divided by the slowest rank's time."""
    return flops_per_step_per_rank * steps * world / max_seconds / 1e12


def head_range(H: int, rank: int, world: int):
    """Heads [h0, h1) of `rank` in the head split of the pages' tensor-parallel attention
    (page "FlashAttention-2的核心设计原理", section "FlashAttention-2反向传播与多GPU训练"):
    H / world consecutive heads per rank, rank r holding heads r*H/world .. (r+1)*H/world - 1."""
    if world <= 0 or H % world != 0:
        raise ValueError(f"H = {H} heads do not split evenly over {world} ranks")
    per = H // world
    return rank * per, (rank + 1) * per


def gather_heads(local, world: int):
    """All-gather every rank's [B, N, H/world, d] output and join them along the head
    dimension (rank order = head order): the full [B, N, H, d] result on every rank."""
    if world == 1:
        return local
    import torch
    import torch.distributed as dist
    B, N, Hl, d = local.shape
    parts = torch.empty((world * B, N, Hl, d), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(parts, local.contiguous())
    # [world * B, N, Hl, d] -> [world, B, N, Hl, d] -> [B, N, world, Hl, d] -> [B, N, H, d]
    return parts.view(world, B, N, Hl, d).permute(1, 2, 0, 3, 4).reshape(B, N, world * Hl, d)


def sources_sha(paths) -> str:
    """Hash of the kernel sources without their // comments and blank lines, so that the
    recorded DRAM traffic of a kernel stays attached to it until its code changes."""
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def read_traffic(kernel: str, workload: str, sha: str):
    """DRAM bytes per launch recorded from an ncu capture, if it matches this source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    for line in open(TRAFFIC_FILE):
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("kernel") == kernel and f.get("workload") == workload and \
                f.get("source_sha") == sha:
            return float(f["bytes_per_launch"])
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), d.get("hbm_gbs"), "measured"
    return FALLBACK_PEAK_TFLOPS, 1400.0, 6650.0, "fallback"


REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    """SM clocks and throttle reasons sampled during the timed region: NVML (the library
    nvidia-smi reads) polled every 20 ms from a thread, so even a region of a few hundred
    milliseconds gets a dozen samples; nvidia-smi in a subprocess when NVML is missing."""

    _BITS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
             "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
             "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
             "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, gpu_index: int):
        self.rows = []          # (sm MHz, max sm MHz, [active reasons])
        self.proc = None
        self.thread = None
        self.source = None
        try:
            import threading
            import pynvml
            import torch
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(torch.cuda._get_nvml_device_index(gpu_index))
            bits = {r: getattr(pynvml, n) for r, n in self._BITS.items()}
            self.stop_flag = threading.Event()

            def poll():
                mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                while True:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    why = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.rows.append((float(sm), float(mx),
                                      [r for r, b in bits.items() if why & b]))
                    if self.stop_flag.wait(0.02):
                        return
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = "nvml, 20 ms"
            return
        except Exception:  # noqa: BLE001 - any NVML failure falls back to nvidia-smi
            self.thread = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            q = ("index,clocks.sm,clocks.max.sm,power.draw," +
                 ",".join(f"clocks_event_reasons.{r}" for r in REASONS))
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(gpu_index)], stdout=self.out, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 100 ms"
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()
            for line in open(self.path):
                r = [x.strip() for x in line.split(",")]
                if len(r) == 4 + len(REASONS) and r[1].replace(".", "").isdigit():
                    self.rows.append((float(r[1]), float(r[2]) if r[2].replace(".", "").isdigit()
                                      else float("nan"),
                                      [REASONS[i] for i in range(len(REASONS))
                                       if r[4 + i].lower() == "active"]))
            os.unlink(self.path)
        if not self.rows:
            return None
        return {"sm_mhz": statistics.median(r[0] for r in self.rows),
                "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": sorted({x for r in self.rows for x in r[2]}),
                "samples": len(self.rows), "source": self.source}


# ------------------------------------------------------------------ oracle timing
_HEAD_CACHE = {}


def oracle_threads() -> int:
    """Threads the oracle runs on: its matrix products go to numpy's BLAS pool (the rest of
    its numpy steps are single-threaded), so the BLAS pool size; the logical CPU count when
    no BLAS pool is visible."""
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except ImportError:
        pass
    return os.cpu_count() or 1


def host_cpus() -> dict:
    """Physical and logical core counts of the host the oracle is timed on."""
    try:
        import psutil
        phys = psutil.cpu_count(logical=False)
    except ImportError:
        phys = None
    return {"physical_cores": phys, "logical_cores": os.cpu_count()}

def oracle_sample_seconds(w, rows: int, head=(0, 0)):
    """Run the fp64 oracle forward + backward for the last `rows` query rows of one head
    against all keys; return (seconds, metric FLOPs of that share, threads)."""
    import numpy as np
    import oracle
    from exact_tiled_attention_33_b200 import workloads as wl
    key = (w.name, w.seed, head)
    if key not in _HEAD_CACHE:
        t = wl.generate(w)
        b, h = head
        if w.varlen:  # the longest packed sequence stands for the head's problem
            cu = w.cu_seqlens()
            seg = int(np.argmax(np.diff(cu)))
            rs = slice(int(cu[seg]), int(cu[seg + 1]))
            _HEAD_CACHE[key] = tuple(wl.to_f64(t[x][rs, h].clone()) for x in ("q", "k", "v", "do"))
        else:
            _HEAD_CACHE[key] = tuple(wl.to_f64(t[x][b, :, h].clone())
                                     for x in ("q", "k", "v", "do"))
    q, k, v, do = _HEAD_CACHE[key]
    N = q.shape[0]
    r0 = N - rows
    t0 = time.perf_counter()
    if w.window is None:
        oracle.attention_forward(q[r0:], k, v, w.softmax_scale, w.causal)
        oracle.attention_backward(q[r0:], k, v, do[r0:], w.softmax_scale, w.causal)
    else:
        # the sampled rows keep their positions: the window is taken against all N keys
        # by running the last rows as a shorter query block (bottom-right alignment)
        oracle.attention_forward(q[r0:], k, v, w.softmax_scale, False, window=w.window)
        oracle.attention_backward(q[r0:], k, v, do[r0:], w.softmax_scale, False,
                                  window=w.window)
    dt = time.perf_counter() - t0
    win = w.window if w.window is not None else ((-1, 0) if w.causal else (-1, -1))
    keys = wl.window_pairs(rows, N, win)
    flops = 3.5 * 4.0 * float(keys) * w.d
    return dt, flops, oracle_threads()


def oracle_full_seconds(name: str) -> dict:
    """The fp64 oracle's forward + backward over every (batch, head) of a small workload,
    timed directly (no sampling)."""
    import oracle
    from exact_tiled_attention_33_b200 import workloads as wl
    w = wl.get(name)
    t = wl.generate(w)
    q, k, v, do = (wl.to_f64(t[x]) for x in ("q", "k", "v", "do"))
    t0 = time.perf_counter()
    for b in range(w.B):
        for h in range(w.H):
            a = (q[b, :, h], k[b, :, h], v[b, :, h])
            oracle.attention_forward(*a, w.softmax_scale, w.causal)
            oracle.attention_backward(*a, do[b, :, h], w.softmax_scale, w.causal)
    dt = time.perf_counter() - t0
    return {"workload": name, "seconds": dt, "gflops": 3.5 * w.fwd_flops() / dt / 1e9}


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    # size the per-step sample so a step takes about a second on this host
    seq = max(w.seqlens) if w.varlen else w.N
    rows = min(64, seq)
    dt, _, _ = oracle_sample_seconds(w, rows)
    while dt < 0.5 and rows < seq:
        rows = min(seq, rows * 2)
        dt, _, _ = oracle_sample_seconds(w, rows)
    for _ in range(args.warmup):
        oracle_sample_seconds(w, rows)
    total_t, total_f = 0.0, 0.0
    threads = oracle_threads()
    for _ in range(args.steps):
        dt, fl, threads = oracle_sample_seconds(w, rows)
        total_t += dt
        total_f += fl
    value = total_f / total_t / 1e12
    where = ("head 0 of the longest packed sequence" if w.varlen else "head (b=0,h=0)")
    sample = (f"last {rows} query rows of {where} of {w.name} against all "
              f"{seq} keys, fp64 oracle fwd+bwd, per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(w.describe(), parallelism=f"dp{world}"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, **host_cpus(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ N = 128..4K sweep
SWEEP = ["tiny_causal", "tiny_noncausal", "a100table_N1024", "a100table_N2048",
         "a100table_N4096", "llama_causal", "varlen3", "varlen64"]


def _timed(fn, stream, dev, flush, reps):
    """CUDA-event times (ms) of `reps` launches of fn, each alone: L2-flushed (a 256 MB
    write before each) and L2-warm (after a launch on the same data, with a ~100 us GPU
    sleep in between that touches no memory).  The flush or the sleep keeps the GPU busy
    while the host enqueues the launch, so the host's launch overhead is not timed."""
    import torch
    for _ in range(5):
        fn()
    cold, warm = [], []
    for _ in range(reps):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        cold.append(a.elapsed_time(b))
    fn()
    for _ in range(reps):
        torch.cuda._sleep(200_000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        warm.append(a.elapsed_time(b))
    return {"median": statistics.median(cold), "min": min(cold), "max": max(cold),
            "warm_median": statistics.median(warm)}


def sweep_small_n(lib, dev):
    """Forward and backward of the pages' other shapes on one GPU: the tiny B1 H2 N128 d64
    case, the A100-table B8 H16 d64 at N = 1K, 2K, 4K, the Llama-style B4 H32 d128 N=4K,
    and the packed varlen batches (3 sequences / 896 tokens, 64 sequences).  Each launch is
    timed alone with CUDA events, L2-flushed (inputs of these sizes fit in L2) and L2-warm;
    200 launches for the microsecond-scale cases, 20 otherwise.  TFLOPS and the forward's
    algorithmic HBM GB/s (Q, K, V read once, O and LSE written once) use the flushed
    median."""
    import torch
    from exact_tiled_attention_33_b200 import _lib
    from exact_tiled_attention_33_b200 import attention as fa
    from exact_tiled_attention_33_b200 import workloads as wl
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    out = []
    for name in SWEEP:
        w = wl.get(name)
        t = wl.generate(w)
        q, k, v, do = (t[x].to(dev) for x in ("q", "k", "v", "do"))
        dt = _lib.FA_BF16 if w.dtype == "bf16" else _lib.FA_FP16
        o = torch.empty_like(q)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        if w.varlen:
            cu = t["cu_seqlens"].to(dev)
            L = max(w.seqlens)
            lse = torch.empty((w.H, w.total), dtype=torch.float32, device=dev)
            ws = fa.varlen_bwd_workspace(w.total, w.H, w.d, dev)

            def fwd():
                fa.varlen_fwd(q, k, v, cu, cu, L, L, w.softmax_scale, w.causal, out=o, lse=lse)

            def bwd():
                fa.varlen_bwd(q, k, v, o, lse, do, cu, cu, L, L, w.softmax_scale, w.causal,
                              workspace=ws, dq=dq, dk=dk, dv=dv)
            shape = {"num_seqs": len(w.seqlens), "total_tokens": w.total}
            rows = w.total
        else:
            B, N, H, d = q.shape
            lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
            ws = fa.bwd_workspace(B, N, H, d, dev)

            def fwd():
                _lib.check(lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), B, N, H, d, w.softmax_scale,
                                      int(w.causal), dt, sh), "fa_fwd")

            def bwd():
                _lib.check(lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                                      dk.data_ptr(), dv.data_ptr(), B, N, H, d,
                                      w.softmax_scale, int(w.causal), ws.data_ptr(),
                                      ws.numel(), dt, sh), "fa_bwd")
            shape = {"B": B, "N": N}
            rows = B * N
        small = w.fwd_flops() < 1e10
        reps = 200 if small else 20
        tf, tb = _timed(fwd, stream, dev, flush, reps), _timed(bwd, stream, dev, flush, reps)
        assert lib.fa_get_device_status(sh) == 0
        f = w.fwd_flops()
        e = q.numel() * q.element_size()
        fwd_bytes = 4 * e + 4 * w.H * rows
        out.append(dict({"workload": name, "H": w.H, "d": w.d, "causal": w.causal}, **shape,
                        fwd_us=1e3 * tf["median"], fwd_us_min=1e3 * tf["min"],
                        fwd_us_max=1e3 * tf["max"], fwd_us_l2_warm=1e3 * tf["warm_median"],
                        bwd_us=1e3 * tb["median"], bwd_us_min=1e3 * tb["min"],
                        bwd_us_max=1e3 * tb["max"], bwd_us_l2_warm=1e3 * tb["warm_median"],
                        fwd_tflops=f / tf["median"] / 1e9,
                        fwd_bwd_tflops=3.5 * f / (tf["median"] + tb["median"]) / 1e9,
                        fwd_hbm_gbs=fwd_bytes / tf["median"] / 1e6, reps=reps))
    del flush
    return out


# ------------------------------------------------------------------ GPU arm
def other_arms(lib, dev, reps=10):
    """The NEXT rows' workloads timed inside the default bench run, so that its line carries
    them: the FP8 forward on the long causal shape (TFLOPS), one KV-cache decode step over
    8 x 16384 cached tokens (GB/s of K/V read), and the causal 4096-key window on the long
    shape (fwd + bwd TFLOPS).  Each launch alone with CUDA events on the launching stream,
    L2 flushed before it (a 256 MB write); median of `reps`."""
    import torch
    from exact_tiled_attention_33_b200 import _lib
    from exact_tiled_attention_33_b200 import attention as fa
    from exact_tiled_attention_33_b200 import workloads as wl
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    out = {}
    # FP8 forward
    w = wl.get("fp8_long_causal")
    t = wl.generate(w, with_grad_out=False)
    q8, k8, v8 = (t[x].to(dev) for x in ("q8", "k8", "v8"))
    sq, sk, sv = t["q_descale"], t["k_descale"], t["v_descale"]
    del t
    o8, l8 = fa.fwd_fp8(q8, k8, v8, sq, sk, sv, w.softmax_scale, w.causal)
    tf = _timed(lambda: fa.fwd_fp8(q8, k8, v8, sq, sk, sv, w.softmax_scale, w.causal, out=o8,
                                   lse=l8), stream, dev, flush, reps)
    out["fp8_long_causal_fwd"] = {"ms": tf["median"], "tflops": w.fwd_flops() / tf["median"] / 1e9,
                                  "unit": "TFLOPS", "reps": reps}
    del q8, k8, v8, o8, l8
    # KV-cache decode, one new token per sequence
    dw = wl.get_decode("decode_b8_l16k")
    g = wl.generate_decode(dw)
    q, kc, vc = g["q"].to(dev), g["k_cache"].to(dev), g["v_cache"].to(dev)
    lens = g["cache_seqlens"].to(dev)
    del g
    max_len = max(dw.cache_lens)
    od = torch.empty_like(q)
    ld = torch.empty((q.shape[0], q.shape[2], q.shape[1]), dtype=torch.float32, device=dev)
    wsd = fa.decode_workspace(q.shape[0], q.shape[1], q.shape[2], q.shape[3], max_len, dev)
    td = _timed(lambda: fa.decode(q, kc, vc, lens, max_len, dw.softmax_scale, dw.causal, out=od,
                                  lse=ld, workspace=wsd), stream, dev, flush, 5 * reps)
    out["decode_b8_l16k"] = {"us": 1e3 * td["median"],
                             "gbs": dw.bytes_moved() / td["median"] / 1e6, "unit": "GB/s",
                             "reps": 5 * reps}
    del q, kc, vc, od, ld, wsd
    # sliding window (4095, 0) on the long shape
    w = wl.get("long_local_w4096")
    t = wl.generate(w)
    q, k, v, do = (t[x].to(dev) for x in ("q", "k", "v", "do"))
    del t
    o, lse = fa.fwd_local(q, k, v, w.window, w.softmax_scale)
    ws = fa.bwd_workspace(w.B, w.N, w.H, w.d, dev)
    tf = _timed(lambda: fa.fwd_local(q, k, v, w.window, w.softmax_scale, out=o, lse=lse), stream,
                dev, flush, reps)
    tb = _timed(lambda: fa.bwd_local(q, k, v, o, lse, do, w.window, w.softmax_scale,
                                     workspace=ws), stream, dev, flush, reps)
    f = w.fwd_flops()
    out["long_local_w4096"] = {"fwd_ms": tf["median"], "bwd_ms": tb["median"],
                               "fwd_tflops": f / tf["median"] / 1e9,
                               "fwd_bwd_tflops": 3.5 * f / (tf["median"] + tb["median"]) / 1e9,
                               "unit": "TFLOPS", "reps": reps}
    assert lib.fa_get_device_status(stream.cuda_stream) == 0
    del q, k, v, do, o, lse, ws, flush
    torch.cuda.empty_cache()
    return out


def run_fattn(args, w):
    import torch
    import torch.distributed as dist

    from exact_tiled_attention_33_b200 import _lib
    from exact_tiled_attention_33_b200 import attention as fa
    from exact_tiled_attention_33_b200 import workloads as wl

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    lib = _lib.load()
    split_heads = getattr(args, "split", "none") == "heads"
    if w.varlen and (split_heads or w.window is not None):
        raise SystemExit("a packed (varlen) workload runs without --split heads or a window")
    if split_heads:
        # one shared problem (same seed on every rank), its heads split over the ranks; each
        # step ends with an all-gather of O along the head dimension
        wr = w
        h0, h1 = head_range(w.H, rank, world)
        full = wl.generate(wr)
        host = {x: full[x][:, :, h0:h1].contiguous() for x in ("q", "k", "v", "do")}
        del full
    else:
        # each rank owns an independent problem of the same size (its own seed)
        wr = wl.Workload(**{**w.__dict__, "seed": w.seed + rank})
        host = wl.generate(wr)
    scale, causal = wr.softmax_scale, int(wr.causal)
    dtype = _lib.FA_BF16 if wr.dtype == "bf16" else _lib.FA_FP16
    q, k, v, do = (host[x].to(dev) for x in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    if wr.varlen:
        # packed sequences [total, H, d] through fa_varlen_fwd / fa_varlen_bwd
        H, d = host["q"].shape[1], wr.d
        T, S, L = wr.total, len(wr.seqlens), max(wr.seqlens)
        cu = host["cu_seqlens"].to(device=dev, dtype=torch.int32)
        lse = torch.empty((H, T), dtype=torch.float32, device=dev)

        def new_ws():
            return fa.varlen_bwd_workspace(T, H, d, dev)
    else:
        B, N, H, d = wr.B, wr.N, host["q"].shape[2], wr.d
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)

        def new_ws():
            return fa.bwd_workspace(B, N, H, d, dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = new_ws()
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    def varlen_fwd(qq, kk, vv, oo, ll, hs):
        _lib.check(lib.fa_varlen_fwd(qq, kk, vv, oo, ll, cu.data_ptr(), cu.data_ptr(), L, L, H,
                                     d, scale, causal, S, T, T, dtype, hs), "fa_varlen_fwd")

    def varlen_bwd(qq, kk, vv, oo, dd, ll, gq, gk, gv, wsb, hs):
        _lib.check(lib.fa_varlen_bwd(qq, kk, vv, oo, dd, ll, gq, gk, gv, cu.data_ptr(),
                                     cu.data_ptr(), L, L, H, d, scale, causal, S, T, T,
                                     wsb.data_ptr(), wsb.numel(), dtype, hs), "fa_varlen_bwd")

    def launch_fwd():
        if wr.varlen:
            varlen_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), sh)
        elif wr.window is None:
            _lib.check(lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), B, N, H, d, scale, causal, dtype, sh), "fa_fwd")
        else:
            _lib.check(lib.fa_fwd_local(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                        lse.data_ptr(), B, N, H, d, scale, wr.window[0],
                                        wr.window[1], dtype, sh), "fa_fwd_local")

    def launch_bwd():
        if wr.varlen:
            varlen_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                       lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws, sh)
        elif wr.window is None:
            _lib.check(lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                  dv.data_ptr(), B, N, H, d, scale, causal, ws.data_ptr(),
                                  ws.numel(), dtype, sh), "fa_bwd")
        else:
            _lib.check(lib.fa_bwd_local(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                        do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                                        dk.data_ptr(), dv.data_ptr(), B, N, H, d, scale,
                                        wr.window[0], wr.window[1], ws.data_ptr(), ws.numel(),
                                        dtype, sh), "fa_bwd_local")

    o_full = [None]

    def step():
        launch_fwd()
        launch_bwd()
        if split_heads:
            o_full[0] = gather_heads(o, world)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert lib.fa_get_device_status(sh) == 0, "device status after warm-up"

    # ---- timed region: inputs (268 MB per tensor) are larger than the 126 MB L2
    sampler = ClockSampler(local) if rank == 0 else None
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        launch_fwd()
        ev[i][1].record(stream)
        launch_bwd()
        ev[i][2].record(stream)
        if split_heads:
            o_full[0] = gather_heads(o, world)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler is not None else None
    status = lib.fa_get_device_status(sh)
    assert status == 0, f"device status {status} in timed region"
    total_ms = t_start.elapsed_time(t_end)
    fwd_ms = [a.elapsed_time(b) for a, b, _ in ev]
    bwd_ms = [b.elapsed_time(c) for _, b, c in ev]
    max_s = max_over_ranks(total_ms / 1e3, world)
    f_fwd = wr.fwd_flops() * H / wr.H   # this rank's share (all of it unless heads are split)
    f_step = 3.5 * f_fwd
    value = throughput_tflops(f_step, args.steps, world, max_s)
    fwd_avg = statistics.mean(fwd_ms)
    bwd_avg = statistics.mean(bwd_ms)

    # ---- the forward alone, as the pages' forward benchmarks time it: `steps` forward
    # launches back to back on the same inputs (each tensor larger than the 126 MB L2),
    # CUDA events around them on the launching stream, max over ranks
    fsampler = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    f_start = torch.cuda.Event(enable_timing=True)
    f_end = torch.cuda.Event(enable_timing=True)
    f_start.record(stream)
    for _ in range(args.steps):
        launch_fwd()
    f_end.record(stream)
    torch.cuda.synchronize(dev)
    fclocks = fsampler.stop() if fsampler is not None else None
    assert lib.fa_get_device_status(sh) == 0, "device status after the forward-only loop"
    fo_s = max_over_ranks(f_start.elapsed_time(f_end) / 1e3, world)
    fwd_only_tflops = throughput_tflops(f_fwd, args.steps, world, fo_s)

    # ---- end to end through the C ABI with pinned host buffers.  Every step copies its
    # inputs q, k, v, dO host -> device, runs fwd + bwd and copies O, LSE, dQ, dK, dV back.
    # Two device buffer sets and three streams pipeline the steps: the copies of one step
    # overlap the compute of the previous / next step (H2D and D2H also run concurrently),
    # as a training loop that feeds a GPU from host memory would.
    e2e = None
    if not args.no_e2e and not split_heads:
        hin = [host[x].pin_memory() for x in ("q", "k", "v", "do")]
        sets = []
        for bset in range(2):
            ins = [q, k, v, do] if bset == 0 else [torch.empty_like(x) for x in (q, k, v, do)]
            outs = [o, lse, dq, dk, dv] if bset == 0 else [torch.empty_like(x)
                                                          for x in (o, lse, dq, dk, dv)]
            hout = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in outs]
            wsb = ws if bset == 0 else new_ws()
            sets.append((ins, outs, hout, wsb))
        h2d = sum(x.numel() * x.element_size() for x in hin)
        d2h = sum(x.numel() * x.element_size() for x in sets[0][2])
        # steady-state throughput of the pipeline: enough steps that its fill (the first
        # step's inputs) and drain (the last step's outputs) are a small share of the region
        e2e_steps = max(16, min(2 * args.steps, 48))
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def compute(ins, outs, wsb, hs):
            qq, kk, vv, dd = (x.data_ptr() for x in ins)
            oo, ll, gq, gk, gv = (x.data_ptr() for x in outs)
            if wr.varlen:
                varlen_fwd(qq, kk, vv, oo, ll, hs)
                varlen_bwd(qq, kk, vv, oo, dd, ll, gq, gk, gv, wsb, hs)
            elif wr.window is None:
                _lib.check(lib.fa_fwd(qq, kk, vv, oo, ll, B, N, H, d, scale, causal, dtype, hs),
                           "fa_fwd")
                _lib.check(lib.fa_bwd(qq, kk, vv, oo, dd, ll, gq, gk, gv, B, N, H, d, scale,
                                      causal, wsb.data_ptr(), wsb.numel(), dtype, hs), "fa_bwd")
            else:
                wl_, wr_ = wr.window
                _lib.check(lib.fa_fwd_local(qq, kk, vv, oo, ll, B, N, H, d, scale, wl_, wr_,
                                            dtype, hs), "fa_fwd_local")
                _lib.check(lib.fa_bwd_local(qq, kk, vv, oo, dd, ll, gq, gk, gv, B, N, H, d,
                                            scale, wl_, wr_, wsb.data_ptr(), wsb.numel(), dtype,
                                            hs), "fa_bwd_local")

        def e2e_step(i):
            ins, outs, hout, wsb = sets[i % 2]
            b_ = i % 2
            s_in.wait_event(ev_cmp[b_])            # inputs of this set consumed (step i - 2)
            with torch.cuda.stream(s_in):
                for hsrc, ddst in zip(hin, ins):
                    ddst.copy_(hsrc, non_blocking=True)
            ev_in[b_].record(s_in)
            s_cmp.wait_event(ev_in[b_])
            s_cmp.wait_event(ev_out[b_])           # outputs of this set copied out (step i - 2)
            compute(ins, outs, wsb, s_cmp.cuda_stream)
            ev_cmp[b_].record(s_cmp)
            s_out.wait_event(ev_cmp[b_])
            with torch.cuda.stream(s_out):
                for dsrc, hdst in zip(outs, hout):
                    hdst.copy_(dsrc, non_blocking=True)
            ev_out[b_].record(s_out)

        for i in range(2):                        # warm-up of the pipeline
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for i in range(e2e_steps):
            e2e_step(i)
        b.record(s_out)                           # after the last step's D2H (all in order)
        torch.cuda.synchronize(dev)
        e2e_s = max_over_ranks(a.elapsed_time(b) / 1e3, world)
        e2e = {"value": throughput_tflops(f_step, e2e_steps, world, e2e_s), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "pipelined": "2 buffer sets; H2D, compute, D2H on 3 streams"}
        assert lib.fa_get_device_status(sh) == 0, "device status after e2e"
        del sets

    peak_burst, peak_sust, hbm, peak_src = load_peaks()
    bwd_sha = sources_sha(BWD_SOURCES)
    fwd_sha = sources_sha(FWD_SOURCES)
    bwd_ach = 2.5 * f_fwd / (bwd_avg / 1e3) / 1e12
    fwd_ach = f_fwd / (fwd_avg / 1e3) / 1e12
    # The timed region lasts well under the seconds a sustained (power-capped) measurement
    # needs, so the fractions are taken against the burst peak; the fraction of the
    # sustained figure is kept beside it, labelled.
    timed_s = total_ms / 1e3
    roofline = {
        "kernel": BWD_KERNEL_DESC,
        "bound": "tensor", "achieved": bwd_ach, "peak": peak_burst, "unit": "TFLOP/s",
        "frac": bwd_ach / peak_burst,
        "peak_source": f"bf16_tflops burst ({peak_src}); timed region {timed_s:.2f} s",
        "frac_of_sustained_peak": bwd_ach / peak_sust,
        "traffic": read_traffic("fa_bwd", wr.name, bwd_sha),
        "flops_per_launch": 2.5 * f_fwd}
    fwd_roof = {"kernel": "fa_fwd_kernel", "bound": "tensor", "achieved": fwd_ach,
                "peak": peak_burst, "unit": "TFLOP/s", "frac": fwd_ach / peak_burst,
                "peak_source": f"bf16_tflops burst ({peak_src})",
                "frac_of_sustained_peak": fwd_ach / peak_sust,
                "traffic": read_traffic("fa_fwd_kernel", wr.name, fwd_sha),
                "flops_per_launch": f_fwd}
    fwd_only = {"ms": 1e3 * fo_s / args.steps, "tflops": fwd_only_tflops,
                "frac_of_burst_peak": fwd_only_tflops / world / peak_burst,
                "frac_of_sustained_peak": fwd_only_tflops / world / peak_sust,
                "clocks": fclocks}

    sweep = None
    if rank == 0 and world == 1 and not args.no_sweep:
        sweep = sweep_small_n(lib, dev)
    arms = None
    if rank == 0 and world == 1 and not args.no_other_arms:
        arms = other_arms(lib, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        seq = max(wr.seqlens) if wr.varlen else wr.N
        rows = min(512, seq)
        dt, fl, threads = oracle_sample_seconds(wr, rows)
        # grow the sample toward ~10 s of CPU work
        while dt < 5.0 and rows < seq:
            rows = min(seq, rows * 2)
            dt, fl, threads = oracle_sample_seconds(wr, rows)
        where = (f"of head 0 of the longest packed sequence against all its {seq} keys"
                 if wr.varlen else f"of head (b=0,h=0) against all {seq} keys")
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, **host_cpus(),
               "kind": "oracle",
               "sample": f"last {rows} query rows {where}"
                         f"{'' if wr.window is None else ' (window ' + str(list(wr.window)) + ')'}"
                         f", fp64 oracle fwd+bwd ({dt:.1f} s)",
               # one whole step (every head of every batch row) at the sample's rate
               "full_step_seconds_extrapolated": f_step / (fl / dt),
               "full_runs": [oracle_full_seconds(n) for n in ("tiny_causal", "a100table_N1024")]}

    tensor_mb = q.numel() * q.element_size() / 1e6
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * max_s / args.steps, "higher_is_better": True,
                "scaling": "strong" if split_heads else "weak", "vs_baseline": None,
                "dtype": wr.dtype, "data": "synthetic",
                "config": dict(wr.describe(), seed=w.seed,
                               parallelism=(f"heads{world} (head split, all-gather of O)"
                                            if split_heads else f"dp{world}"),
                               l2=(f"inputs larger than L2 ({tensor_mb:.0f} MB per tensor), "
                                   "no flush" if tensor_mb > 126 else
                                   f"inputs smaller than L2 ({tensor_mb:.1f} MB per tensor), "
                                   "L2-warm, no flush")),
                "fwd_tflops": f_fwd / (fwd_avg / 1e3) / 1e12,
                "bwd_tflops": bwd_ach,
                "pct_of_bf16_peak": {"fwd_bwd": value / world / peak_burst,
                                     "fwd": fwd_ach / peak_burst,
                                     "peak_tflops": peak_burst, "peak_source": peak_src},
                "ms_fwd": fwd_avg, "ms_bwd": bwd_avg,
                "gpu_launches": 4 * args.steps,
                "roofline": roofline, "roofline_fwd": fwd_roof, "fwd_only": fwd_only,
                "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu, "sweep_small_n": sweep,
                "other_arms": arms}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_decode_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from exact_tiled_attention_33_b200 import workloads as wl
    g = wl.generate_decode(w)
    n = 1
    dt, _, _ = oracle_decode_seconds(w, g, n)
    while dt < 0.5 and n < w.H:
        n = min(w.H, n * 2)
        dt, _, _ = oracle_decode_seconds(w, g, n)
    reps = max(1, int(0.5 / max(dt, 1e-3)))
    for _ in range(args.warmup):
        oracle_decode_seconds(w, g, n, reps)
    tot_t = tot_b = 0.0
    threads = oracle_threads()
    for _ in range(args.steps):
        dt, by, threads = oracle_decode_seconds(w, g, n, reps)
        tot_t += dt
        tot_b += by
    value = tot_b / tot_t / 1e9
    sample = (f"sequence 0 ({w.cache_lens[0]} cached rows), {n} heads x {reps} passes, "
              f"fp64 oracle decode, per step")
    print(json.dumps({"impl": "reference", "metric": DECODE_METRIC, "value": value,
                      "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                      "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                      "dtype": "f64", "data": "synthetic",
                      "config": dict(w.describe(), parallelism=f"dp{world}"),
                      "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads,
                                       **host_cpus(),
                                       "kind": "oracle", "sample": sample},
                      "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                              "d2h_bytes_per_step": 0}}), flush=True)
    return 0


# ------------------------------------------------------------------ FP8 forward arm
FP8_METRIC = "FP8 (E4M3) attention forward TFLOPS and % of B200 FP8 tensor peak"


def oracle_fp8_seconds(w, host, rows: int, reps: int = 1):
    """fp64 oracle forward of the last `rows` query rows of head (0, 0), FP8 inputs."""
    import numpy as np
    import oracle
    from exact_tiled_attention_33_b200 import workloads as wl
    q8, k8, v8 = (host[x][0, :, 0].view(torch_uint8()).numpy() for x in ("q8", "k8", "v8"))
    N = q8.shape[0]
    r = np.arange(N - rows, N)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.attention_forward_fp8(q8, k8, v8, host["q_descale"], host["k_descale"],
                                     host["v_descale"], w.softmax_scale, w.causal, rows=r)
    dt = time.perf_counter() - t0
    win = (-1, 0) if w.causal else (-1, -1)
    return dt, 4.0 * w.d * wl.window_pairs(rows, N, win) * reps, oracle_threads()


def run_fp8_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from exact_tiled_attention_33_b200 import workloads as wl
    host = wl.generate(w, with_grad_out=False)
    rows = 64
    dt, _, _ = oracle_fp8_seconds(w, host, rows)
    while dt < 0.5 and rows < w.N:
        rows = min(w.N, rows * 2)
        dt, _, _ = oracle_fp8_seconds(w, host, rows)
    for _ in range(args.warmup):
        oracle_fp8_seconds(w, host, rows)
    tot_t = tot_f = 0.0
    threads = oracle_threads()
    for _ in range(args.steps):
        dt, fl, threads = oracle_fp8_seconds(w, host, rows)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = (f"last {rows} query rows of head (b=0,h=0) of {w.name} against all {w.N} keys, "
              f"fp64 oracle forward of the dequantised FP8 inputs, per step")
    print(json.dumps({"impl": "reference", "metric": FP8_METRIC, "value": value, "unit": UNIT,
                      "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
                      "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic", "config": dict(w.describe(), parallelism=f"dp{world}"),
                      "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads,
                                       **host_cpus(),
                                       "kind": "oracle", "sample": sample},
                      "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                              "d2h_bytes_per_step": 0}}), flush=True)
    return 0


def torch_uint8():
    import torch
    return torch.uint8


def run_fp8(args, w):
    import torch
    import torch.distributed as dist

    from exact_tiled_attention_33_b200 import _lib
    from exact_tiled_attention_33_b200 import workloads as wl

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    lib = _lib.load()
    wr = wl.Workload(**{**w.__dict__, "seed": w.seed + rank})
    host = wl.generate(wr, with_grad_out=False)
    B, N, H, d = wr.B, wr.N, wr.H, wr.d
    q8, k8, v8 = (host[x].to(dev) for x in ("q8", "k8", "v8"))
    sq, sk, sv = host["q_descale"], host["k_descale"], host["v_descale"]
    odt = _lib.FA_BF16 if wr.dtype == "bf16" else _lib.FA_FP16
    o = torch.empty(q8.shape, dtype=torch.bfloat16 if wr.dtype == "bf16" else torch.float16,
                    device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    def step():
        _lib.check(lib.fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), B, N, H, d, wr.softmax_scale, sq, sk, sv,
                                  int(wr.causal), odt, sh), "fa_fwd_fp8")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert lib.fa_get_device_status(sh) == 0, "device status after warm-up"
    # timed region: the inputs (134 MB per tensor) are larger than the 126 MB L2
    sampler = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler is not None else None
    assert lib.fa_get_device_status(sh) == 0, "device status in timed region"
    max_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, world)
    f = wr.fwd_flops()
    value = throughput_tflops(f, args.steps, world, max_s)
    per = statistics.mean(a.elapsed_time(b) for a, b in ev) / 1e3

    e2e = None
    if not args.no_e2e:
        hin = [host[x].view(torch.uint8).pin_memory() for x in ("q8", "k8", "v8")]
        dins = [x.view(torch.uint8) for x in (q8, k8, v8)]
        hout = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (o, lse)]
        n_e2e = max(2, min(args.steps, 5))

        def e2e_step():
            for hs, dd in zip(hin, dins):
                dd.copy_(hs, non_blocking=True)
            step()
            for ds, hd in zip((o, lse), hout):
                hd.copy_(ds, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        e2e_s = max_over_ranks(a.elapsed_time(b_) / 1e3, world)
        e2e = {"value": throughput_tflops(f, n_e2e, world, e2e_s), "unit": UNIT,
               "h2d_bytes_per_step": sum(x.numel() for x in hin),
               "d2h_bytes_per_step": sum(x.numel() * x.element_size() for x in hout),
               "steps": n_e2e}

    burst, sust, _, src = load_peaks()
    # no measured FP8 peak: the measured bf16 figure times the nominal FP8/BF16 ratio (2)
    peak_b, peak_s = 2 * burst, 2 * sust
    ach = f / per / 1e12
    sha = sources_sha(FP8_SOURCES)
    roofline = {"kernel": "fa_fwd_kernel<128, bf16 out, fp8>", "bound": "tensor",
                "achieved": ach, "peak": peak_s, "unit": "TFLOP/s", "frac": ach / peak_s,
                "frac_of_burst_peak": ach / peak_b,
                "peak_source": f"2 x bf16_tflops_sustained ({src}; nominal fp8/bf16 ratio)",
                "traffic": read_traffic("fa_fwd_kernel_fp8", wr.name, sha),
                "flops_per_launch": f}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = 256
        dt, fl, threads = oracle_fp8_seconds(wr, host, rows)
        while dt < 5.0 and rows < N:
            rows = min(N, rows * 2)
            dt, fl, threads = oracle_fp8_seconds(wr, host, rows)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, **host_cpus(),
               "kind": "oracle",
               "sample": f"last {rows} query rows of head (b=0,h=0) against all {N} keys, "
                         f"fp64 oracle forward of the dequantised FP8 inputs ({dt:.1f} s)"}
    if rank == 0:
        line = {"metric": FP8_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * max_s / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 (bf16 out)",
                "data": "synthetic",
                "config": dict(wr.describe(), seed=w.seed, parallelism=f"dp{world}",
                               l2="inputs larger than L2 (134 MB per tensor), no flush"),
                "gpu_launches": args.steps, "roofline": roofline, "clocks": clocks,
                "e2e": e2e, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ KV-cache decode arm
DECODE_METRIC = "KV-cache decode: HBM GB/s of the cached K/V read (and attention TFLOPS)"
DECODE_SOURCES = ["exact_tiled_attention_33_b200/csrc/decode_kernel.cuh",
                  "exact_tiled_attention_33_b200/csrc/sm100.cuh",
                  "exact_tiled_attention_33_b200/csrc/fattn_internal.h"]


def oracle_decode_seconds(w, g, n_heads: int, reps: int = 1):
    """fp64 oracle decode of sequence 0 for the first n_heads heads, `reps` times:
    (seconds, algorithmic K/V bytes of that work, threads)."""
    import oracle
    import torch
    L = w.cache_lens[0]
    if w.page_size:
        row = g["block_table"][0].numpy()
        kb = torch.from_numpy(oracle.kv_cache_gather(g["k_pages"].view(torch.int16).numpy(),
                                                     row, L)).view(g["q"].dtype)
        vb = torch.from_numpy(oracle.kv_cache_gather(g["v_pages"].view(torch.int16).numpy(),
                                                     row, L)).view(g["q"].dtype)
    else:
        kb, vb = g["k_cache"][0, :L], g["v_cache"][0, :L]
    q = g["q"][0].double().numpy()
    kb, vb = kb[:, :n_heads].double().numpy(), vb[:, :n_heads].double().numpy()
    t0 = time.perf_counter()
    for _ in range(reps):
        for h in range(n_heads):
            oracle.attention_forward(q[:, h], kb[:, h], vb[:, h], w.softmax_scale, w.causal)
    dt = time.perf_counter() - t0
    return dt, 2.0 * L * n_heads * w.d * 2 * reps, oracle_threads()


def run_decode(args, w):
    import torch
    import torch.distributed as dist

    from exact_tiled_attention_33_b200 import _lib
    from exact_tiled_attention_33_b200 import attention as fa
    from exact_tiled_attention_33_b200 import workloads as wl

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wr = wl.DecodeWorkload(**{**w.__dict__, "seed": w.seed + rank})
    host = wl.generate_decode(wr)
    lib = _lib.load()
    q = host["q"].to(dev)
    lens = host["cache_seqlens"].to(dev)
    B, Nq, H, d = q.shape
    max_len = max(wr.cache_lens)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    ws = fa.decode_workspace(B, Nq, H, d, max_len, dev)
    wsp, wsn = (0, 0) if ws is None else (ws.data_ptr(), ws.numel())
    dtype = _lib.FA_BF16 if wr.dtype == "bf16" else _lib.FA_FP16
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    if wr.page_size:
        kc, vc = host["k_pages"].to(dev), host["v_pages"].to(dev)
        bt = host["block_table"].to(dev)

        def step():
            _lib.check(lib.fa_decode_paged(q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                           o.data_ptr(), lse.data_ptr(), bt.data_ptr(),
                                           lens.data_ptr(), B, Nq, H, d, wr.page_size,
                                           kc.shape[0], bt.shape[1], max_len,
                                           wr.softmax_scale, int(wr.causal), wsp, wsn, dtype, sh),
                       "fa_decode_paged")
    else:
        kc, vc = host["k_cache"].to(dev), host["v_cache"].to(dev)

        def step():
            _lib.check(lib.fa_decode(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), o.data_ptr(),
                                     lse.data_ptr(), lens.data_ptr(), B, Nq, H, d, wr.capacity,
                                     max_len, wr.softmax_scale, int(wr.causal), wsp, wsn, dtype,
                                     sh), "fa_decode")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert lib.fa_get_device_status(sh) == 0, "device status after warm-up"
    # ---- timed region: the cache (>= 1 GB) is far larger than the 126 MB L2
    sampler = ClockSampler(local) if rank == 0 else None
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler is not None else None
    assert lib.fa_get_device_status(sh) == 0, "device status in timed region"
    max_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, world)
    per = statistics.mean(a.elapsed_time(b) for a, b in ev) / 1e3
    nbytes = wr.bytes_moved()
    value = nbytes * args.steps * world / max_s / 1e9
    splits_ws = lib.fa_decode_workspace_size(B, Nq, H, d, max_len)

    e2e = None
    if not args.no_e2e:
        # per step: H2D of the new tokens' q, the decode call, D2H of O and LSE (the cache
        # stays resident on the device, as a KV cache does between steps)
        hq = host["q"].pin_memory()
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        n_e2e = max(2, min(args.steps, 10))

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        e2e_s = max_over_ranks(a.elapsed_time(b_) / 1e3, world)
        e2e = {"value": nbytes * n_e2e * world / e2e_s / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": hq.numel() * hq.element_size(),
               "d2h_bytes_per_step": ho.numel() * ho.element_size() + hl.numel() * hl.element_size(),
               "steps": n_e2e}

    _, _, hbm, src = load_peaks()
    sha = sources_sha(DECODE_SOURCES)
    roofline = {"kernel": "fa_decode_kernel" + (" + fa_decode_combine_kernel" if splits_ws else ""),
                "bound": "hbm", "achieved": nbytes / per / 1e9, "peak": hbm, "unit": "GB/s",
                "frac": nbytes / per / 1e9 / hbm, "peak_source": f"hbm_gbs ({src})",
                "traffic": read_traffic("fa_decode", wr.name, sha), "bytes_per_launch": nbytes}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        reps = 1
        dt, by, threads = oracle_decode_seconds(wr, host, H, reps)
        while dt < 5.0:
            reps *= 2
            dt, by, threads = oracle_decode_seconds(wr, host, H, reps)
        cpu = {"value": by / dt / 1e9, "unit": "GB/s", "cores": threads, **host_cpus(),
               "kind": "oracle",
               "sample": f"sequence 0 ({wr.cache_lens[0]} cached rows), all {H} heads, "
                         f"{reps} passes, fp64 oracle decode ({dt:.1f} s)"}
    if rank == 0:
        line = {"metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * max_s / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": wr.dtype, "data": "synthetic",
                "config": dict(wr.describe(), seed=w.seed, parallelism=f"dp{world}",
                               l2="cache larger than L2, no flush"),
                "tflops": wr.flops() * args.steps * world / max_s / 1e12,
                "gpu_launches": (2 if splits_ws else 1) * args.steps,
                "roofline": roofline, "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="fattn", choices=["fattn", "reference"])
    ap.add_argument("--workload", default="long_causal")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the small-shape sweep of the default bench line")
    ap.add_argument("--no-other-arms", action="store_true",
                    help="skip the FP8, decode and window timings of the default bench line")
    ap.add_argument("--split", default="none", choices=["none", "heads"],
                    help="heads: one shared problem with its heads split over the ranks and O "
                         "all-gathered every step (strong scaling); none: one independent "
                         "problem per rank (weak scaling)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3) if args.impl == "fattn" else args.warmup
    from exact_tiled_attention_33_b200 import workloads as wl
    if args.workload in wl.DECODE_WORKLOADS:
        if args.impl == "reference":
            return run_decode_reference(args, wl.get_decode(args.workload))
        return run_decode(args, wl.get_decode(args.workload))
    w = wl.get(args.workload)
    if w.fp8:
        if args.impl == "reference":
            return run_fp8_reference(args, w)
        return run_fp8(args, w)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_fattn(args, w)


if __name__ == "__main__":
    sys.exit(main())
