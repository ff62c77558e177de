"""Benchmark of the fused group-wise dequant matmul on B200.

Default workload (the headline): pre-packed int4 decode GEMV, M = 1, over the
24-layer Qwen2.5-0.5B linear-layer set (q/k/v/o/gate/up/down, hidden 896),
fp16 scale/zero per 64-block, fp32 x.  One step = one grouped launch over
all 168 matrices of the set.  The metric is HBM GB/s of algorithmic bytes
(packed codes + scales/zeros + x + y), plus the fraction of the measured
HBM copy peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Under torchrun (N > 1) every rank runs its own replica of the workload
("weak" scaling: the path needs no exchange); rank 0 prints one JSON line.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the
same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "fused dequant-matmul: HBM GB/s (M=1 GEMV), TFLOP/s (M≥128), % roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

WORKLOADS = {
    # name: (shape set, layers, mode, bits, group, M, workload seed)
    "qwen2.5-0.5b-int4-decode": ("qwen2.5-0.5b", 24, "packed", 4, 64, 1, 1),
    "qwen3-0.6b-rtn3-decode": ("qwen3-0.6b", 28, "runtime", 3, 64, 1, 2),
    "qwen3-0.6b-rtn3-channel-decode": ("qwen3-0.6b", 28, "runtime", 3, 0, 1, 2),
    "qwen3-0.6b-fp16-decode": ("qwen3-0.6b", 28, "runtime", 16, 64, 1, 2),
    "qwen3-8b-int4-decode": ("qwen3-8b", 36, "packed", 4, 64, 1, 4),
    "qwen3-8b-int4-decode-m16": ("qwen3-8b", 36, "packed", 4, 64, 16, 4),
    "qwen3-8b-rtn3-decode": ("qwen3-8b", 36, "runtime", 3, 64, 1, 4),
    "qwen3-8b-rtn3-decode-m16": ("qwen3-8b", 36, "runtime", 3, 64, 16, 4),
    # prefill: bf16 x, tcgen05 tensor-core GEMM; packed int4 W, or fp16 W
    # re-quantized inline (runtime RTN at 3 bits, and the fp16 passthrough)
    "qwen2.5-0.5b-int4-prefill-m128": ("qwen2.5-0.5b", 24, "packed", 4, 64, 128, 3),
    "qwen2.5-0.5b-int4-prefill-m2048": ("qwen2.5-0.5b", 24, "packed", 4, 64, 2048, 3),
    "qwen2.5-0.5b-rtn3-prefill-m128": ("qwen2.5-0.5b", 24, "runtime", 3, 64, 128, 3),
    "qwen2.5-0.5b-rtn3-prefill-m2048": ("qwen2.5-0.5b", 24, "runtime", 3, 64, 2048, 3),
    "qwen2.5-0.5b-fp16-prefill-m2048": ("qwen2.5-0.5b", 24, "runtime", 16, 64, 2048, 3),
    # the bit-width-independent precompute: ranges stored, scale/zero in-kernel
    "qwen3-0.6b-rtn3range-decode": ("qwen3-0.6b", 28, "range", 3, 64, 1, 2),
    # Qwen3-0.6B's tied LM head (fp16 passthrough) reduced to a token id
    "qwen3-0.6b-lmhead-argmax": ("qwen3-0.6b-lmhead", 1, "runtime", 16, 64, 1, 2),
}
# The lever sweep 16 -> 2 of the Qwen3-0.6B set, per group and per channel.
for _b in (2, 4, 5, 6, 7, 8):
    WORKLOADS[f"qwen3-0.6b-rtn{_b}-decode"] = ("qwen3-0.6b", 28, "runtime", _b, 64, 1, 2)
for _b in (2, 4, 5, 6, 7, 8):
    WORKLOADS[f"qwen3-0.6b-rtn{_b}-channel-decode"] = ("qwen3-0.6b", 28, "runtime", _b, 0, 1, 2)
# The 1024 x 1024 single layer (seed 0) at bits {2, 3, 4, 8}, per group and
# per channel: one matmul per step, L2 flushed before each timed step.
for _b in (2, 3, 4, 8):
    WORKLOADS[f"single-1024-rtn{_b}-decode"] = ("single-1024", 1, "runtime", _b, 64, 1, 0)
    WORKLOADS[f"single-1024-rtn{_b}-channel-decode"] = ("single-1024", 1, "runtime", _b, 0, 1, 0)


def is_argmax(name: str) -> bool:
    return WORKLOADS[name][0] == "qwen3-0.6b-lmhead"


def is_tiny(name: str) -> bool:
    """Workloads far smaller than L2: each timed step is preceded by an L2
    flush (outside the timed region) and timed on its own."""
    return WORKLOADS[name][0] == "single-1024"


def is_prefill(name: str) -> bool:
    return WORKLOADS[name][5] >= 64
DEFAULT_WORKLOAD = "qwen2.5-0.5b-int4-decode"


# ---------------------------------------------------------------------------
# host-side helpers (no GPU needed; covered by the CPU tests)
# ---------------------------------------------------------------------------

def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained",
                                                     d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def workload_bytes(name: str) -> int:
    shape_set, layers, mode, bits, group, M, _ = WORKLOADS[name]
    xb = 2 if is_prefill(name) else 4
    return sum(wl.gemv_bytes(m.K, m.N, M, mode, bits, m.K if group == 0 else group,
                             x_bytes_per_elem=xb)
               for m in wl.layer_set(shape_set, layers))


def workload_flops(name: str) -> int:
    shape_set, layers, _, _, _, M, _ = WORKLOADS[name]
    return sum(2 * M * m.N * m.K for m in wl.layer_set(shape_set, layers))


def decode_kernel(name: str) -> str:
    """The decode kernel the library picks for a workload's grouped call:
    the streaming kernels when the call has at least 74 row blocks of 128
    (half the SMs), else the general GEMV."""
    shape_set, layers, mode, bits, _, M, _ = WORKLOADS[name]
    units = sum(-(-m.N // 128) for m in wl.layer_set(shape_set, layers))
    if units < 74:
        return "general"
    if M <= 4:
        return "stream"
    if M <= 16 and (mode == "packed" or bits <= 8):
        return "tc"
    return "general"


def launches_per_step(name: str, count: int) -> int:
    """Kernel launches the library makes for one grouped call (its own
    chunking of the descriptor list: 80 matrices per tensor-core GEMM
    launch; 168 per streaming decode launch, plus the activation pre-pass
    before each launch of the tensor-core decode kernel; 368 x 16-row
    chunks of M for the general GEMV)."""
    M = WORKLOADS[name][5]
    if is_prefill(name):
        return -(-count // 80)
    extra = 2 if is_argmax(name) else 0       # the two reduction kernels
    kind = decode_kernel(name)
    if kind == "stream":
        return -(-count // 168) + extra
    if kind == "tc":
        return 2 * -(-count // 168) + extra
    return -(-M // 16) * -(-count // 368) + extra


KERNEL_SOURCES = {"decode": ("bc_gemv_stream.cu", "bc_gemv.cu", "bc_internal.cuh", "bc_tc.cuh",
                             "bc_rtn.cuh"),
                  "prefill": ("bc_gemm_sm100.cu", "bc_internal.cuh", "bc_tc.cuh", "bc_rtn.cuh")}


def kernel_source_digest(kind: str = "decode") -> str:
    """Digest of the sources of the kernels a workload runs; a recorded DRAM
    traffic figure is only reported while it still matches."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        path = os.path.join(ROOT, "quantized_matmul_02_b200", "csrc", f)
        if os.path.exists(path):
            with open(path, "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(name: str):
    """DRAM bytes per launch from a committed ncu summary, if the summary's
    kernel-source digest matches the current sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"traffic_{name}.txt")
    try:
        fields = dict(line.split(":", 1) for line in open(path) if ":" in line)
    except OSError:
        return None
    kind = "prefill" if name in WORKLOADS and is_prefill(name) else "decode"
    if fields.get("source_digest", "").strip() != kernel_source_digest(kind):
        return None
    try:
        return int(fields["dram_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


def aggregate_times(times_ms, n_gpus: int, units_per_rank: float):
    """Whole-job throughput from per-rank elapsed times: the job takes the
    slowest rank's time; every rank processed `units_per_rank`."""
    t = max(times_ms)
    return {"ms": t, "value": units_per_rank * n_gpus / (t / 1e3)}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML on a thread."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown",
               0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self._stop = [], threading.Event()
        self.window = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report no clocks
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
                r = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def in_window(self, t0, t1):
        return [s for s in self.samples if t0 <= s[0] <= t1]

    def summary(self, extra=None):
        """Median SM clock and throttle reasons over the samples taken inside
        the timed region.  A timed region shorter than the sampling period
        holds none; then `extra` = (t0, t1, what) names an untimed window of
        the same step loop, sampled instead and labelled as such."""
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0}
        t0, t1 = self.window
        inside = self.in_window(t0, t1)
        used, source = inside, "timed region"
        if not inside and extra is not None:
            used, source = self.in_window(extra[0], extra[1]), extra[2]
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "samples_in_timed_region": 0,
                    "source": "no sample fell inside the timed region"}
        reasons = set()
        for _, _, r in used:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in used),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(used), "samples_in_timed_region": len(inside),
                "source": source}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--copies", type=int, default=0,
                    help="weight copies rotated between steps (0 = enough to "
                         "exceed 4x the L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="run only the first N layers of the workload (a smaller "
                         "case of the same kernels, e.g. for a profiler capture)")
    args = ap.parse_args(argv)
    if args.layers:
        w = list(WORKLOADS[args.workload])
        w[1] = min(w[1], args.layers)
        WORKLOADS[args.workload] = tuple(w)
    return args


# ---------------------------------------------------------------------------
# workload construction on the GPU
# ---------------------------------------------------------------------------

def build_workload(qmm, torch, name: str, copies: int):
    """Upload the seeded fp16 weights, run the one-time precompute (group
    params / int4 pack) with the library, and return `copies` independent
    device copies of the step's inputs plus the shared x / y buffers."""
    shape_set, layers, mode, bits, group, M, seed = WORKLOADS[name]
    mats = wl.layer_set(shape_set, layers)
    sigma = wl.SIGMA[shape_set]
    prefill = is_prefill(name)
    # every distinct x lives in one device buffer and every y in another, so a
    # step's inputs and outputs each cross PCIe as one copy (e2e)
    x_keys, x_off, x_total = [], {}, 0
    for m in mats:
        key = (m.layer, m.x_tag)
        if key not in x_off:
            x_off[key] = (x_total, m.K)
            x_keys.append(key)
            x_total += M * m.K
    x_all_host = np.empty(x_total, dtype=np.int16 if prefill else np.float32)
    for key in x_keys:
        off, K = x_off[key]
        xh = wl.activation(seed, key[0], key[1], M, K)
        x_all_host[off:off + M * K] = (wl.bf16_bits(xh).view(np.int16) if prefill
                                       else xh).reshape(-1)
    x_all_dev = torch.from_numpy(x_all_host).cuda()
    if prefill:
        x_all_dev = x_all_dev.view(torch.bfloat16)
    xs_dev = {key: x_all_dev[off:off + M * K].view(M, K)
              for key, (off, K) in x_off.items()}
    y_all_dev = torch.empty(sum(M * m.N for m in mats), dtype=torch.float32, device="cuda")
    per_copy = [[] for _ in range(copies)]
    ys = []
    y_at = 0
    for m in mats:
        key = (m.layer, m.x_tag)
        W = torch.from_numpy(wl.weight(seed, m.layer, m.name, m.K, m.N, sigma)).cuda()
        if mode == "packed":
            s, z = qmm.group_params(W, 4, 64, torch.float16)
            Wk = qmm.pack_int4(W, s, z)
            del W
        elif bits == 16:
            s = z = None
            Wk = W
        elif mode == "range":
            s, z = qmm.group_minmax(W, group), None
            Wk = W
        else:
            s, z = qmm.group_params(W, bits, group, torch.float32)
            Wk = W
        y = y_all_dev[y_at:y_at + M * m.N].view(M, m.N)
        y_at += M * m.N
        ys.append(y)
        for c in range(copies):
            if c == 0:
                per_copy[c].append((xs_dev[key], Wk, s, z, y))
            else:
                per_copy[c].append((xs_dev[key], Wk.clone(),
                                    None if s is None else s.clone(),
                                    None if z is None else z.clone(), y))
    torch.cuda.synchronize()
    descs = [qmm.make_descs(items) for items in per_copy]
    return {"mats": mats, "descs": descs, "x_all_host": x_all_host, "x_all_dev": x_all_dev,
            "xs_dev": xs_dev, "y_all_dev": y_all_dev, "ys": ys, "per_copy": per_copy,
            "mode": mode, "bits": bits, "group": group, "M": M}


def _oracle_x(name: str, seed: int, m) -> np.ndarray:
    """The activation exactly as the GPU path sees it, as fp64."""
    M = WORKLOADS[name][5]
    x = wl.activation(seed, m.layer, m.x_tag, M, m.K)
    if is_prefill(name):
        x = wl.bf16_to_f32(wl.bf16_bits(x))
    return x.astype(np.float64)


def cpu_baseline_sample(name: str, target_s: float = 12.0):
    """The oracle (as it stands) on a bounded sample of the workload: for
    whole matrices of the first layers, dequantize the codes and multiply
    (the work one GPU step does), until about `target_s` seconds of that
    work have passed.  When one pass over the set takes less, the matrices
    prepared in the first pass (up to ~1 GB of weights) are run again."""
    import oracle
    shape_set, layers, mode, bits, group, M, seed = WORKLOADS[name]
    mats = wl.layer_set(shape_set, layers)
    sigma = wl.SIGMA[shape_set]
    done_bytes, done_flops, spent = 0, 0, 0.0
    done = 0
    cache, cache_bytes = [], 0

    def work(item):
        x, W, q, s, z, g = item
        t0 = time.perf_counter()
        if mode == "runtime" and bits == 16:
            oracle.matmul(x, oracle.half_to_f64(W))
        else:
            if mode != "packed":    # runtime mode re-derives the codes per step
                s, z = oracle.group_params(W, bits, g, False)
                q = oracle.codes(W, s, z, bits, g)
            oracle.matmul(x, oracle.dequant(q, s, z, g))
        return time.perf_counter() - t0

    for m in mats:
        W = wl.weight(seed, m.layer, m.name, m.K, m.N, sigma)
        x = _oracle_x(name, seed, m)
        g = m.K if group == 0 else group
        q = s = z = None
        if not (mode == "runtime" and bits == 16):
            s, z = oracle.group_params(W, bits, g, mode == "packed")
            q = oracle.codes(W, s, z, bits, g)
        item = (x, W, q, s, z, g)
        spent += work(item)
        mb = wl.gemv_bytes(m.K, m.N, M, mode, bits, g,
                           x_bytes_per_elem=2 if is_prefill(name) else 4)
        mf = 2 * M * m.N * m.K
        done_bytes += mb
        done_flops += mf
        done += 1
        if cache_bytes < (1 << 30):
            cache.append((item, mb, mf))
            cache_bytes += W.nbytes + (q.nbytes if q is not None else 0)
        if spent >= target_s:
            break
    passes = 1
    while spent < target_s and cache:
        for item, mb, mf in cache:
            spent += work(item)
            done_bytes += mb
            done_flops += mf
            done += 1
            if spent >= target_s:
                break
        passes += 1
    if is_prefill(name):
        value, unit = done_flops / spent / 1e12, "TFLOP/s"
    else:
        value, unit = done_bytes / spent / 1e9, "GB/s"
    return {"value": value, "unit": unit,
            "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{done} matrix products over {min(len(cache), len(mats))} of the "
                      f"{len(mats)} matrices of {name} (first layers, {passes} passes), "
                      f"fp64 dequant + matmul, {spent:.1f} s"}


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def _reference_sample(name: str, rows: int):
    """Layer 0's matrices of the workload, first `rows` rows of each, with
    the codes precomputed (the one-time part): what one oracle step eats."""
    import oracle
    shape_set, layers, mode, bits, group, M, seed = WORKLOADS[name]
    out = []
    for m in wl.layer_set(shape_set, 1):
        n = min(rows, m.N)
        W = wl.weight(seed, m.layer, m.name, m.K, m.N, wl.SIGMA[shape_set])[:n]
        x = _oracle_x(name, seed, m)
        g = m.K if group == 0 else group
        item = {"W": W, "x": x, "g": g,
                "bytes": wl.gemv_bytes(m.K, n, M, mode, bits, g)}
        if not (mode == "runtime" and bits == 16):
            s, z = oracle.group_params(W, bits, g, mode == "packed")
            item.update(s=s, z=z, q=oracle.codes(W, s, z, bits, g))
        out.append(item)
    return out


def _reference_pass(name: str, sample) -> None:
    import oracle
    _, _, mode, bits, _, _, _ = WORKLOADS[name]
    for it in sample:
        if mode == "runtime" and bits == 16:
            oracle.matmul(it["x"], oracle.half_to_f64(it["W"]))
            continue
        s, z, q = it["s"], it["z"], it["q"]
        if mode != "packed":      # runtime mode re-derives the codes per step
            s, z = oracle.group_params(it["W"], bits, it["g"], False)
            q = oracle.codes(it["W"], s, z, bits, it["g"])
        oracle.matmul(it["x"], oracle.dequant(q, s, z, it["g"]))


def run_reference(args, rank, world):
    """The oracle as it stands, timed on this host's cores: each step is one
    pass over a bounded sample of the workload (the first rows of every
    matrix of layer 0), sized so the whole run stays within ~2 minutes."""
    if rank != 0:
        return 0
    import oracle
    name = args.workload
    rows = 512
    sample = _reference_sample(name, rows)
    t0 = time.perf_counter()
    _reference_pass(name, sample)
    one = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    if one > budget:
        rows = max(8, int(rows * budget / one))
        sample = _reference_sample(name, rows)
    for _ in range(args.warmup):
        _reference_pass(name, sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _reference_pass(name, sample)
    spent = time.perf_counter() - t0
    sbytes = sum(it["bytes"] for it in sample)
    value = sbytes * args.steps / spent / 1e9
    desc = (f"first {rows} rows of each of layer 0's {len(sample)} matrices "
            f"({sbytes} algorithmic bytes per step), fp64 oracle")
    line = {"metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": spent / max(1, args.steps) * 1e3,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": name, "sample": desc},
            "cpu_baseline": {"value": value, "unit": "GB/s",
                             "cores": oracle.threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "GB/s",
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, rank, world, local_rank):
    import torch
    import quantized_matmul_02_b200 as qmm
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    name = args.workload
    shape_set, layers, mode, bits, group, M, _ = WORKLOADS[name]
    step_bytes = workload_bytes(name)
    l2 = torch.cuda.get_device_properties(local_rank).L2_cache_size
    copies = args.copies or max(2, int(np.ceil(4 * l2 / step_bytes)) + 1)
    copies = 1 if is_tiny(name) else min(copies, 8)
    W = build_workload(qmm, torch, name, copies)
    mode_id = {"packed": qmm.BC_MODE_PACKED_INT4, "range": qmm.BC_MODE_RUNTIME_RANGE,
               "runtime": qmm.BC_MODE_RUNTIME}[mode]
    prefill = is_prefill(name)
    argmax = is_argmax(name)
    x_dtype = qmm.BC_BF16 if prefill else qmm.BC_F32
    if argmax:
        m0 = W["mats"][0]
        ws_bytes = qmm.workspace_size_argmax(M, m0.N, m0.K, mode_id, x_dtype)
        token = torch.empty((M,), dtype=torch.int32, device="cuda")
    else:
        ws_bytes = max(qmm.workspace_size_batched(d, M, mode_id, x_dtype) for d in W["descs"])
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    # The weights are fixed for the whole run, so decode steps may start while
    # the previous step finishes (BC_FLAG_STATIC_WEIGHTS; x and y still wait).
    def step(i):
        if argmax:      # the LM head reduced to one token id per x row
            xx, Wk, s, z, _ = W["per_copy"][i % copies][0]
            st = qmm.lib.bc_matmul_q_argmax(
                xx.data_ptr(), x_dtype, Wk.data_ptr(), None if s is None else s.data_ptr(),
                None if z is None else z.data_ptr(), M, Wk.shape[0], xx.shape[1], bits, group,
                mode_id, token.data_ptr(), ws.data_ptr(), ws.numel(), stream.cuda_stream)
            if st != qmm.BC_OK:
                raise qmm.BCError(st, "bc_matmul_q_argmax")
            return
        qmm.matmul_q_batched(W["descs"][i % copies], M, bits, group, mode_id,
                             x_dtype=x_dtype, workspace=ws, static_weights=True)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.05)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    start.record(stream)
    for i in range(args.steps):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if dist:
        dist.barrier()
    sampler.mark(t0, t1)
    clock_extra = None
    if not sampler.in_window(t0, t1):
        # the timed region was shorter than the sampling period: keep the
        # same step loop running, untimed, for ~0.2 s and sample that
        c0 = time.perf_counter()
        i = args.steps
        while time.perf_counter() - c0 < 0.2:
            for _ in range(20):
                step(i)
                i += 1
            torch.cuda.synchronize()
        clock_extra = (c0, time.perf_counter(),
                       "untimed continuation of the same step loop (0.2 s), "
                       "the timed region being shorter than the sampling period")
    time.sleep(0.02)
    sampler.stop()
    elapsed_ms = start.elapsed_time(end)
    hot_ms = None
    if is_tiny(name):
        # far smaller than L2: time each step alone after writing a buffer
        # larger than L2, and report that; the back-to-back figure is "hot"
        hot_ms = elapsed_ms
        flush = torch.empty(4 * l2, dtype=torch.uint8, device="cuda")
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i, (a, b) in enumerate(evs):
            flush.fill_(i & 0xFF)
            a.record(stream)
            step(i)
            b.record(stream)
        torch.cuda.synchronize()
        elapsed_ms = sum(a.elapsed_time(b) for a, b in evs)
        del flush
    times = [elapsed_ms]
    if dist:
        t = torch.tensor([elapsed_ms], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        times = [float(t.item())]
    step_flops = workload_flops(name)
    # units of the metric per step: GB (decode GEMV) or TFLOP (prefill GEMM)
    step_units = step_flops / 1e12 if prefill else step_bytes / 1e9
    unit = "TFLOP/s" if prefill else "GB/s"
    agg = aggregate_times(times, world, step_units * args.steps)
    ms_per_step = agg["ms"] / args.steps

    # ---- end to end through the public API: pinned host x in, y out ----
    x_pinned = torch.from_numpy(W["x_all_host"]).pin_memory()
    if prefill:
        x_pinned = x_pinned.view(torch.bfloat16)
    out_dev = token if argmax else W["y_all_dev"]     # argmax: one token id per row
    y_pinned = torch.empty(out_dev.shape, dtype=out_dev.dtype).pin_memory()
    h2d = x_pinned.numel() * x_pinned.element_size()
    d2h = y_pinned.numel() * y_pinned.element_size()

    def e2e_step(i):      # every x of the step in, the step, every output out
        W["x_all_dev"].copy_(x_pinned, non_blocking=True)
        step(i)
        y_pinned.copy_(out_dev, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    e_steps = max(10, min(args.steps, 200))
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    es.record(stream)
    for i in range(e_steps):
        e2e_step(i)
    ee.record(stream)
    torch.cuda.synchronize()
    e_ms = es.elapsed_time(ee)
    if dist:
        t = torch.tensor([e_ms], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e_ms = float(t.item())
    e2e_value = step_units * e_steps * world / (e_ms / 1e3)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = measured_peaks()
    # one launch of the dominant kernel per step, back to back on one stream:
    # its average duration is the timed region over the steps
    avg_launch_ms = elapsed_ms / args.steps
    traffic = recorded_traffic(name)
    if prefill:
        achieved = step_flops / (avg_launch_ms / 1e3) / 1e12
        # a prefill step lasts milliseconds, not seconds: the burst figure
        roof = {"bound": "tensor", "achieved": achieved,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "traffic": traffic,
                "peak_source": f"{peaks['source']} dense bf16, burst "
                               "(MEASURED_PEAKS.json bf16_tflops); sustained "
                               f"{peaks['bf16_tflops_sustained']}",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "hbm_gbs_achieved": step_bytes / (avg_launch_ms / 1e3) / 1e9,
                "kernel": "gemm_kernel (bc_gemm_sm100.cu)",
                "avg_step_us": avg_launch_ms * 1e3}
    else:
        achieved = step_bytes / (avg_launch_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "traffic": traffic,
                "peak_source": f"{peaks['source']} copy bandwidth "
                               "(MEASURED_PEAKS.json hbm_gbs)",
                "kernel": {"stream": "gemv_stream_kernel (bc_gemv_stream.cu)",
                           "tc": "gemv_tc_kernel (bc_gemv_stream.cu)",
                           "general": "gemv_kernel (bc_gemv.cu)"}[decode_kernel(name)],
                "avg_step_us": avg_launch_ms * 1e3}
    line = {
        "metric": METRIC, "value": agg["value"], "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if prefill else "f32",
        "data": "synthetic",
        "config": {"workload": name, "shape_set": shape_set, "layers": layers,
                   "matrices": len(W["mats"]), "mode": mode, "bits": bits,
                   "group": group if group else "per-channel", "M": M,
                   "weights": {"packed": "int4 packed, fp16 scale/zero per 64-block",
                               "runtime": "fp16, runtime RTN" if bits != 16
                               else "fp16 passthrough",
                               "range": "fp16, runtime RTN from stored group ranges "
                                        "(scale/zero derived in the kernel)"}[mode],
                   "x": "bf16" if prefill else "fp32", "bytes_per_step": step_bytes,
                   "flops_per_step": step_flops,
                   "l2": (f"L2 flushed ({4 * l2 / 1e6:.0f} MB written) before each timed "
                          "step; each step timed on its own"
                          if is_tiny(name) else
                          f"inputs larger than L2: {copies} weight copies "
                          f"({copies * step_bytes / 1e6:.0f} MB) rotated between "
                          f"steps, L2 {l2 / 1e6:.0f} MB"),
                   "launch": ("one call per step: the GEMV, then two reduction kernels "
                              "(token id per row)" if argmax else
                              "one grouped launch per step; decode steps launched "
                              "as programmatic dependent launches (static weights)")},
        "roofline": roof,
        **({"hot": {"us_per_step": hot_ms / args.steps * 1e3,
                    "value": step_units * args.steps / (hot_ms / 1e3), "unit": unit,
                    "note": "steps back to back, weights resident in L2"}}
           if hot_ms is not None else {}),
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "ms_per_step": e_ms / e_steps, "steps": e_steps},
        "gpu_launches": args.steps * launches_per_step(name, len(W["mats"])),
        "clocks": sampler.summary(clock_extra),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_sample(name)
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
