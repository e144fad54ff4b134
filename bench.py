#!/usr/bin/env python
"""Benchmark of MLA decode attention (ETAP form) on B200.

One step = one pass of the whole decode path over one batch: split-KV plan,
ETAP decode kernel, and the log-sum-exp merge of the split-KV partials (inside
the CTA-pair kernel; a combine kernel behind the M = 256 kernel that serves the
bf16 cache above 16 query columns).  Default workload: B=16 sequences,
16 heads, one query token, 65536 contiguous cache rows each (1.21 GB of bf16
latent KV, larger than the 126 MB L2, so no flush is needed between steps;
workloads smaller than L2 get a 256 MB write before every timed step, outside
the CUDA events around the step).

Reported value: whole-job KV throughput in TB/s (algorithmic bytes: 1152 per
cached token read once, 580 for the FP8 cache) over the max-over-ranks device
time of K steps, replayed from CUDA graphs of the same calls (--no-graph launches
them from the host).  The line also carries TFLOPS (2*(576+512) flops per visible
(query column, token) pair), the decode kernel's roofline fraction (CUDA-event
timing of back-to-back launches of that kernel on its stream, taken right before
the timed steps), an end-to-end figure through the C ABI with host buffers, the
fp64 oracle timed on the host as a CPU baseline, and GPU clocks sampled while the
steps run.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
  python bench.py --workload NAME --form untransposed   # the same decode in the S = Q K^T form
  python bench.py --ablation    # transposed vs untransposed tensor-core cost per KV tile

N > 1 runs under torchrun, one process per GPU; every rank decodes its own
batch (independent sequences, no collective on the data path: weak scaling).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MLA decode TB/s & TFLOPS (B=16,h=16,64K KV) as % of B200 roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
L2_BYTES = 126e6              # B200 L2: workloads below this are timed with an L2 flush between steps
FLUSH_BYTES = 256 << 20       # the flush writes a buffer twice the L2 size
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
_CSRC = "mla_decode_attention_etap_b200/csrc/"
# The sources each decode kernel is compiled from (its ncu traffic figure is valid while they hash the
# same); the plan and combine kernels are separate kernels with their own sources.
KERNEL_SOURCES = {
    "etap_pair_kernel": [_CSRC + f for f in ("etap_pair_kernel.cuh", "etap_common.cuh", "ptx_sm100.cuh",
                                             "plan_core.h", "merge.cuh")],
    "etap_duo_kernel": [_CSRC + f for f in ("etap_duo_kernel.cuh", "etap_common.cuh", "ptx_sm100.cuh",
                                            "plan_core.h")],
}
PROFILE_SUMMARIES = {
    "etap_pair_kernel": [os.path.join(ROOT, "profiles", "etap_pair_kernel_ncu.md"),
                         os.path.join(ROOT, "profiles", "etap_pair_kernel_e4m3_ncu.md")],
    "etap_duo_kernel": [os.path.join(ROOT, "profiles", "etap_duo_kernel_ncu.md")],
}


def decode_kernel_of(ncols: int, fp8: bool) -> str:
    """The decode kernel a shape runs on (plan_core.h: uses_duo)."""
    return "etap_duo_kernel" if (not fp8 and ncols > 16) else "etap_pair_kernel"

WORKLOADS = {
    "b16_h16_64k": dict(batch=16, heads=16, seqlen=65536),
    "b16_h16_32k": dict(batch=16, heads=16, seqlen=32768),
    "b16_h16_16k": dict(batch=16, heads=16, seqlen=16384),
    "b16_h16_4k": dict(batch=16, heads=16, seqlen=4096),
    "b1_h16_1k": dict(batch=1, heads=16, seqlen=1024),
    "b64_h16_paged": dict(kind="b64_paged"),
    "b32_h128_paged": dict(kind="b32_h128"),
    "b16_h16_q4_causal": dict(kind="q4_causal"),
    "b16_h16_ragged_q4_causal": dict(kind="ragged_q4_causal"),
    "b16_h16_append_q16": dict(kind="append_q16"),
    # FP8 latent cache (E4M3 codes + one fp32 scale per row): 580 bytes per cached token
    "b16_h16_64k_fp8": dict(batch=16, heads=16, seqlen=65536, fp8=True),
    "b16_h16_16k_fp8": dict(batch=16, heads=16, seqlen=16384, fp8=True),
    "b16_h16_4k_fp8": dict(batch=16, heads=16, seqlen=4096, fp8=True),
    "b64_h16_paged_fp8": dict(kind="b64_paged_fp8"),
    "b16_h16_q4_causal_fp8": dict(kind="q4_causal_fp8"),
    "b32_h128_paged_fp8": dict(kind="b32_h128_fp8"),
    "b16_h16_append_q16_fp8": dict(kind="append_q16_fp8"),
}


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def weak_scaling_value(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: units all ranks processed / max-over-ranks time."""
    return units_per_rank * world / seconds_max


# ---------------------------------------------------------------- workload
def make_workload(name: str, rank: int, device):
    from mla_decode_attention_etap_b200 import workloads as W
    spec = WORKLOADS[name]
    seed = 1000 * rank
    kind = spec.get("kind")
    if kind == "b64_paged":
        return W.workload_b64_h16_paged(seed=seed, device=device), "mla_decode_b64_h16_q1_Lunif1to65536_paged64"
    if kind == "b32_h128":
        return W.workload_b32_h128_paged(seed=seed, device=device), "mla_decode_b32_h128_q1_Lunif8192to32768_paged64"
    if kind == "q4_causal":
        return (W.workload_b16_h16_q4_causal(seed=seed, device=device),
                "mla_decode_b16_h16_q4_causal_L32768_spikes5pct_x8")
    if kind == "ragged_q4_causal":
        return (W.workload_b16_h16_ragged_q4_causal(seed=seed, device=device),
                "mla_decode_b16_h16_ragged_q1to4_causal_L32768_spikes5pct_x8")
    if kind == "append_q16":
        return (W.workload_b16_h16_append_q16(seed=seed, device=device),
                "mla_decode_b16_h16_append_q16_causal_L32768")
    if kind == "q4_causal_fp8":
        return (W.make_workload(16, 16, [32768] * 16, q_len=4, causal=True, seed=seed, device=device,
                                spike_frac=0.05, spike_scale=8.0, kv_dtype="e4m3"),
                "mla_decode_b16_h16_q4_causal_L32768_spikes5pct_x8_e4m3cache")
    if kind == "b32_h128_fp8":
        lens = W.draw_seqlens(32, 8192, 32768, seed)
        return (W.make_workload(32, 128, lens, paged=True, seed=seed, device=device, kv_dtype="e4m3"),
                "mla_decode_b32_h128_q1_Lunif8192to32768_paged64_e4m3cache")
    if kind == "append_q16_fp8":
        return (W.make_workload(16, 16, [32768] * 16, q_len=16, causal=True, seed=seed, device=device,
                                kv_dtype="e4m3"),
                "mla_decode_b16_h16_append_q16_causal_L32768_e4m3cache")
    if kind == "b64_paged_fp8":
        return (W.workload_b64_h16_paged_fp8(seed=seed, device=device),
                "mla_decode_b64_h16_q1_Lunif1to65536_paged64_e4m3cache")
    fp8 = bool(spec.get("fp8"))
    w = W.make_workload(spec["batch"], spec["heads"], [spec["seqlen"]] * spec["batch"], seed=seed, device=device,
                        kv_dtype="e4m3" if fp8 else "bf16")
    return w, f"mla_decode_b{spec['batch']}_h{spec['heads']}_q1_L{spec['seqlen']}_contiguous" + (
        "_e4m3cache" if fp8 else "")


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained",
                                                                              pk["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def code_only(text: str) -> str:
    """Source text without // comments and blank lines: what the compiler sees, for the hash."""
    out = []
    for line in text.splitlines():
        code = line.split("//", 1)[0].rstrip()
        if code.strip():
            out.append(code)
    return "\n".join(out)


def kernel_source_hash(read=None, kernel: str = "etap_pair_kernel") -> str:
    """Hash of a decode kernel's sources (code only, so that comment edits keep a profile valid)."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        if read is None:
            with open(os.path.join(ROOT, rel)) as f:
                text = f.read()
        else:
            text = read(rel)
        h.update(code_only(text).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str = "etap_pair_kernel"):
    """DRAM bytes per decode launch from the committed ncu summaries, if taken on the current kernel source."""
    for path in PROFILE_SUMMARIES.get(kernel, []):
        try:
            text = open(path).read()
        except OSError:
            continue
        src = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
        if not src or src.group(1) != kernel_source_hash(kernel=kernel):
            continue
        m = re.search(rf"traffic_bytes_per_launch\[{re.escape(workload)}\]:\s*([0-9.eE+]+)", text)
        if m:
            return float(m.group(1))
    return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML (SM clock, max clock, throttle reasons) in a thread while the steps run."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting", 0x10: "sync_boost", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.idx, self.period = device_index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = None
            try:  # the CUDA device's own UUID: NVML indices ignore CUDA_VISIBLE_DEVICES
                import torch
                uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:  # pragma: no cover - NVML missing
            self.error = repr(e)
        return self

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception as e:  # pragma: no cover
                self.error = repr(e)
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=2)
        return False

    def summary(self):
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples),
               "window": "NVML polled every 5 ms from the first warm-up step to the end of the timed steps"}
        if self.error:
            out["error"] = self.error
        return out


# ---------------------------------------------------------------- CPU baseline (oracle)
def W_flops(seqlens, w, q_lens=None) -> int:
    """Algorithmic flops of the listed sequences of workload ``w`` (q_lens: their token counts)."""
    from mla_decode_attention_etap_b200 import workloads as W
    return W.algorithmic_flops(seqlens, w.q_len, w.num_heads, w.causal,
                               None if q_lens is None else [int(x) for x in q_lens])


def oracle_baseline(w, target_s: float = 12.0):
    """Time the fp64 oracle on whole sequences of the workload until ~target_s of CPU work."""
    import numpy as np
    from mla_decode_attention_etap_b200.workloads import bf16_bits
    from oracle import mla_oracle as om
    cores = len(os.sched_getaffinity(0))
    os.environ["OMP_NUM_THREADS"] = str(cores)
    om.build()
    done_bytes, done_flops, t_total, seqs = 0, 0, 0.0, []
    order = list(range(w.batch))
    for b in order:
        L = int(w.seqlens[b])
        if L == 0:
            continue
        q = bf16_bits(w.q[b:b + 1].cpu())
        ql = None if w.q_lens is None else w.q_lens[b:b + 1].numpy()
        run = _oracle_call(w, b, L)
        t0 = time.perf_counter()
        run(q, np.array([L], np.int32), ql)
        t_total += time.perf_counter() - t0
        done_bytes += L * (580 if w.fp8 else 1152)
        done_flops += W_flops([L], w, ql)
        seqs.append(b)
        if t_total >= target_s:
            break
    return {"value": done_bytes / t_total / 1e12, "unit": "TB/s", "cores": cores, "kind": "oracle",
            "tflops": done_flops / t_total / 1e12,
            "sample": f"{len(seqs)} whole sequence(s) of the workload (index {seqs[0]}..{seqs[-1]}), "
                      f"{done_bytes / 1e9:.3f} GB of KV, fp64 C oracle with OpenMP, {t_total:.2f} s"}


def _oracle_call(w, b: int, rows: int):
    """The oracle on the first `rows` cache rows of sequence b (bf16 or E4M3 cache) as a callable
    (q_bits, seqlens, q_lens) -> (O, LSE); the cache rows are gathered before it is timed."""
    from mla_decode_attention_etap_b200.workloads import bf16_bits
    from oracle import mla_oracle as om

    def seq_rows(t):
        L = int(w.seqlens[b])
        if w.block_table is None:
            out = t[b, :L]
        else:
            nb = (L + 63) // 64
            out = t[w.block_table[b, :nb].long().to(t.device)].reshape(nb * 64, *t.shape[2:])[:L]
        return out[:rows].cpu()

    if w.fp8:
        codes = seq_rows(w.kv8).numpy().reshape(1, rows, 576)
        sc = seq_rows(w.kv_scale).numpy().reshape(1, rows)
        return lambda q, sl, ql: om.mla_decode_fp8(q, codes, sc, sl, None, w.softmax_scale, w.causal, q_lens=ql)
    kv = bf16_bits(seq_rows(w.kv).reshape(1, rows, 576))
    return lambda q, sl, ql: om.mla_decode(q, kv, sl, None, w.softmax_scale, w.causal, q_lens=ql)


# ---------------------------------------------------------------- arms
def run_reference(args):
    """Reference arm: the fp64 oracle on the host, same workload/metric/unit, bounded sample per step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import torch
    w, wname = make_workload(args.workload, 0, "cpu")
    import numpy as np
    from mla_decode_attention_etap_b200.workloads import bf16_bits
    from oracle import mla_oracle as om
    cores = len(os.sched_getaffinity(0))
    os.environ["OMP_NUM_THREADS"] = str(cores)
    om.build()
    # one step = the oracle over a bounded slice of the workload: the first sequence, first 4096 rows
    b = 0
    L = min(int(w.seqlens[b]), args.reference_rows)
    run = _oracle_call(w, b, L)
    q = bf16_bits(w.q[b:b + 1].cpu())
    sl = np.array([L], np.int32)
    ql = None if w.q_lens is None else w.q_lens[b:b + 1].numpy()
    for _ in range(args.warmup):
        run(q, sl, ql)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run(q, sl, ql)
    dt = (time.perf_counter() - t0) / args.steps
    value = L * (580 if w.fp8 else 1152) / dt / 1e12
    sample = f"sequence 0, first {L} cache rows, all {w.num_heads} heads x {w.q_len} token(s), per step"
    line = {"metric": METRIC, "value": value, "unit": "TB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "tflops": W_flops([L], w, ql) / dt / 1e12,
            "config": {"workload": wname, "reference_sample": sample},
            "cpu_baseline": {"value": value, "unit": "TB/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist
    import mla_decode_attention_etap_b200 as mla
    from mla_decode_attention_etap_b200 import workloads as W

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    mla.lib()  # fails loudly when the CUDA library is missing

    w, wname = make_workload(args.workload, rank, dev)
    if args.form == "untransposed" and (w.fp8 or w.q_lens is not None):
        raise SystemExit("--form untransposed: bf16 cache with one q_len for every sequence only")
    q, kv, sl = w.q, w.kv, w.seqlens.to(dev)
    bt = w.block_table.to(dev) if w.block_table is not None else None
    B, q_len, h = w.batch, w.q_len, w.num_heads
    dec = mla.MlaDecoder(B, q_len, h, device=dev)
    o = torch.empty(B, q_len, h, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, q_len, h, dtype=torch.float32, device=dev)
    seqlens = [int(x) for x in w.seqlens]
    fp8 = w.fp8
    if fp8:
        kv, kv_scale = w.kv8, w.kv_scale  # the cache the decode reads: E4M3 codes + row scales
    kv_bytes = W.algorithmic_kv_bytes(seqlens, fp8=fp8)
    q_lens = w.q_lens.to(dev) if w.q_lens is not None else None
    flops = W.algorithmic_flops(seqlens, q_len, h, w.causal, None if w.q_lens is None else w.q_lens.tolist())
    stream = torch.cuda.current_stream()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    def decode(q_, kv_, sl_, bt_, ql_, sc_=None):
        # the fused call: the split-KV merge runs inside the pair kernel, or in the combine kernel that
        # the M = 256 path launches behind its decode
        if args.form == "untransposed":
            mla.mla_decode_fwd_untransposed(q_, kv_, sl_, bt_, w.softmax_scale, w.causal, o, lse, dec.workspace,
                                            dec.n_sms, 0)
        elif fp8:
            mla.mla_decode_fwd_fp8(q_, kv_, sc_, sl_, bt_, w.softmax_scale, w.causal, o, lse, dec.workspace,
                                   dec.n_sms, 0, q_lens=ql_)
        else:
            mla.mla_decode_fwd(q_, kv_, sl_, bt_, w.softmax_scale, w.causal, o, lse, dec.workspace, dec.n_sms, 0,
                               q_lens=ql_)

    def decode_on(strm):
        if args.form == "untransposed":
            mla.mla_decode_fwd_untransposed(q, kv, sl, bt, w.softmax_scale, w.causal, o, lse, dec.workspace,
                                            dec.n_sms, 0, strm)
        elif fp8:
            mla.mla_decode_fwd_fp8(q, kv, kv_scale, sl, bt, w.softmax_scale, w.causal, o, lse, dec.workspace,
                                   dec.n_sms, 0, strm, q_lens=q_lens)
        else:
            mla.mla_decode_fwd(q, kv, sl, bt, w.softmax_scale, w.causal, o, lse, dec.workspace, dec.n_sms, 0, strm,
                               q_lens=q_lens)

    def step(i=None):
        dec.plan(sl)
        if i is not None:
            ev[i][0].record(stream)
        decode(q, kv, sl, bt, q_lens, kv_scale if fp8 else None)
        if i is not None:
            ev[i][1].record(stream)

    # L2 flush for inputs smaller than the 126 MB L2: a 256 MB write between timed iterations
    flush_l2 = kv_bytes < L2_BYTES and not args.no_flush
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush_l2 else None

    def flush():
        flush_buf.fill_(1)

    sampler = ClockSampler(local)
    with sampler:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        # The steps are replayed from CUDA graphs (one of G steps, one of a single step), so that
        # the host's per-call work (argument checks, tensor maps, two launches) is not what a short
        # step measures; the graphs hold exactly the launches of the eager steps (programmatic
        # launches become programmatic edges).
        graphs = None
        if not args.no_graph:
            g_steps = min(10, args.steps)
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            graphs = []
            with torch.cuda.stream(side):
                for n in (g_steps, 1):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=side):
                        for _ in range(n):
                            dec.plan(sl, stream=side)
                            decode_on(side)
                    graphs.append((n, g))
            stream.wait_stream(side)
            for n, g in graphs:  # warm replays
                g.replay()
            torch.cuda.synchronize()
        # the decode kernel alone, n_kern launches back to back after one plan (each a programmatic
        # dependent of the previous one, as in the steps; the plan in the workspace stays valid and
        # the in-kernel merge leaves its counters reset): its duration in a steady stream, taken
        # right before the timed region (sustained runs of this HBM-bound kernel slow down by up
        # to ~10 % after some tens of milliseconds, which later passes would see)
        n_kern = min(args.steps, 50)
        if flush_l2:
            # inputs smaller than L2: every launch starts from a flushed L2 (the flush is outside
            # the events), so the figure is the HBM-cold one
            kern_cold = []
            for _ in range(n_kern):
                dec.plan(sl)
                flush()
                kb0, kb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                kb0.record(stream)
                decode(q, kv, sl, bt, q_lens, kv_scale if fp8 else None)
                kb1.record(stream)
                kern_cold.append((kb0, kb1))
        else:
            dec.plan(sl)
            kb0, kb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            kb0.record(stream)
            for _ in range(n_kern):
                decode(q, kv, sl, bt, q_lens, kv_scale if fp8 else None)
            kb1.record(stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        # timed region: K whole steps back to back, nothing else in the stream (an event
        # between plan and decode would serialise their programmatic overlap); with inputs
        # smaller than L2, a flush of L2 before every step and events around each step instead
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        step_cold = []
        t_start.record(stream)
        if flush_l2:
            for _ in range(args.steps):
                flush()
                s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s0.record(stream)
                if graphs is None:
                    step()
                else:
                    graphs[1][1].replay()
                s1.record(stream)
                step_cold.append((s0, s1))
        elif graphs is None:
            for _ in range(args.steps):
                step()
        else:
            (gn, g_many), (_, g_one) = graphs
            for _ in range(args.steps // gn):
                g_many.replay()
            for _ in range(args.steps % gn):
                g_one.replay()
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        # more steps with CUDA events around each decode launch (no overlap with the plan)
        for i in range(n_kern):
            step(i)
        torch.cuda.synchronize()
        # attainable read bandwidth of the decode's TMA pattern on this GPU: the streaming probe
        # (same grid, split, slots and L2 prefetch, no computation) over the same bf16 cache tensor
        probe_s = None
        if not fp8:
            kv_flat = kv.reshape(-1, 576)
            probe_rows = (kv_flat.shape[0] // 128) * 128
            probe_err = torch.zeros(1, dtype=torch.int32, device=dev)
            probe_units = dec.n_sms // 2
            for _ in range(3):
                mla.mla_stream_probe(kv_flat[:probe_rows], probe_units, probe_err)
            pe0, pe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            pe0.record(stream)
            n_probe = max(3, min(args.steps, 50))
            for _ in range(n_probe):
                mla.mla_stream_probe(kv_flat[:probe_rows], probe_units, probe_err)
            pe1.record(stream)
            torch.cuda.synchronize()
            probe_s = pe0.elapsed_time(pe1) / 1e3 / n_probe
            if int(probe_err.item()) != 0:
                raise RuntimeError("streaming probe: a bounded wait ran out")
    status = dec.status()
    if status != 0:
        raise RuntimeError(f"device status {mla.STATUS.get(status, status)}")
    if flush_l2:
        step_all = [a.elapsed_time(b) / 1e3 for a, b in step_cold]
        step_s = statistics.mean(step_all)
        kern_cold_s = [a.elapsed_time(b) / 1e3 for a, b in kern_cold]
        kern_s = statistics.median(kern_cold_s)
    else:
        step_all = None
        step_s = t_start.elapsed_time(t_end) / 1e3 / args.steps
        kern_s = kb0.elapsed_time(kb1) / 1e3 / n_kern
    step_s_max = reduce_max(step_s, dev)
    kern_all = [a.elapsed_time(b) / 1e3 for a, b in ev[:n_kern]]
    # plan + decode per step, + the combine kernel behind the M = 256 decode (the pair kernel merges
    # its splits itself at n_sms = 148)
    launches = (3 if (decode_kernel_of(q_len * h, fp8) == "etap_duo_kernel" or args.form == "untransposed")
                else 2) * args.steps

    # ---------------- end to end through the C ABI: pinned host inputs in, outputs back, every step
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    hq = q.cpu().pin_memory()
    hkv = kv.cpu().pin_memory()
    hsc = kv_scale.cpu().pin_memory() if fp8 else None
    dsc = torch.empty_like(kv_scale) if fp8 else None
    hsl = w.seqlens.clone().pin_memory()
    hbt = w.block_table.clone().pin_memory() if w.block_table is not None else None
    ho = torch.empty_like(o, device="cpu").pin_memory()
    hl = torch.empty_like(lse, device="cpu").pin_memory()
    dq, dkv, dsl = torch.empty_like(q), torch.empty_like(kv), torch.empty_like(sl)
    dbt = torch.empty_like(bt) if bt is not None else None
    hql = w.q_lens.clone().pin_memory() if w.q_lens is not None else None
    dql = torch.empty_like(q_lens) if q_lens is not None else None
    h2d = (hq.numel() * 2 + hkv.numel() * hkv.element_size() + hsl.numel() * 4
           + (hbt.numel() * 4 if hbt is not None else 0) + (hql.numel() * 4 if hql is not None else 0)
           + (hsc.numel() * 4 if hsc is not None else 0))
    d2h = ho.numel() * 2 + hl.numel() * 4

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dkv.copy_(hkv, non_blocking=True)
        dsl.copy_(hsl, non_blocking=True)
        if dbt is not None:
            dbt.copy_(hbt, non_blocking=True)
        if dql is not None:
            dql.copy_(hql, non_blocking=True)
        if dsc is not None:
            dsc.copy_(hsc, non_blocking=True)
        dec.plan(dsl)
        decode(dq, dkv, dsl, dbt, dql, dsc)
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_s = reduce_max(e0.elapsed_time(e1) / 1e3 / e2e_steps, dev)

    if rank == 0:
        hbm_gbs, tc_tflops, tc_sust, peak_src = load_peaks()
        # a contraction takes the peak of its own operand type: E4M3 MMAs at the nominal 2x the measured bf16
        tc_ratio = 2.0 if fp8 else 1.0
        tc_tflops *= tc_ratio
        achieved_gbs = kv_bytes / kern_s / 1e9
        bound = "hbm" if (kv_bytes / (hbm_gbs * 1e9)) >= (flops / (tc_tflops * 1e12)) else "tensor"
        if bound == "hbm":
            roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_gbs, "unit": "GB/s",
                    "frac": achieved_gbs / hbm_gbs}
        else:
            ach = flops / kern_s / 1e12
            roof = {"bound": "tensor", "achieved": ach, "peak": tc_tflops, "unit": "TFLOP/s", "frac": ach / tc_tflops}
        kname = "untransposed_kernel" if args.form == "untransposed" else decode_kernel_of(q_len * h, fp8)
        roof["traffic"] = profiled_traffic(wname, kname)
        roof["peak_source"] = (f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})"
                               + ("; tensor peak = 2 x the measured bf16 GEMM peak (E4M3 operands, the nominal "
                                  "fp8 : bf16 ratio)" if fp8 else ""))
        if probe_s is not None:
            roof["attainable_read_gbs"] = probe_rows * 1152 / probe_s / 1e9
            roof["frac_of_attainable"] = roof["achieved"] / roof["attainable_read_gbs"] if bound == "hbm" else None
            roof["attainable_note"] = ("streaming probe: the decode's TMA read pattern (same grid, column split, "
                                       "5 V-pair slots, L2 prefetch) without computation, over the same cache")
        else:
            roof["attainable_read_gbs"] = None
            roof["attainable_note"] = "no streaming probe for the E4M3 cache's read pattern"
        if kname == "untransposed_kernel":
            roof["kernel"] = ("untransposed_kernel + combine_kernel (S = Q K^T form for the A/B comparison; both "
                              "inside the events)")
        elif kname == "etap_duo_kernel":
            roof["kernel"] = ("etap_duo_kernel + combine_kernel (the split merge, started on the SMs the decode "
                              "leaves; both inside the events)")
        else:
            roof["kernel"] = "etap_pair_kernel<PairCfg16E4>" if fp8 else "etap_pair_kernel"
        roof["kernel_ms"] = kern_s * 1e3
        roof["kernel_ms_isolated_mean"] = statistics.mean(kern_all) * 1e3
        roof["kernel_ms_isolated_median"] = statistics.median(kern_all) * 1e3
        if flush_l2:
            roof["kernel_timing"] = (f"median of CUDA events on the launch stream around each of {n_kern} decode "
                                     "launches, each after a plan and a 256 MB L2 flush (HBM-cold), right before "
                                     "the timed region; kernel_ms_isolated_*: events around each decode of "
                                     f"{n_kern} plan + decode steps after it, L2-warm")
            roof["kernel_ms_cold_best"] = min(kern_cold_s) * 1e3
        else:
            roof["kernel_timing"] = (f"CUDA events on the launch stream around {n_kern} decode launches issued back "
                                     "to back after one plan (each a programmatic dependent of the previous, as in "
                                     "the steps), right before the timed region; kernel_ms_isolated_*: events "
                                     f"around each decode of {n_kern} separate plan + decode steps after it (no "
                                     "overlap with the plan)")
        roof["tflops"] = flops / kern_s / 1e12
        roof["algorithmic_bytes_per_launch"] = kv_bytes
        roof["algorithmic_flops_per_launch"] = flops
        line = {
            "metric": METRIC,
            "value": weak_scaling_value(kv_bytes, world, step_s_max) / 1e12,
            "unit": "TB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": step_s_max * 1e3,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "e4m3" if fp8 else "bf16",
            "form": args.form,
            "data": "synthetic",
            "tflops": weak_scaling_value(flops, world, step_s_max) / 1e12,
            "config": {"workload": wname, "batch_per_gpu": B, "heads": h, "q_len": q_len,
                       "q_lens": None if w.q_lens is None else w.q_lens.tolist(),
                       "seqlens": (seqlens[0] if len(set(seqlens)) == 1 else
                                   f"{min(seqlens)}..{max(seqlens)} (mean {sum(seqlens) / len(seqlens):.0f})"),
                       "d_qk": 576, "d_v": 512, "kv_layout": "paged64" if bt is not None else "contiguous",
                       "kv_cache": ("E4M3 codes + fp32 scale per row (580 B/token)" if fp8 else
                                    "bf16 (1152 B/token)"),
                       "causal": bool(w.causal), "kv_bytes_per_gpu": kv_bytes,
                       "timed_launches": ("replayed from CUDA graphs (10-step and 1-step graphs of plan + decode)"
                                          if not args.no_graph else "launched from the host, one call each"),
                       "l2": ("inputs larger than L2 (no flush)" if not flush_l2 else
                              "inputs smaller than L2: a 256 MB write flushes L2 before every timed step, outside "
                              "the CUDA events around that step (value and ms_per_step: mean over the steps)"),
                       "parallelism": f"dp{world} (independent sequences per GPU, no collective)"},
            "roofline": roof,
            "e2e": {"value": weak_scaling_value(kv_bytes, world, e2e_s) / 1e12, "unit": "TB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "ms_per_step": e2e_s * 1e3},
            "gpu_launches": launches,
            **({"ms_per_step_median": statistics.median(step_all) * 1e3,
                "ms_per_step_best": min(step_all) * 1e3} if step_all else {}),
            "clocks": sampler.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_baseline(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()
    return 0


def run_ablation(args):
    """Transposed vs untransposed contraction cost per 128-row KV tile (the pages' padding argument):
    tensor-core instructions only, every SM, h in {16, 32, 64, 128}; one JSON line."""
    import torch
    import mla_decode_attention_etap_b200 as mla
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    tiles = 64
    cycles = torch.zeros(ctas, dtype=torch.int64, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    rows = []
    for heads in (16, 32, 64, 128):
        entry = {"heads": heads, "useful_flop_per_tile": 2 * 128 * heads * (576 + 512)}
        for form, fname in ((0, "transposed"), (1, "untransposed")):
            for streams, sname in ((1, "scores"), (2, "output"), (3, "both")):
                for _ in range(2):  # the first launch warms the clocks and the instruction cache
                    mla.mla_form_ablation(form, heads, streams, tiles, cycles, err)
                torch.cuda.synchronize()
                if int(err.item()) != 0:
                    raise RuntimeError("form ablation: a bounded wait ran out")
                cyc = cycles.max().item() / tiles
                entry[f"{fname}_{sname}_cycles_per_tile"] = round(cyc, 1)
            entry[f"{fname}_useful_flop_per_cycle_per_sm"] = round(
                entry["useful_flop_per_tile"] / entry[f"{fname}_both_cycles_per_tile"], 1)
        entry["untransposed_over_transposed"] = round(entry["untransposed_both_cycles_per_tile"] /
                                                      entry["transposed_both_cycles_per_tile"], 3)
        rows.append(entry)
    print(json.dumps({"ablation": "transposed vs untransposed MMAs per 128-row KV tile, bf16, d_qk 576, d_v 512",
                      "ctas": ctas, "tiles_per_cta": tiles, "rows": rows}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="b16_h16_64k")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps from the host instead of replaying them from CUDA graphs")
    ap.add_argument("--ablation", action="store_true",
                    help="print the transposed-vs-untransposed tensor-core cost table instead of a bench line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-flush", action="store_true",
                    help="do not flush L2 between timed steps of workloads smaller than L2 (L2-warm numbers)")
    ap.add_argument("--reference-rows", type=int, default=4096)
    ap.add_argument("--form", choices=["etap", "untransposed"], default="etap",
                    help="time the untransposed S = Q K^T decode instead of ETAP (the form comparison)")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps
    if args.ablation:
        return run_ablation(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
