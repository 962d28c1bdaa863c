"""Benchmark of the packed-varlen attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one call of the library's varlen_attention over the packed-varlen
causal prefill workload (batch 8, seqLen ~ U[64, 2048] seeded, headNum 32,
kvHeadNum 8, headSize 128, bf16, qkScale 1/sqrt(128)): one prefill kernel
launch into the op's workspace, which holds the op's schedule since its first
execution (ala_op_bind_workspace).  The metric is attention TFLOPS on valid
tokens: 4 * headSize * headNum * (allowed query/key pairs) per step.

Timing: W untimed warm-up steps, then K timed steps bracketed by a barrier
and a device synchronise; each step is timed with CUDA events on the launch
stream, with the L2 flushed (a 256 MiB write) before every step, outside its
events.  Under torchrun every rank runs the same workload on its own GPU
(independent sequences, no collective on the data path; weak scaling), and
the per-step time is the max over ranks.

Also reported on rank 0:
  * roofline of the prefill kernel against the measured dense bf16 peak;
  * e2e: the same metric through the public call with inputs copied from
    pinned host memory and the output copied back inside the timed region;
  * cpu_baseline: the fp64 oracle on the host cores over a bounded sample of
    the same workload's rows;
  * extra: the other workloads (paged ALiBi prefix encoder fp16, long ALiBi
    bf16 in both variants, the causal batch at head size 256, MLA decode/spec
    when built) measured the same way.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

PROFILE = os.path.join(ROOT, "profiles", "prefill_varlen_causal_bf16.md")
MLA_PROFILE = os.path.join(ROOT, "profiles", "mla_decode_qs1_bf16.md")
MLA_INT8_PROFILE = os.path.join(ROOT, "profiles", "mla_decode_qs1_int8.md")
PROFILE_D256 = os.path.join(ROOT, "profiles", "prefill_d256_varlen_causal_bf16.md")
KERNEL_SOURCES = ["paged_attention_varlen_b200/csrc/prefill.cu", "paged_attention_varlen_b200/csrc/ptx.cuh"]
D256_KERNEL_SOURCES = ["paged_attention_varlen_b200/csrc/prefill_d256.cu", "paged_attention_varlen_b200/csrc/ptx.cuh"]
MLA_KERNEL_SOURCES = ["paged_attention_varlen_b200/csrc/mla.cu", "paged_attention_varlen_b200/csrc/mla_common.cuh",
                      "paged_attention_varlen_b200/csrc/ptx.cuh"]
# the workload each committed ncu summary was captured on: its dram bytes describe that workload's launch only
PROFILED_WORKLOADS = {"varlen_causal_bf16": PROFILE, "varlen_causal_bf16_d256": PROFILE_D256,
                      "long_alibi_sqrt_bf16": os.path.join(ROOT, "profiles", "prefill_long_alibi_sqrt_bf16.md"),
                      "mla_decode_qs1_bf16": MLA_PROFILE, "mla_decode_qs1_int8": MLA_INT8_PROFILE}
DEFAULT_WORKLOAD = "varlen_causal_bf16"
WORKLOADS = {
    "varlen_causal_bf16": lambda: synth.varlen_causal_bf16(),
    "prefix_paged_alibi_fp16": lambda: synth.prefix_paged_alibi_fp16(),
    "long_alibi_sqrt_bf16": lambda: synth.long_alibi_bf16(synth.MASK_ALIBI_SQRT),
    "long_alibi_left_bf16": lambda: synth.long_alibi_bf16(synth.MASK_ALIBI_LEFT),
    "varlen_causal_bf16_d256": lambda: synth.varlen_causal_bf16(heads=16, kv_heads=4, head_size=256),
    "mla_decode_qs1_bf16": lambda: synth.mla_decode_bf16(1),
    "mla_spec_qs4_bf16": lambda: synth.mla_decode_bf16(4),
    "mla_decode_qs1_int8": lambda: synth.mla_decode_int8(),
}
L2_FLUSH_BYTES = 256 << 20


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The largest per-rank value (the slowest rank's step time); identity without a process group."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, work_per_rank: float, ms: float, scale: float) -> float:
    """Whole-job rate: every rank processes the same work (weak scaling) in at most `ms`."""
    return world * work_per_rank / (ms * 1e-3) / scale


def kernel_source_hash(paths=KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def profiled_traffic(workload, src_hash):
    """dram bytes per launch from the committed ncu summary of this workload, if there is one and it was taken
    on the current kernel source (None otherwise)."""
    path = PROFILED_WORKLOADS.get(workload)
    if path is None or not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line and line.strip().startswith(("traffic_bytes_per_launch", "kernel_source_sha256")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256") != src_hash or "traffic_bytes_per_launch" not in vals:
        return None
    return float(vals["traffic_bytes_per_launch"])


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index):
        self.samples, self.reasons, self.ok = [], set(), False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------- workloads

def prefill_flops(case) -> float:
    return 4.0 * case.head_size * case.heads * case.valid_pairs()


def prefill_bytes(case) -> float:
    es = case.q.element_size()
    kv_tokens = int(case.kv_seq_len.sum())
    return es * case.head_size * (2 * case.n_tokens * case.heads + 2 * kv_tokens * case.kv_heads)


def mla_flops(case) -> float:
    return case.heads * (2 * 576 + 2 * 512) * case.valid_pairs()


def mla_bytes(case) -> float:
    """Each cached ctKV + kRope row once, the query, the output and the fp32 lse (per-head descales: 1 KB)."""
    es = case.q_rope.element_size()
    kv = int(case.context_lens.sum()) * (512 * case.ct_kv.element_size() + 64 * es)
    q = case.n_tokens * case.heads * (512 * case.q_nope.element_size() + 64 * es)
    o = case.n_tokens * case.heads * 512 * es + case.n_tokens * case.heads * 4
    return kv + q + o


def device_inputs(case, device):
    """Device copies of a workload's inputs (and fp32 lse / per-head descale buffers for MLA)."""
    if isinstance(case, synth.MlaCase):
        t = {"q_nope": case.q_nope.to(device), "q_rope": case.q_rope.to(device), "ct_kv": case.ct_kv.to(device),
             "k_rope": case.k_rope.to(device), "bt": torch.from_numpy(case.block_tables).to(device)}
        t["lse"] = torch.empty((case.n_tokens, case.heads, 1), dtype=torch.float32, device=device)
        if case.qk_descale is not None:  # int8 latent cache
            t["qk_descale"] = torch.from_numpy(case.qk_descale).to(device)
            t["pv_descale"] = torch.from_numpy(case.pv_descale).to(device)
        return t
    t = {"q": case.q.to(device), "k": case.k.to(device), "v": case.v.to(device)}
    t["slopes"] = None if case.slopes is None else torch.from_numpy(case.slopes).to(device)
    if case.paged:
        t["bt"] = torch.from_numpy(case.block_tables).to(device)
    return t


def plan_on(ala, case, t, out=None):
    """Plan the workload's call on device inputs `t` (the public *_get_workspace_size path); returns (op, out)."""
    if isinstance(case, synth.MlaCase):
        return ala.plan_mla(t["q_nope"], t["q_rope"], t["ct_kv"], t["k_rope"], t["bt"], case.context_lens,
                            case.q_seq_len if case.calc_type == synth.MLA_CALC_SPEC else None, case.heads,
                            case.qk_scale, case.mask_type, case.calc_type, lse=t["lse"], out=out,
                            qk_descale=t.get("qk_descale"), pv_descale=t.get("pv_descale"))
    if case.paged:
        return ala.plan_prefix_encoder(t["q"], t["k"], t["v"], t["bt"], case.seq_len, case.kv_seq_len,
                                       case.mask_type, case.heads, case.kv_heads, case.qk_scale, t["slopes"], out=out)
    return ala.plan_varlen_attention(t["q"], t["k"], t["v"], case.seq_len, case.kv_seq_len, case.mask_type,
                                     case.heads, case.kv_heads, case.qk_scale, t["slopes"], out=out)


def plan_case(ala, case, device):
    """Device copies of the inputs and a planned op; returns (op, tensors dict)."""
    t = device_inputs(case, device)
    op, t["out"] = plan_on(ala, case, t)
    return op, t


def host_costs(ala, case, t, reps=15):
    """Host-side cost of a call, reported apart from the kernel time (the schedule is host work):
    plan = *_get_workspace_size (validation, per-sequence table, work units and their longest-first packing,
    or the MLA lane plan) plus the output / workspace tensors from torch's caching allocator;
    first_run_extra = the extra host time of an op's first execution (tensor-map encoding);
    launch = host time of a later execution (schedule upload and kernel launches enqueued)."""
    plan_ms, first_ms, later_ms = [], [], []
    for _ in range(reps):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        op, _ = plan_on(ala, case, t, out=t["out"])
        t1 = time.perf_counter()
        op()
        t2 = time.perf_counter()
        op()
        t3 = time.perf_counter()
        torch.cuda.synchronize()
        plan_ms.append((t1 - t0) * 1e3)
        first_ms.append((t2 - t1) * 1e3)
        later_ms.append((t3 - t2) * 1e3)
        del op
    med = statistics.median
    return {"plan_ms": med(plan_ms), "first_run_extra_ms": max(0.0, med(first_ms) - med(later_ms)),
            "launch_ms": med(later_ms), "reps": reps}


def time_steps(op, steps, warmup, flush, stream, barrier=lambda: None):
    for _ in range(warmup):
        op(stream)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        op(stream)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    assert op.device_status() == 0, "device status nonzero after the timed steps"
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def e2e_prefill(ala, case, tens, op, steps, stream):
    """Same metric through the public call, inputs from pinned host memory and output back to host."""
    host = {k: case_t.pin_memory() for k, case_t in (("q", case.q), ("k", case.k), ("v", case.v))}
    out_host = torch.empty(tens["out"].shape, dtype=tens["out"].dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in host.values())
    d2h = out_host.numel() * out_host.element_size()
    times = []
    for i in range(steps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        with torch.cuda.stream(stream):
            for k in ("q", "k", "v"):
                tens[k].copy_(host[k], non_blocking=True)
            op(stream)
            out_host.copy_(tens["out"], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1))
    ms = statistics.mean(times)
    # the same, with the call planned inside the timed region every step (a caller whose lengths change
    # every step pays get_workspace_size and the tensor-map encoding each time); wall clock
    wall = []
    for i in range(steps + 2):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            for k in ("q", "k", "v"):
                tens[k].copy_(host[k], non_blocking=True)
            op2, _ = plan_on(ala, case, tens, out=tens["out"])
            op2(stream)
            out_host.copy_(tens["out"], non_blocking=True)
        torch.cuda.synchronize()
        if i >= 2:
            wall.append((time.perf_counter() - t0) * 1e3)
        del op2
    ms_plan = statistics.mean(wall)
    return {"value": prefill_flops(case) / (ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "with_plan": {"value": prefill_flops(case) / (ms_plan * 1e-3) / 1e12, "unit": "TFLOPS",
                          "ms_per_step": ms_plan, "timing": "wall clock, synchronised on both sides"}}


def cpu_baseline(case, sample_s=12.0):
    """The fp64 oracle, as it stands, on a bounded random sample of the workload's rows."""
    import oracle
    cu = np.concatenate([[0], np.cumsum(case.seq_len)])
    tok_seq = np.repeat(np.arange(len(case.seq_len)), case.seq_len)
    rng = np.random.Generator(np.random.PCG64(7))
    n_rows = 256
    total_flops, total_s, rows_done = 0.0, 0.0, 0
    while total_s < sample_s:
        rows = rng.choice(case.n_tokens * case.heads, size=n_rows, replace=False)
        t0 = time.perf_counter()
        oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                         case.kv_heads, case.qk_scale, slopes=case.slopes, block_tables=case.block_tables,
                         block_size=case.block_size, rows=rows)
        total_s += time.perf_counter() - t0
        tok = rows // case.heads
        b = tok_seq[tok]
        i = tok - cu[b]
        allowed = np.minimum(i + (case.kv_seq_len[b] - case.seq_len[b]) + 1, case.kv_seq_len[b])
        total_flops += float((4.0 * case.head_size * allowed).sum())
        rows_done += n_rows
        n_rows = min(n_rows * 2, case.n_tokens * case.heads)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": total_flops / total_s / 1e12, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
            "sample": f"{rows_done} random (token, head) rows of the {case.name} workload, {total_s:.1f} s "
                      f"fp64 on the host (valid FLOPs of the sampled rows / time)"}


def mla_kernel_name(case):
    return "mla_kernel<bf16, int8 cache>" if case.qk_descale is not None else "mla_kernel<bf16>"


def case_dtype(case):
    return case.q_rope.dtype if isinstance(case, synth.MlaCase) else case.dtype


def op_has_combine(op):
    # the MLA workspace holds fp32 partials only when some key range was split (then a combine launch follows)
    return op.workspace_size > 1 << 20


def base_config(case):
    l2 = "flushed before every step (256 MiB write, outside the step events)"
    if isinstance(case, synth.MlaCase):
        return {"workload": case.name, "global_batch": len(case.context_lens), "tokens": case.n_tokens,
                "context_lens": "U[1024,16384] per batch", "heads": case.heads, "kv_lora": 512, "rope": 64,
                "qseqlen": int(case.q_seq_len[0]), "block_size": case.block_size,
                "cache": ("int8 ctKV and qNope codes, per-head qkDescale / pvDescale" if case.qk_descale is not None
                          else str(case.q_rope.dtype).replace("torch.", "")),
                "parallelism": "replicas (independent batches)", "l2": l2}
    mask = {0: "none", 3: "alibi right", 4: "alibi sqrt", 5: "alibi left", 9: "causal"}[case.mask_type]
    return {"workload": case.name, "global_batch": len(case.seq_len), "tokens": case.n_tokens,
            "seq_len": "U[64,2048] per sequence" if case.name.startswith("varlen") else "see workload",
            "heads": case.heads, "kv_heads": case.kv_heads, "head_size": case.head_size, "mask": mask,
            "paged": case.paged, "parallelism": "replicas (independent sequences)", "l2": l2}


def _row_flops(case, rows):
    """Valid FLOPs of the given flattened (token * heads + head) rows."""
    tok = rows // case.heads
    if isinstance(case, synth.MlaCase):
        cu = np.concatenate([[0], np.cumsum(case.q_seq_len)])
        b = np.searchsorted(cu, tok, side="right") - 1
        allowed = case.context_lens[b] - case.q_seq_len[b] + (tok - cu[b]) + 1
        return float((allowed * (2 * 576 + 2 * 512)).sum())
    cu = np.concatenate([[0], np.cumsum(case.seq_len)])
    b = np.searchsorted(cu, tok, side="right") - 1
    i = tok - cu[b]
    if case.mask_type == synth.MASK_NONE:
        allowed = case.kv_seq_len[b]
    else:
        allowed = np.minimum(i + (case.kv_seq_len[b] - case.seq_len[b]) + 1, case.kv_seq_len[b])
    return float((4.0 * case.head_size * allowed).sum())


def _oracle_rows(case, rows):
    import oracle
    if isinstance(case, synth.MlaCase):
        oracle.mla(case.q_nope, case.q_rope, case.ct_kv, case.k_rope, case.block_tables, case.block_size,
                   case.context_lens, case.q_seq_len, case.heads, case.qk_scale, rows=rows)
    else:
        oracle.attention(case.q, case.k, case.v, case.seq_len, case.kv_seq_len, case.mask_type, case.heads,
                         case.kv_heads, case.qk_scale, slopes=case.slopes, block_tables=case.block_tables,
                         block_size=case.block_size, rows=rows)


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores: every step computes the same fixed random sample
    of the workload's (token, head) rows, sized so that warm-up plus timed steps take about a minute."""
    if rank != 0:
        return
    case = WORKLOADS[args.workload]()
    is_mla = isinstance(case, synth.MlaCase)
    n_total = case.n_tokens * case.heads
    perm = np.random.Generator(np.random.PCG64(7)).permutation(n_total).astype(np.int64)
    probe = np.sort(perm[:64])
    t0 = time.perf_counter()
    _oracle_rows(case, probe)
    s_per_flop = (time.perf_counter() - t0) / max(_row_flops(case, probe), 1.0)
    flops_per_row = _row_flops(case, perm[:4096]) / min(4096, n_total)  # the workload's mean row cost
    step_s = min(10.0, max(0.5, 60.0 / (args.steps + args.warmup)))
    n = int(min(n_total, max(64, step_s / (s_per_flop * flops_per_row))))
    rows = np.sort(perm[:n])
    flops = _row_flops(case, rows)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        _oracle_rows(case, rows)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    if is_mla:
        value, unit = mla_bytes(case) * n / n_total / (ms * 1e-3) / 1e9, "GB/s"
        metric = "attention HBM GB/s (MLA decode)"
    else:
        value, unit = flops / (ms * 1e-3) / 1e12, "TFLOPS"
        metric = "attention TFLOPS on valid tokens (prefill)"
    sample = (f"each step: the same {n} random (token, head) rows of the {case.name} workload "
              f"({n / n_total:.2%} of its rows, {flops / 1e9:.2f} valid GFLOP), fp64 oracle on the host")
    config = base_config(case)
    config["reference_sample_rows"] = n
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS),
                    help="workload of the timed steps (the default is the metric's prefill configuration)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import paged_attention_varlen_b200 as ala
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    barrier = (lambda: dist.barrier()) if dist else (lambda: None)

    case = WORKLOADS[args.workload]()
    is_mla = isinstance(case, synth.MlaCase)
    op, tens = plan_case(ala, case, device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    with ClockSampler(local) as clk:
        times = time_steps(op, args.steps, args.warmup, flush, stream, barrier)
    ms = max_over_ranks(statistics.mean(times), dist, device)
    flops = mla_flops(case) if is_mla else prefill_flops(case)
    nbytes = mla_bytes(case) if is_mla else prefill_bytes(case)
    if is_mla:
        value = job_throughput(world, nbytes, ms, 1e9)
        metric, unit = "attention HBM GB/s (MLA decode)", "GB/s"
    else:
        value = job_throughput(world, flops, ms, 1e12)
        metric, unit = "attention TFLOPS on valid tokens (prefill)", "TFLOPS"

    if rank == 0:
        peaks = measured_peaks()
        mean_ms = statistics.mean(times)
        if is_mla:
            src = kernel_source_hash(MLA_KERNEL_SOURCES)
            achieved = nbytes / (mean_ms * 1e-3) / 1e9
            roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": achieved / peaks["hbm_gbs"],
                        "traffic": profiled_traffic(args.workload, src),
                        "algorithmic_bytes": nbytes, "peak_source": peaks["source"] + " (copy bandwidth)",
                        "tflops": flops / (mean_ms * 1e-3) / 1e12,
                        "kernel": mla_kernel_name(case) + " + mla_combine_kernel",
                        "kernel_source_sha256": src}
            launches = args.steps * (2 if op_has_combine(op) else 1)
        else:
            d256 = case.head_size > 128
            src = kernel_source_hash(D256_KERNEL_SOURCES if d256 else KERNEL_SOURCES)
            achieved = flops / (mean_ms * 1e-3) / 1e12
            roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": achieved / peaks["bf16_tflops"],
                        "traffic": profiled_traffic(args.workload, src),
                        "algorithmic_bytes": nbytes, "peak_source": peaks["source"] + " (burst bf16)",
                        "kernel": "prefill_d256_kernel" if d256 else "prefill_kernel", "kernel_source_sha256": src}
            launches = args.steps
        line = {"metric": metric, "value": value, "unit": unit,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "fp16" if case_dtype(case) == torch.float16 else "bf16",
                "data": "synthetic", "config": base_config(case), "roofline": roofline,
                "clocks": clk.summary(), "gpu_launches": launches, "valid_flops_per_step": flops}
        if not is_mla:
            line["padding_positions"] = int(len(case.seq_len) * case.seq_len.max() - case.seq_len.sum())
        args.no_e2e = args.no_e2e or is_mla
        args.no_cpu = args.no_cpu or is_mla
        args.no_extra = args.no_extra or args.workload != DEFAULT_WORKLOAD
        if not args.no_e2e:
            line["e2e"] = e2e_prefill(ala, case, tens, op, min(args.steps, 10), stream)
        line["host"] = host_costs(ala, case, tens)
        if not args.no_extra:
            line["extra"] = extra_workloads(ala, device, flush, stream, peaks, case, args)
        if world == 1 and not args.no_cpu:
            line["cpu_baseline"] = cpu_baseline(case)
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def extra_workloads(ala, device, flush, stream, peaks, main_case, args):
    out = {}
    steps = max(5, min(args.steps, 20))
    # padded layout of the same batch: same kernel, the work a padded batch carries
    pad = synth.padded_from(main_case)
    op, _ = plan_case(ala, pad, device)
    ms = statistics.mean(time_steps(op, steps, 3, flush, stream))
    out["varlen_causal_bf16_padded"] = {
        "ms": ms, "padding_positions": pad.meta["padding_positions"],
        "pairs_ratio_vs_packed": pad.valid_pairs() / main_case.valid_pairs(),
        "valid_tflops": prefill_flops(main_case) / (ms * 1e-3) / 1e12}
    del op
    for case in (synth.prefix_paged_alibi_fp16(), synth.long_alibi_bf16(synth.MASK_ALIBI_SQRT),
                 synth.long_alibi_bf16(synth.MASK_ALIBI_LEFT),
                 synth.varlen_causal_bf16(heads=16, kv_heads=4, head_size=256)):
        op, t = plan_case(ala, case, device)
        ms = statistics.mean(time_steps(op, steps, 3, flush, stream))
        tf = prefill_flops(case) / (ms * 1e-3) / 1e12
        out[case.name] = {"ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
                          "host": host_costs(ala, case, t, reps=5)}
        del op
    for case in (synth.mla_decode_bf16(1), synth.mla_decode_bf16(4), synth.mla_decode_int8()):
        try:
            op, t = plan_case(ala, case, device)
            ms = statistics.mean(time_steps(op, steps, 3, flush, stream))
        except ala.AlaError as e:
            out[case.name] = {"unavailable": str(e)}
            continue
        gbs = mla_bytes(case) / (ms * 1e-3) / 1e9
        tf = mla_flops(case) / (ms * 1e-3) / 1e12
        out[case.name] = {"ms": ms, "hbm_gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"], "tflops": tf,
                          "frac_of_bf16_peak": tf / peaks["bf16_tflops"], "kernel": mla_kernel_name(case),
                          "host": host_costs(ala, case, t, reps=5)}
        del op
    return out


if __name__ == "__main__":
    main()
