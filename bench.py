#!/usr/bin/env python
"""Benchmark: packed LM-head tokens/s with the decode HBM / prefill tensor roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the logit path (prologue, residual contraction with the rank
epilogue) over each token batch of the workload: for the Qwen3-8B-shaped decode head that
is one archead_logits call at each of N = 1, 4, 16, 64 (85 tokens).  Inputs are seeded
synthetic data of the workload's shapes; the head is built by the construction (Algorithm
1) on the GPU before timing.  Under torchrun every rank holds its own replica of the head
and evaluates its own tokens (replicas only, weak scaling, no collective on the data
path); rank 0 prints one JSON line.  The default line also carries a "prefill" block: the
N = 4096 prefill workload on the same head, with its TFLOP/s against the BF16 peaks.

--mode vocab times the vocabulary-parallel NLL instead: the fused-NLL head split by rows
over the ranks, the same tokens on every rank, one NCCL all-gather of the per-token
partials per step (strong scaling).

--impl reference times the CPU oracle (fp64, host cores) on a bounded vocabulary sample of
the same workload, scaled to the full vocabulary.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import (WORKLOADS, bf16_bits, make_channel_scales, make_hidden,  # noqa: E402
                       make_targets, make_weight)

L2_BYTES = 126 * 2 ** 20
METRIC = "packed LM-head tokens/s; decode HBM GB/s and prefill TFLOP/s vs B200 roofline"
MAIN_KERNEL_SRC = ["packed_int4_lm_b200/csrc/residual_dec.cu",
                   "packed_int4_lm_b200/csrc/residual_mma.cu",
                   "packed_int4_lm_b200/csrc/residual_tc.cu",
                   "packed_int4_lm_b200/csrc/tc_common.cuh",
                   "packed_int4_lm_b200/csrc/archead_internal.cuh"]
# token counts up to this go to the persistent decode kernel, larger ones to the tcgen05
# kernel (for the workloads here; shapes whose shared-memory plan fails use the token-block
# warp-MMA kernel)
DEC_MAX_N = 16


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--mode", choices=["logits", "vocab"], default="logits",
                    help="vocab: the vocabulary-parallel NLL (rows split over the GPUs, one "
                         "all-gather per step) on the fused-NLL workload")
    ap.add_argument("--workload", default="qwen_decode", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--ns", default=None,
                    help="comma-separated token counts replacing the workload's (profiling "
                         "a smaller case of the same head)")
    return ap.parse_args()


DEFAULT_STEPS = {"tiny": (500, 20), "qwen_decode": (600, 20), "qwen_prefill": (20, 3),
                 "llama_batched": (100, 5), "wide_nll": (10, 3)}


# ----------------------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def kernel_source_sha():
    h = hashlib.sha256()
    for f in MAIN_KERNEL_SRC:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, Ns):
    """Mean DRAM bytes per launch of the main kernel over the step's batches, from the
    committed ncu summary; None when the kernel source changed since those counters were
    taken or a batch size was not captured."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(workload)
    if not d or d.get("source_sha") != kernel_source_sha():
        return None
    by_n = d.get("bytes_per_launch_by_N", {})
    if not all(str(N) in by_n for N in Ns):
        return None
    return sum(by_n[str(N)] for N in Ns) / len(Ns)


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(self.NAMES, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------------------
def build_head(w, device, keep_dense=False):
    """The packed head of workload w, the channel scales of its activations, and the
    construction's wall seconds (Algorithm 1 on `device`, synchronised); with keep_dense
    also the dense head W (FP32, on `device`) for the quality comparisons."""
    from packed_int4_lm_b200 import pack
    W = make_weight(w.V, w.D, w.rank, w.sigma0, w.noise, w.seed_w, device=device)
    s = make_channel_scales(w.D, w.sigma_s, w.n_outliers, w.outlier_mult, w.seed_scales)
    Hc = make_hidden(w.n_cal, s, w.seed_hcal).to(device)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    head = pack.build_head(W, Hc, w.r_c, w.r_r, w.g, w.p, w.lam, seed=w.seed_rsvd)
    torch.cuda.synchronize()
    cons_s = time.perf_counter() - t0
    if keep_dense:
        return head, s, cons_s, W, Hc
    del W, Hc
    torch.cuda.empty_cache()
    return head, s, cons_s


def agreement_quality(ah, w, head, W, Hcal, Hq, dev):
    """Quality context on the decode head, through the library's GPU path only: the packed
    head and its storage-matched baselines (Sec. 5, Tables 3 and 8: plain group INT4 at a
    matching storage, the quantized core without the correction, Row INT8 at about twice
    the storage) against the dense head in BF16 on the same tokens.  Per head: storage over
    BF16, relative logit error ||Y - Y_dense||_F / ||Y_dense||_F, mean KL(dense || head),
    and the fraction of tokens whose dense top-1 id is among the head's top 1 / 5 / 10."""
    from packed_int4_lm_b200 import pack
    H = Hq.to(dev)
    Yd = torch.matmul(H, W.to(torch.bfloat16).t()).float()  # the dense comparator (cuBLAS)
    heads = {"archead": head}
    heads["group_int4_g32"] = pack.build_head(W, Hcal, 0, 0, 32, w.p, w.lam, seed=w.seed_rsvd)
    heads["core_only"] = pack.build_head(W, Hcal, w.r_c, 0, w.g, w.p, w.lam, seed=w.seed_rsvd)
    heads["row_int8"] = pack.build_row8_head(W, g=w.g)
    out = {"tokens": int(H.shape[0]), "dense": "H W^T with W in BF16 (torch.matmul, comparator)",
           "synthetic_W": "rank-64 decaying spectrum plus N(0, 0.02^2) noise: the noise "
                          "dominates, so these figures are not the paper's real-head ones"}
    for name, hd in heads.items():
        dh = ah.DeviceHead.from_canonical(hd, dev)
        Y = ah.logits(H, dh)
        a = ah.agreement(H, dh, Yd, 10)
        ah.check()
        top = a["topk"].long()
        t1 = a["top1_dense"].long()[:, None]
        out[name] = {"storage_vs_bf16": pack.storage_ratio(hd),
                     "rel_logit_err": float((Y - Yd).norm() / Yd.norm()),
                     "mean_kl": float(a["kl"].double().mean()),
                     "top1_agree": float((top[:, :1] == t1).any(1).float().mean()),
                     "top5_agree": float((top[:, :5] == t1).any(1).float().mean()),
                     "top10_agree": float((top[:, :10] == t1).any(1).float().mean())}
        del dh
    torch.cuda.empty_cache()
    return out


def nll_quality(head, Wb, Hcpu, tg, ours, sample=16):
    """Quality context for the fused-NLL workload: mean NLL of the packed head (the timed
    path's output), of the dense head in BF16 on the same tokens (torch.matmul +
    cross_entropy, a comparator only), and of the fp64 oracle on the first `sample` tokens
    next to the packed head's values for them."""
    import oracle
    dev = Wb.device
    H = Hcpu.to(dev)
    tgt = tg.to(dev).long()
    dense = []
    for i in range(0, H.shape[0], 512):
        logits = torch.matmul(H[i:i + 512], Wb.t()).float()
        dense.append(torch.nn.functional.cross_entropy(logits, tgt[i:i + 512], reduction="none"))
    dense = torch.cat(dense)
    ref = oracle.nll(head, bf16_bits(Hcpu[:sample]), tg[:sample].numpy())
    mine = ours[:sample].double().cpu().numpy()
    return {"mean_nll_packed": float(ours.double().mean()),
            "mean_nll_dense_bf16": float(dense.double().mean()),
            "oracle_sample_tokens": sample,
            "mean_nll_oracle_sample": float(np.mean(ref)),
            "mean_nll_packed_sample": float(np.mean(mine)),
            "max_abs_nll_diff_vs_oracle": float(np.max(np.abs(mine - ref)))}


def l2_note(head):
    mb = sum(head[k].nbytes for k in head if isinstance(head[k], np.ndarray)) / 1e6
    if mb * 1e6 > L2_BYTES:
        return "inputs larger than L2: packed head %.1f MB > 126 MB L2, no flush" % mb
    return "packed head %.1f MB is L2-resident (a parity workload, no roofline claim)" % mb


def job_throughput(local_ms, tokens_per_rank, world, device):
    """Whole-job tokens/s of `world` ranks that each ran the same steps: the job takes as long
    as its slowest rank, so the local device times are reduced with MAX.  Returns
    (tokens/s, job ms)."""
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms = float(t.item())
    return tokens_per_rank * world / (ms / 1e3), ms


def main_kernel_bytes(head, N):
    """Algorithmic bytes one launch of the residual kernel must move: the packed rows it
    reads (nibbles, codes, super-scales, A_c / A_w and their scales), the FP16 hidden
    states and t, and the FP32 logits it writes (none in NLL mode)."""
    per_head = sum(head[k].nbytes for k in ("r_nib", "r_code", "r_super", "Ac", "sAc", "Aw", "sAw"))
    RR = head["r_c"] + head["r_r"]
    return per_head + 2 * N * head["D"] + 4 * N * RR


def flops(head, N):
    V, D, RR = head["V"], head["D"], head["r_c"] + head["r_r"]
    return 2.0 * N * V * D + 2.0 * N * RR * (V + D)


def oracle_step(head, Hs, targets, Ns, nll_mode, rows):
    """One step of the CPU oracle on the first `rows` vocabulary rows; returns seconds."""
    import oracle
    t0 = time.perf_counter()
    for N in Ns:
        Y = oracle.logits(head, Hs[N], rows=slice(0, rows))
        if nll_mode:
            oracle.nll_from_logits(Y, np.minimum(targets[N], rows - 1))
    return time.perf_counter() - t0


def oracle_rows_for(head, Hs, targets, Ns, nll_mode, budget_s):
    """Vocabulary rows whose oracle step takes about budget_s (from a small probe)."""
    V = head["V"]
    probe_rows = min(V, 1024)
    tp = oracle_step(head, Hs, targets, Ns, nll_mode, probe_rows)
    return int(min(V, max(128, probe_rows * budget_s / max(tp, 1e-4))))


def cpu_oracle_rate(head, Hs, targets, Ns, nll_mode, budget_s):
    """Oracle tokens/s on a vocabulary sample, time scaled to the full vocabulary."""
    rows = oracle_rows_for(head, Hs, targets, Ns, nll_mode, budget_s)
    t = oracle_step(head, Hs, targets, Ns, nll_mode, rows)
    return sum(Ns) / (t * head["V"] / rows), rows, t


def reference_arm(a, w, K, Wm, Ns, nll_mode, cfg):
    """--impl reference: the CPU oracle as it stands, on a bounded vocabulary sample of the
    same workload (rank 0 only; the other ranks exit without work)."""
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if rank != 0:
        return
    torch.cuda.set_device(local)
    head, s, _ = build_head(w, torch.device("cuda", local))
    Hs = {N: bf16_bits(make_hidden(N, s, w.seed_heval)) for N in Ns}
    tg = {N: make_targets(N, w.V, w.seed_targets).numpy() for N in Ns}
    import oracle  # noqa: F401
    budget = max(0.02, 150.0 / (K + Wm))  # whole run within a few minutes
    rows_used = oracle_rows_for(head, Hs, tg, Ns, nll_mode, budget)
    vals = []
    for i in range(Wm + K):
        t = oracle_step(head, Hs, tg, Ns, nll_mode, rows_used)
        if i >= Wm:
            vals.append(t * w.V / rows_used)  # scaled to the full vocabulary
    ms_full = 1e3 * statistics.mean(vals)          # scaled to the full vocabulary
    ms_sample = ms_full * rows_used / w.V            # the measured step: the sample
    value = sum(Ns) / (ms_full / 1e3)
    cores = len(os.sched_getaffinity(0))
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": a.gpus,
            "steps": K, "warmup": Wm, "ms_per_step": ms_sample,
            "ms_per_step_full_vocab": ms_full, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(cfg, l2=l2_note(head)), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{sum(Ns)} tokens x {rows_used} of {w.V} vocab rows "
                                       "per step (ms_per_step is that measured sample; "
                                       "value scales its time by V/rows)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure_calls(call, reps, stream):
    """Mean milliseconds of one call (CUDA events around `reps` back-to-back calls on the
    launching stream), then the mean main-kernel milliseconds from the library's events
    around that kernel in a second pass of the same calls (events between the prologue
    and the main kernel stop their overlap, so they stay out of the first pass)."""
    import packed_int4_lm_b200 as ah
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(reps):
        call()
    f1.record(stream)
    torch.cuda.synchronize()
    call_ms = f0.elapsed_time(f1) / reps
    ah.profile(True)
    for _ in range(reps):
        call()
    torch.cuda.synchronize()
    ah.profile(False)
    ah.check()
    kms, kn = ah.profile_read()
    return call_ms, kms / max(kn, 1)


def prefill_block(ah, head, dh, s, dev, stream, peaks, steps):
    """The prefill workload on the decode head: one archead_logits call of N = 4096 tokens
    per step, with its own TFLOP/s against the sustained and burst BF16 peaks."""
    w = WORKLOADS["qwen_prefill"]
    N = w.Ns[0]
    H = make_hidden(N, s, w.seed_heval).to(dev)
    Y = torch.empty(N, w.V, device=dev)

    def call():
        ah.logits(H, dh, out=Y)

    for _ in range(3):
        call()
    ah.check()
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    call_ms, kern_ms = measure_calls(call, max(5, steps), stream)
    ck = clocks.stop()
    fl = flops(head, N)
    tf = fl / (kern_ms / 1e3) / 1e12
    out = {"N": N, "calls": max(5, steps), "call_us": 1e3 * call_ms,
           "main_kernel_us": 1e3 * kern_ms, "tokens_per_s": N / (call_ms / 1e3),
           "kernel": "residual_tc_kernel", "flops_per_call": fl, "TFLOPs": tf,
           "frac_of_sustained": tf / peaks["bf16_sustained"], "frac_of_burst": tf / peaks["bf16"],
           "peak_sustained": peaks["bf16_sustained"], "peak_burst": peaks["bf16"],
           "peak_source": peaks["source"],
           "traffic": profiled_traffic("qwen_prefill", [N]), "clocks": ck}
    del H, Y
    torch.cuda.empty_cache()
    return out


def vocab_main(a, world, rank, local):
    """--mode vocab: one head split by vocabulary rows over the ranks; every step evaluates
    the per-token NLL of the same N tokens on all ranks: shard partials, one NCCL all-gather
    of N x 3 floats per rank, merge (strong scaling: the head is divided, the tokens are
    not)."""
    import packed_int4_lm_b200 as ah
    from packed_int4_lm_b200 import pack
    w = WORKLOADS[a.workload if WORKLOADS[a.workload].nll else "wide_nll"]
    K, Wm = DEFAULT_STEPS[w.name]
    K = a.steps if a.steps is not None else K
    Wm = a.warmup if a.warmup is not None else Wm
    N = int(a.ns.split(",")[0]) if a.ns else w.Ns[0]
    if world > 1:
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=180),
            device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    head, s, cons_s = build_head(w, dev)
    v0, v1 = w.V * rank // world, w.V * (rank + 1) // world
    dh = ah.DeviceHead.from_canonical(pack.shard_rows(head, v0, v1), dev)
    Hc = make_hidden(N, s, w.seed_heval)
    H = Hc.to(dev)
    tg = make_targets(N, w.V, w.seed_targets)
    tgd = tg.to(dev)
    stream = torch.cuda.current_stream()

    def step():
        return ah.vocab_parallel_nll(H, dh, tgd, v0, w.V)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(Wm):
        step()
    ah.check()
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ah.nll_partials(H, dh, tgd, v0, w.V)
    per_step = ah.last_launches() + 1  # the partials call's kernels, then the merge
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(K):
        out = step()
    e1.record(stream)
    launches = per_step * K
    torch.cuda.synchronize()
    barrier()
    ck = clocks.stop()
    ah.check()
    local_ms = e0.elapsed_time(e1)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    job_ms = float(t.item())
    value = N * K / (job_ms / 1e3)  # the job evaluates N tokens per step
    # partials kernel of this rank's shard (same launch as in the timed steps)
    peaks = load_peaks()
    _, kern_ms = measure_calls(lambda: ah.nll_partials(H, dh, tgd, v0, w.V), max(3, K), stream)
    shard = pack.shard_rows(head, v0, v1)
    tf = flops(shard, N) / (kern_ms / 1e3) / 1e12
    # end to end: host H and targets in, host NLL out, every step
    Hpin, tgpin = Hc.pin_memory(), tg.pin_memory()
    outh = torch.empty(N, pin_memory=True)

    def step_host():
        Hd = Hpin.to(dev, non_blocking=True)
        td = tgpin.to(dev, non_blocking=True)
        outh.copy_(ah.vocab_parallel_nll(Hd, dh, td, v0, w.V), non_blocking=True)

    KE = max(1, min(a.e2e_steps, K))
    for _ in range(2):
        step_host()
    barrier()
    torch.cuda.synchronize()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(KE):
        step_host()
    g1.record(stream)
    torch.cuda.synchronize()
    barrier()
    te = torch.tensor([float(g0.elapsed_time(g1))], dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(te, op=torch.distributed.ReduceOp.MAX)
    e2e_value = N * KE / (float(te.item()) / 1e3)
    nll_mean = float(out.double().mean())
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": Wm, "ms_per_step": job_ms / K, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": f"{w.name} vocabulary-parallel NLL: V={w.V} D={w.D} N={N} "
                                   f"r_c={w.r_c} r_r={w.r_r} g={w.g}, rows split over {world} GPUs",
                       "V": w.V, "D": w.D, "tokens_per_step": N,
                       "parallelism": f"vocab{world}", "l2": l2_note(head),
                       "construction_s": cons_s},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_sustained"],
                         "unit": "TFLOP/s", "frac": tf / peaks["bf16_sustained"],
                         "peak_source": peaks["source"], "kernel": "residual_tc_kernel (shard)",
                         "traffic": None},
            "cpu_baseline": None,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": N * w.D * 2 + 4 * N,
                    "d2h_bytes_per_step": 4 * N, "steps": KE},
            "gpu_launches": launches, "clocks": ck, "mean_nll": nll_mean}
    print(json.dumps(line), flush=True)


def main():
    a = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if a.mode == "vocab" and a.impl == "ours":
        return vocab_main(a, world, rank, local)
    w = WORKLOADS[a.workload]
    K, Wm = DEFAULT_STEPS[a.workload]
    K = a.steps if a.steps is not None else K
    Wm = a.warmup if a.warmup is not None else Wm
    Ns = [int(x) for x in a.ns.split(",")] if a.ns else list(w.Ns)
    nll_mode = w.nll
    cfg = {"workload": f"{w.name}: V={w.V} D={w.D} N={','.join(map(str, Ns))} "
                       f"r_c={w.r_c} r_r={w.r_r} g={w.g} p={w.p} lam={w.lam}"
                       + (" fused NLL" if nll_mode else ""),
           "V": w.V, "D": w.D, "tokens_per_step_per_gpu": sum(Ns), "parallelism": f"replicas{world}"}

    if a.impl == "reference":
        return reference_arm(a, w, K, Wm, Ns, nll_mode, cfg)

    import packed_int4_lm_b200 as ah
    from packed_int4_lm_b200 import pack

    if world > 1:
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=180),
            device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    Wb = Wf = Hcal = None
    if rank == 0 and (nll_mode or w.name == "qwen_decode") and not a.ns:
        head, s, cons_s, Wf, Hcal = build_head(w, dev, keep_dense=True)
        if nll_mode:
            Wb = Wf.to(torch.bfloat16)
            del Wf, Hcal
            Wf = Hcal = None
            torch.cuda.empty_cache()
    else:
        head, s, cons_s = build_head(w, dev)
    dh = ah.DeviceHead.from_canonical(head, dev)
    # each rank evaluates its own tokens
    Hcpu = {N: make_hidden(N, s, w.seed_heval + 7919 * rank) for N in Ns}
    H = {N: Hcpu[N].to(dev) for N in Ns}
    tg = {N: make_targets(N, w.V, w.seed_targets + 7919 * rank) for N in Ns}
    tgd = {N: tg[N].to(dev) for N in Ns}
    Y = {N: torch.empty(N, w.V, device=dev) for N in Ns} if not nll_mode else None
    out = {N: torch.empty(N, device=dev) for N in Ns} if nll_mode else None
    stream = torch.cuda.current_stream()

    def call(N):
        if nll_mode:
            ah.nll(H[N], dh, tgd[N], out=out[N])
        else:
            ah.logits(H[N], dh, out=Y[N])

    def step():
        launches = 0
        for N in Ns:
            call(N)
            launches += ah.last_launches()
        return launches

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(Wm):
        step()
    ah.check()
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    launches = 0
    for _ in range(K):
        launches += step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ck = clocks.stop()
    ah.check()
    elapsed_ms = e0.elapsed_time(e1)
    value, elapsed_ms = job_throughput(elapsed_ms, sum(Ns) * K, world, dev)
    peaks = load_peaks()

    # Per batch size: call time, and the main kernel's own time from the library's events
    # around it (a second pass of the same calls; see measure_calls).  The same numbers give
    # per_n and the roofline of the main kernel over the step.
    per_n = {}
    kern_s_total = 0.0
    for N in Ns:
        call_ms, kern_ms = measure_calls(lambda: call(N), max(5, min(200, K)), stream)
        kern_s_total += kern_ms / 1e3
        b = main_kernel_bytes(head, N) + (0 if nll_mode else 4 * N * w.V)
        per_n[str(N)] = {"call_us": 1e3 * call_ms, "main_kernel_us": 1e3 * kern_ms,
                         "tokens_per_s": N / (call_ms / 1e3),
                         "main_GBps": b / (kern_ms / 1e3) / 1e9,
                         "hbm_frac": b / (kern_ms / 1e3) / 1e9 / peaks["hbm"],
                         "main_TFLOPs": flops(head, N) / (kern_ms / 1e3) / 1e12}

    # roofline of the residual kernel over the step's launches (one per batch size)
    bytes_step = sum(main_kernel_bytes(head, N) + (0 if nll_mode else 4 * N * w.V) for N in Ns)
    flops_step = sum(flops(head, N) for N in Ns)
    if w.name in ("qwen_decode", "tiny") or max(Ns) <= 64:
        achieved = bytes_step / kern_s_total / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": achieved / peaks["hbm"]}
    else:
        achieved = flops_step / kern_s_total / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_sustained"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_sustained"],
                "frac_of_burst": achieved / peaks["bf16"]}
    roof["peak_source"] = peaks["source"]
    roof["kernel"] = ", ".join(
        (["residual_dec_kernel (N<=%d)" % DEC_MAX_N] if min(Ns) <= DEC_MAX_N else [])
        + (["residual_tc_kernel (N>%d)" % DEC_MAX_N] if max(Ns) > DEC_MAX_N else []))
    roof["traffic"] = profiled_traffic(w.name, Ns)
    roof["main_kernel_share"] = sum(v["main_kernel_us"] for v in per_n.values()) / 1e3 * K / max(elapsed_ms, 1e-9)

    # the prefill workload shares the decode head: its block rides on the default line
    prefill = None
    if w.name == "qwen_decode" and not a.ns:
        prefill = prefill_block(ah, head, dh, s, dev, stream, peaks, max(5, min(20, K)))

    # end to end through the host-buffer entry points
    Hpin = {N: Hcpu[N].pin_memory() for N in Ns}
    tgpin = {N: tg[N].pin_memory() for N in Ns}
    Yh = {N: torch.empty(N, w.V, pin_memory=True) for N in Ns} if not nll_mode else None
    oh = {N: torch.empty(N, pin_memory=True) for N in Ns} if nll_mode else None

    def step_host():
        for N in Ns:
            if nll_mode:
                ah.nll_host(Hpin[N], dh, tgpin[N], out=oh[N])
            else:
                ah.logits_host(Hpin[N], dh, out=Yh[N])

    KE = max(1, min(a.e2e_steps, K))
    for _ in range(3):
        step_host()
    barrier()
    torch.cuda.synchronize()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(KE):
        step_host()
    g1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_value, _ = job_throughput(g0.elapsed_time(g1), sum(Ns) * KE, world, dev)
    h2d = sum(N * w.D * 2 + (4 * N if nll_mode else 0) for N in Ns)
    d2h = sum(4 * N if nll_mode else 4 * N * w.V for N in Ns)

    quality = None
    if Wf is not None:  # the decode head: agreement with the dense head, GPU path
        quality = agreement_quality(ah, w, head, Wf, Hcal, Hcpu[max(Ns)], dev)
        del Wf, Hcal
        torch.cuda.empty_cache()
    if nll_mode and rank == 0 and Wb is not None:
        Nq = Ns[0]
        ah.nll(H[Nq], dh, tgd[Nq], out=out[Nq])
        torch.cuda.synchronize()
        quality = nll_quality(head, Wb, Hcpu[Nq], tg[Nq], out[Nq].clone())
        del Wb
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        Hs = {N: bf16_bits(Hcpu[N]) for N in Ns}
        tgs = {N: tg[N].numpy() for N in Ns}
        rate, rows, tcpu = cpu_oracle_rate(head, Hs, tgs, Ns, nll_mode, 15.0)
        cpu = {"value": rate, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)),
               "kind": "oracle",
               "sample": f"{sum(Ns)} tokens x {rows} of {w.V} vocab rows ({tcpu:.1f} s), "
                         "time scaled by V/rows"}

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": Wm, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": dict(cfg, l2=l2_note(head), construction_s=cons_s,
                           storage_ratio_vs_bf16=pack.storage_ratio(head),
                           serialized_bytes=pack.serialized_nbytes(head)),
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": KE},
            "gpu_launches": launches, "clocks": ck, "per_n": per_n}
    if prefill is not None:
        line["prefill"] = prefill
    if quality is not None:
        line["quality"] = quality
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
