#!/usr/bin/env python
"""Benchmark of one SpecOPD target-scoring step on B200.

A step is one pass of the whole hot path over one batch of synthetic trees:
mask build -> RoPE + tree-masked GQA attention -> fused overlap / E2E-TV loss /
gradient.  The metric is supervised tokens (predictions contributing to the
loss, sum_b W) scored per second.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 5] [--impl reference]

The default workload is the largest single-GPU one ("scale27b": trunk 32,768,
512 branches x 16 samples, 40/8 heads of 128, vocabulary 248,320).

N > 1 runs under torchrun and splits one logical batch over the ranks (strong
scaling): each rank scores a contiguous run of the packed query tiles,
balanced by visible (row, column) pairs, and a contiguous share of whole
branches for the overlap / loss / gradient, normalised by the whole batch's
prediction count; one NCCL all-reduce per step sums the ranks' loss shares.
The timed region is bracketed by barriers and the slowest rank's time is used.
`--impl reference` times the fp64 CPU oracle on the host cores instead (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "supervised tokens/s scored (tree attn + E2E-TV) on 1 B200; % of roofline"
WORKLOAD_DEFAULT = 5

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a
# step's kernels, each from one ncu capture (the profiles/ summary named in
# "profile" gives the command).  Each entry records a digest of the kernel's
# source files at capture time; when the sources differ from it the bench
# reports null, so a figure never outlives the kernel it was taken on.
KERNEL_SOURCES = {
    "tree_attention": ["tree_attention_masked_b200/csrc/tree_attn_sm100.cu", "tree_attention_masked_b200/csrc/ptx.cuh"],
    "tv_overlap_e2e": ["tree_attention_masked_b200/csrc/tv_bf16.cu", "tree_attention_masked_b200/csrc/overlap_common.cuh",
                       "tree_attention_masked_b200/csrc/ptx.cuh"],
}
MEASURED_TRAFFIC = {  # {(workload, kernel): {"bytes": B, "sha": digest, "profile": file}}
    (5, "tree_attention"): {"bytes": 3460822272.0 + 454361856.0, "sha": "4bdfe3fbb81768aa",
                            "profile": "profiles/dram_traffic_scale27b.md"},
    (5, "tv_overlap_e2e"): {"bytes": 17651496192.0 + 8334336512.0, "sha": "2b82289312ce03e1",
                            "profile": "profiles/dram_traffic_scale27b.md"},
}


def source_digest(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: int, kernel: str):
    e = MEASURED_TRAFFIC.get((workload, kernel))
    if e is None or e["sha"] != source_digest(kernel):
        return None
    return e["bytes"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d.get("bf16_tflops_sustained"),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ----------------------------------------------------------------- workload figures
def visible_pairs(case) -> int:
    """sum over packed rows of |vis(r)|: trunk row j sees j+1 columns, sample
    y_{b,i} sees a_b+1 trunk columns plus i samples."""
    total = 0
    a_off = 0
    for T, B in zip(case.trunk_len, case.num_branches):
        total += T * (T + 1) // 2
        anc = case.anchors[a_off:a_off + B].astype(np.int64)
        rpb = case.rows_per_branch
        total += int(rpb * (anc + 1).sum()) + B * rpb * (rpb + 1) // 2
        a_off += B
    return total


def attention_executed_flops(meta: np.ndarray, Hkv: int, G: int, d: int) -> float:
    """FLOPs the tensor-core tree attention issues for one run of query-tile
    records (the kernel's own metadata, in launch order): per (query head, tile
    slot) and visited 128-column key block, Q K^T and P V of 128 x 128 x d each.
    Work items follow the kernel: per pair of tiles (2k, 2k+1), two heads of one
    tile per item, and for odd G the last head of each KV group on both tiles of
    a pair over the union of their column spans (one tile at a time when the
    pair straddles two trees).  Columns come in whole blocks: the trunk span
    [tree_base, max trunk_hi) and the branch span [min br_lo, max br_hi)."""
    def nblk(ms):
        base = int(ms[0][2])
        n = -(-(max(int(m[3]) for m in ms) - base) // 128)
        br = [(int(m[5]), int(m[6])) for m in ms if m[6] > m[5]]
        if br:
            n += -(-(max(h for _, h in br) - min(lo for lo, _ in br)) // 128)
        return n
    nt = len(meta)
    slots = 0
    for k in range((nt + 1) // 2):
        tiles = [t for t in (2 * k, 2 * k + 1) if t < nt]
        for t in tiles:
            slots += 2 * (G // 2) * Hkv * nblk([meta[t]])
        if G % 2:
            if len(tiles) == 2 and meta[tiles[0]][2] == meta[tiles[1]][2]:
                slots += 2 * Hkv * nblk([meta[t] for t in tiles])
            else:
                slots += sum(Hkv * nblk([meta[t]]) for t in tiles)
    return 4.0 * d * 128 * 128 * slots


def case_figures(case):
    pairs = visible_pairs(case)
    flops = 4.0 * case.d * case.Hq * pairs
    es = 2 if case.dtype == "bf16" else 4
    R = case.num_predictions
    ov_bytes = float(R) * case.vocab * (2 * es + 4)
    return dict(pairs=pairs, flops=flops, ov_bytes=ov_bytes, R=R)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------- CPU oracle timing
# One sample of the oracle per call: the same plan for the native arm's
# cpu_baseline (three samples) and for each step of the reference arm, so the
# two estimate the same quantity.
ORACLE_PLAN = dict(attn_rows=8, branches=2, mask_rows=256)


def oracle_sample(case, rng, attn_rows: int, branches: int, mask_rows: int, f64=None):
    """Time the oracle on a bounded sample of one step; returns the estimated
    seconds of a whole step and a description of the sample.

    Per-unit work (a packed row's mask fields, a packed row's attention over
    all heads, a branch's overlap + loss + gradient) is scaled by the number of
    units in the step; work done once per step whatever the sample (tree
    structure, RoPE of every key row) is counted once."""
    from oracle import attention as OA
    from oracle import overlap as OO
    from oracle import tree as OT
    from synthetic import to_f64

    t0 = time.perf_counter()
    pt = OT.pack(case.trunk_len, case.prompt_len, case.num_branches, case.anchors, case.W, case.pack_terminal)
    pos = OT.positions(pt)
    OT.prediction_rows(pt)
    t_struct = time.perf_counter() - t0
    N = pt.num_rows
    rows = rng.choice(N, size=min(mask_rows, N), replace=False)
    t0 = time.perf_counter()
    OT.compact_fields(pt, rows)
    t_mask = (time.perf_counter() - t0) / len(rows) * N
    q, k, v = f64 if f64 is not None else (to_f64(x, case.dtype) for x in (case.q, case.k, case.v))
    t0 = time.perf_counter()
    OA.rope(k, pos, case.theta)  # the once-per-step part of tree_attention below
    t_rope_k = time.perf_counter() - t0
    rows = rng.choice(N, size=min(attn_rows, N), replace=False)
    t0 = time.perf_counter()
    OA.tree_attention(pt, q, k, v, theta=case.theta, rows=rows)
    t_rows = max(time.perf_counter() - t0 - t_rope_k, 0.0)
    t_attn = t_rope_k + t_rows / len(rows) * N
    nb = int(sum(case.num_branches))
    bs = rng.choice(nb, size=min(branches, nb), replace=False)
    t0 = time.perf_counter()
    for b in bs:
        r = np.arange(b * case.W, (b + 1) * case.W)
        z = to_f64(case.draft[r], case.dtype)
        t = to_f64(case.teacher[r], case.dtype)
        a = OO.overlap(z, t)
        OO.e2e_tv_loss(a, case.W, count=nb * case.W)
        OO.e2e_tv_grad_draft(z, t, case.W, count=nb * case.W)
    t_ov = (time.perf_counter() - t0) / len(bs) * nb
    total = t_struct + t_mask + t_attn + t_ov
    desc = (f"oracle on {len(rows)} of {N} packed rows (attention, all {case.Hq} heads; RoPE of all key rows "
            f"counted once), {len(bs)} of {nb} branches (overlap + loss + gradient over all {case.W} rows), "
            f"mask fields of {mask_rows} rows; per-row and per-branch times scaled to the full step")
    return total, desc


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [x.get("num_threads", 1) for x in threadpool_info() if x.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_inputs(case):
    from synthetic import to_f64
    return tuple(to_f64(x, case.dtype) for x in (case.q, case.k, case.v))


def cpu_baseline(case, samples: int = 3):
    rng = np.random.default_rng(123)
    f64 = oracle_inputs(case)
    ests = []
    t0 = time.perf_counter()
    for _ in range(samples):
        est, desc = oracle_sample(case, rng, f64=f64, **ORACLE_PLAN)
        ests.append(est)
    wall = time.perf_counter() - t0
    est = statistics.mean(ests)
    return {"value": case.num_predictions / est, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": desc + f"; mean of {samples} samples, {wall:.1f} s wall", "est_step_s": est}


def config_dict(case, figs, workload: int, seed: int, world: int) -> dict:
    """The workload description printed by both arms."""
    import synthetic as SY
    in_bytes = case.q.nbytes + case.k.nbytes + case.v.nbytes
    if case.draft is not None:
        in_bytes += case.draft.nbytes + case.teacher.nbytes
    return {"workload": SY.WORKLOADS[workload], "supervised_tokens_per_step": figs["R"],
            "packed_rows": case.num_rows, "visible_pairs": figs["pairs"], "seed": seed,
            "l2": "inputs larger than L2 (%.2f GB per step > 126 MB); each step streams them from HBM" % (in_bytes / 1e9),
            "parallelism": ("1 GPU" if world == 1 else
                            f"{world} GPUs, one batch: query tiles split by visible pairs, whole branches split, "
                            "loss shares summed by one NCCL all-reduce per step")}


# ----------------------------------------------------------------- GPU run
def run_gpu(args):
    import torch
    import torch.distributed as dist
    import synthetic as SY
    from tree_attention_masked_b200.build import build
    build()
    from tree_attention_masked_b200 import specopd as S
    from tree_attention_masked_b200.scoring import ScoringStep
    from tree_attention_masked_b200 import parallel as PAR

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    # the same logical batch on every rank; each scores its share of it
    case = SY.make_workload(args.workload, seed=args.seed, workers=min(8, os.cpu_count() or 1))
    figs = case_figures(case)
    nb = int(sum(case.num_branches))
    count = float(nb * case.W)  # the whole batch's predictions, known on the host
    costs = PAR.tile_costs(case.trunk_len, case.num_branches, case.anchors, case.W, case.pack_terminal)
    t0, t1 = PAR.split_tiles(costs, world, rank)
    trows = PAR.tile_rows(case.trunk_len, case.num_branches, case.W, case.pack_terminal)
    r0, r1 = (int(trows[t0, 0]), int(trows[t1 - 1, 1])) if t1 > t0 else (0, 0)
    b0, b1 = PAR.shard_range(nb, world, rank)
    split = world > 1
    st = ScoringStep(case.trunk_len, case.prompt_len, case.num_branches, case.W, case.Hq, case.Hkv, case.d,
                     torch.bfloat16 if case.dtype == "bf16" else torch.float32, case.vocab, device=dev,
                     pack_terminal=case.pack_terminal, theta=case.theta)
    st.load(case)
    stream = torch.cuda.current_stream(dev)

    ev = lambda: torch.cuda.Event(enable_timing=True)
    K, Wm = args.steps, args.warmup
    marks = [[ev() for _ in range(4)] for _ in range(K)]

    def step(i=None):
        if i is not None:
            marks[i][0].record(stream)
        st.build_mask(stream)
        if i is not None:
            marks[i][1].record(stream)
        if split:
            st.attention(stream, tiles=(t0, t1), rows=(r0, r1))
        else:
            st.attention(stream)
        if i is not None:
            marks[i][2].record(stream)
        if split:
            st.overlap(stream, count=count, branches=(b0, b1))
            dist.all_reduce(st.loss)  # sum of the ranks' L_r; L = sum - (world - 1)
        else:
            st.overlap(stream)
        if i is not None:
            marks[i][3].record(stream)

    for _ in range(Wm):
        step()
    torch.cuda.synchronize()
    if st.check_status() != 0:
        raise RuntimeError(f"device status {st.check_status()}")
    # the attention's executed FLOPs, from the tile records its launch reads
    meta = st.tile_meta[t0:t1] if split else st.tile_meta[:st.num_tiles]
    attn_exec = attention_executed_flops(meta.cpu().numpy(), case.Hkv, case.Hq // case.Hkv, case.d)
    if split:
        attn_exec = float(PAR.global_count(attn_exec, device=dev))

    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.3)
    start, end = ev(), ev()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = start.elapsed_time(end)
    clk = clocks.stop()
    t_mask = statistics.mean(m[0].elapsed_time(m[1]) for m in marks)
    t_attn = statistics.mean(m[1].elapsed_time(m[2]) for m in marks)
    t_ov = statistics.mean(m[2].elapsed_time(m[3]) for m in marks)
    elapsed_ms = PAR.max_time_ms(elapsed_ms, device=dev)  # slowest rank (identity at N = 1)

    # ---- end to end through the public API with host buffers
    # each rank copies what its share reads: every key/value row, its query
    # rows, its branches' logits; and reads back the loss and its alphas
    pin = lambda x, dt: (torch.from_numpy(x).view(torch.bfloat16) if dt == "bf16" else torch.from_numpy(x)).pin_memory()
    pr0, pr1 = (r0, r1) if split else (0, case.num_rows)
    lr0, lr1 = (b0 * case.W, b1 * case.W) if split else (0, st.R)
    h_in = [torch.from_numpy(case.anchors).pin_memory(), pin(case.q[pr0:pr1], case.dtype), pin(case.k, case.dtype),
            pin(case.v, case.dtype), pin(case.draft[lr0:lr1], case.dtype), pin(case.teacher[lr0:lr1], case.dtype)]
    d_in = [st.anchors, st.q[pr0:pr1], st.k, st.v, st.draft[lr0:lr1], st.teacher[lr0:lr1]]
    h_loss = torch.empty(1, dtype=torch.float32).pin_memory()
    h_alpha = torch.empty(max(lr1 - lr0, 1), dtype=torch.float32).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in h_in)
    d2h = h_loss.numel() * 4 + (lr1 - lr0) * 4

    def e2e_step():
        for h, d in zip(h_in, d_in):
            d.copy_(h, non_blocking=True)
        step()
        h_loss.copy_(st.loss, non_blocking=True)
        h_alpha[:lr1 - lr0].copy_(st.alpha[lr0:lr1], non_blocking=True)

    Ke = min(K, 50 if h2d < 2e9 else 10)  # the host copies dominate; a few steps are plenty
    for _ in range(max(1, Wm // 2)):
        e2e_step()
    torch.cuda.synchronize()
    e_start, e_end = ev(), ev()
    if world > 1:
        dist.barrier()
    e_start.record(stream)
    for _ in range(Ke):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_end)
    e2e_ms = PAR.max_time_ms(e2e_ms, device=dev)
    if split:  # bytes moved per step by all ranks together
        h2d = int(PAR.global_count(h2d, device=dev))
        d2h = int(PAR.global_count(d2h, device=dev))
    status = st.check_status()

    peaks = load_peaks()
    attn_tflops = figs["flops"] / (t_attn * 1e-3) / 1e12
    ov_gbs = figs["ov_bytes"] / (t_ov * 1e-3) / 1e9
    kernels = {
        "tree_attention": {"bound": "tensor", "ms": t_attn, "achieved": attn_tflops, "unit": "TFLOP/s",
                           "peak": peaks["bf16"], "frac": attn_tflops / peaks["bf16"],
                           "useful_flops": figs["flops"], "visible_pairs": figs["pairs"],
                           "executed_flops": attn_exec, "useful_over_executed": figs["flops"] / attn_exec,
                           "executed_tflops": attn_exec / (t_attn * 1e-3) / 1e12},
        "tv_overlap_e2e": {"bound": "hbm", "ms": t_ov, "achieved": ov_gbs, "unit": "GB/s", "peak": peaks["hbm"],
                           "frac": ov_gbs / peaks["hbm"], "algorithmic_bytes": figs["ov_bytes"]},
        "build_tree_mask": {"ms": t_mask},
    }
    # A kernel timed inside a step run back to back for a second or more works
    # under the power cap: its tensor peak is the sustained GEMM figure; the
    # burst figure is reported beside it.
    long_region = elapsed_ms >= 1000.0 and peaks.get("bf16_sustained")
    tpeak = peaks["bf16_sustained"] if long_region else peaks["bf16"]
    kt = kernels["tree_attention"]
    kt["frac_burst"] = kt["frac"]
    kt["peak_burst"] = kt["peak"]
    kt["peak"] = tpeak
    kt["frac"] = kt["achieved"] / tpeak
    kt["traffic"] = measured_traffic(args.workload, "tree_attention")
    kernels["tv_overlap_e2e"]["traffic"] = measured_traffic(args.workload, "tv_overlap_e2e")
    dom = "tree_attention" if t_attn >= t_ov else "tv_overlap_e2e"
    kd = kernels[dom]
    peak_src = ("bf16_tflops_sustained: timed region %.1f s" % (elapsed_ms / 1e3) if long_region else "bf16_tflops burst"
                ) if dom == "tree_attention" else "hbm_gbs"
    roofline = {"bound": kd["bound"], "achieved": kd["achieved"], "peak": kd["peak"], "unit": kd["unit"],
                "frac": kd["frac"], "traffic": kd["traffic"], "kernel": dom,
                "peak_source": f"{peaks['source']} ({peak_src})"}
    if dom == "tree_attention":
        roofline["frac_burst"] = kd["frac_burst"]
    tokens = figs["R"]  # one logical batch, whatever the number of ranks
    value = tokens * K / (elapsed_ms * 1e-3)
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": Wm,
        "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": case.dtype, "data": "synthetic (seeded; no datasets or weights)",
        "config": config_dict(case, figs, args.workload, args.seed, world),
        "roofline": roofline,
        "kernels": kernels,
        "clocks": clk,
        "e2e": {"value": tokens * Ke / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / Ke, "steps": Ke},
        # mask, RoPE (two calls when split: query rows, key rows), attention, fused overlap
        "gpu_launches": (5 if split else 4) * K,
        "device_status": status,
    }
    if split:
        out["loss"] = st.loss.item() - (world - 1)
        out["shard"] = {"tiles": [t0, t1], "rows": [r0, r1], "branches": [b0, b1]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(case)
    if world == 1 and not args.no_lm_head:
        del st
        torch.cuda.empty_cache()
        out["kernels"]["lm_head_overlap"] = lm_head_measure(dev, peaks, args.seed, args.lm_head_vocab)
        out["kernels"]["gdn_tree"] = gdn_measure(dev, peaks, args.seed)
        try:  # a secondary measurement: an error is recorded, not raised
            out["kernels"]["sparse_tree_attention"] = sparse_measure(dev, peaks, args.seed)
        except Exception as exc:  # noqa: BLE001
            out["kernels"]["sparse_tree_attention"] = {"error": f"{type(exc).__name__}: {exc}"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands on the host cores, each
    step one bounded sample of the workload (ORACLE_PLAN, the plan the native
    arm's cpu_baseline uses) scaled to the full step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synthetic as SY
    world = int(os.environ.get("WORLD_SIZE", "1"))
    case = SY.make_workload(args.workload, seed=args.seed, workers=min(8, os.cpu_count() or 1))
    figs = case_figures(case)
    f64 = oracle_inputs(case)
    rng = np.random.default_rng(7)
    for _ in range(args.warmup):
        oracle_sample(case, rng, f64=f64, **ORACLE_PLAN)
    ests = []
    t0 = time.perf_counter()
    desc = ""
    for _ in range(args.steps):
        est, desc = oracle_sample(case, rng, f64=f64, **ORACLE_PLAN)
        ests.append(est)
    wall = time.perf_counter() - t0
    est = statistics.mean(ests)
    value = figs["R"] / est
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": est * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; no datasets or weights)",
           "impl": "reference",
           "config": config_dict(case, figs, args.workload, args.seed, world),
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                            "sample": desc + f"; mean of {args.steps} samples, {wall:.1f} s wall"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def attention_only(args):
    """Mask + RoPE + tree attention of one workload, no logits (a small
    device footprint, for profiling the attention kernel alone)."""
    import torch
    import synthetic as SY
    from tree_attention_masked_b200.build import build
    build()
    from tree_attention_masked_b200.scoring import ScoringStep
    dev = torch.device("cuda", 0)
    case = SY.make_workload(args.workload, seed=args.seed, workers=min(8, os.cpu_count() or 1), with_logits=False)
    figs = case_figures(case)
    st = ScoringStep(case.trunk_len, case.prompt_len, case.num_branches, case.W, case.Hq, case.Hkv, case.d,
                     torch.bfloat16 if case.dtype == "bf16" else torch.float32, 1, device=dev,
                     pack_terminal=case.pack_terminal, theta=case.theta, with_grad=False)
    st.load(case)
    stream = torch.cuda.current_stream(dev)
    st.build_mask(stream)
    for _ in range(args.warmup):
        st.attention(stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        st.attention(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    peaks = load_peaks()
    tf = figs["flops"] / (ms * 1e-3) / 1e12
    print(json.dumps({"metric": "RoPE + tree attention", "value": ms, "unit": "ms", "higher_is_better": False,
                      "workload": SY.WORKLOADS[args.workload], "achieved_tflops": tf,
                      "frac_burst": tf / peaks["bf16"], "useful_flops": figs["flops"],
                      "device_status": st.check_status()}), flush=True)


def lm_head_measure(dev, peaks, seed: int, V: int = 151936) -> dict:
    """The LM-head path timed on its own (not part of the step): overlap
    statistics, L and dL/dalpha straight from bf16 hidden states and heads at
    the 8B-style shape (64 branches x W 16 = 1,024 rows, hidden 4,096 for both
    models, V = 151,936).  The logits are formed twice (normalisers, then alpha)
    and never stored: useful FLOPs count each logit once (2 GEMMs), executed
    FLOPs both passes (4).  ms_with_grad_draft adds the third (draft-only) pass
    that writes dL/dz."""
    import torch
    import synthetic as SY
    from tree_attention_masked_b200 import specopd as S
    nb, W, H = 64, 16, 4096
    case = SY.make_lm_head_case("gqa8b-lm-head", nb, W, V, H, H, sig_t=3.0, sig_n=1.5, seed=seed,
                                workers=min(8, os.cpu_count() or 1))
    t = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    hd, wd, ht, wt = t(case.h_draft), t(case.w_draft), t(case.h_teacher), t(case.w_teacher)
    R = case.rows
    alpha = torch.empty(R, device=dev)
    loss = torch.empty(1, device=dev)
    ga = torch.empty(R, device=dev)
    ws = torch.empty(S.specopd_lm_head_workspace_bytes(R, V), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    grad = torch.empty(R, V, device=dev)
    call = lambda g: S.specopd_lm_head_overlap(hd, wd, ht, wt, nb, W, 0.0, alpha, loss, ws, status, grad_alpha=ga,
                                               grad=g, stream=stream)

    def time_ms(g, n=10):
        for _ in range(3):
            call(g)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            call(g)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    ms = time_ms(None)
    ms_grad = time_ms(grad)
    gemm = 2.0 * R * H * V
    useful = 2 * gemm / (ms * 1e-3) / 1e12
    executed = 4 * gemm / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "ms": ms, "achieved": useful, "unit": "TFLOP/s", "peak": peaks["bf16"],
            "frac": useful / peaks["bf16"], "useful_flops": 2 * gemm, "executed_flops": 4 * gemm,
            "executed_tflops": executed, "executed_frac": executed / peaks["bf16"], "device_status": status.item(),
            "ms_with_grad_draft": ms_grad, "launches_with_grad_draft": 6,
            "shape": f"rows {R} (B {nb} x W {W}), hidden {H} (draft and teacher), V {V}, bf16",
            "launches": 5}


def gdn_measure(dev, peaks, seed: int, H: int = 32) -> dict:
    """The GDN linear-attention path timed on its own (not part of the step):
    gated delta rule over the 8B-style tree (T 4,096, 64 branches x W 16,
    5,120 packed rows) with H heads of d_k = d_v = 128.  Work counts the
    sequential recurrence's multiply-adds (3 d_k d_v per token and head) over
    the trunk, the tokens between each anchor's C = 64 checkpoint and the
    anchor, and the branch tokens; the kernels run the chunked form, whose
    only sequential part is one step per trunk chunk, so the bound is the
    latency of one chunk step times the chunk count, not a throughput peak."""
    import torch
    import synthetic as SY
    from tree_attention_masked_b200 import specopd as S
    T, P, B, W = 4096, 1024, 64, 16
    case = SY.make_gdn_case("gqa8b-gdn", [(T, P, B)], W=W, H=H, seed=seed)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    anchors = torch.from_numpy(case.anchors).to(dev)
    trees = S.Trees(case.trunk_len, case.prompt_len, case.num_branches, W, anchors, True)
    q, k, v = bf(case.q), bf(case.k), bf(case.v)
    alpha, beta = torch.from_numpy(case.alpha).to(dev), torch.from_numpy(case.beta).to(dev)
    out = torch.empty(case.num_rows, H, 128, device=dev)
    ws = torch.empty(S.specopd_gdn_workspace_bytes(trees, H), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda: S.specopd_gdn_tree(trees, q, k, v, alpha, beta, out, ws, status, stream=stream)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    n = 10
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    replay = int(sum((int(a) + 1) % 64 for a in case.anchors))
    tokens = T + replay + B * W
    flops = 2.0 * 3 * 128 * 128 * H * tokens
    return {"bound": "latency (sequential over the trunk's chunks)", "ms": ms,
            "achieved": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "flops": flops, "trunk_tokens": T,
            "trunk_chunks": T // 64, "anchor_offsets": replay, "branch_tokens": B * W,
            "device_status": status.item(),
            "shape": f"T {T}, B {B} x W {W}, {H} heads, d_k = d_v = 128, bf16 features, fp32 state",
            "launches": 4}


def sparse_measure(dev, peaks, seed: int) -> dict:
    """Sparse attention with branch-consistent indexer groups timed on its own
    (not part of the step), on the shape of the GPU parity test's full-size
    case: the 8B-style tree (T 4,096, 64 branches x W 16), 32/8 heads, d 128,
    64-token groups, top-8, 64-wide indexer features.  Useful FLOPs count the
    attended (row, column) pairs, 4 d per pair and query head; the tensor-core
    kernel executes the tree's visible key blocks with the unselected groups
    masked (executed FLOPs count every visible pair)."""
    import torch
    import synthetic as SY
    from tree_attention_masked_b200 import specopd as S
    g, topk, W = 64, 8, 16
    case = SY.make_sparse_case("gqa8b-sparse", [(4096, 1024, 64)], W, 32, 8, 64, seed=seed)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    anchors = torch.from_numpy(case.anchors).to(dev)
    trees = S.Trees(case.trunk_len, case.prompt_len, case.num_branches, W, anchors, True)
    N = case.num_rows
    i32 = dict(dtype=torch.int32, device=dev)
    pos, trunk_limit, branch_of = (torch.empty(N, **i32) for _ in range(3))
    anc_bits = torch.empty(N, dtype=torch.int64, device=dev)
    pred_rows = torch.empty(max(int(sum(case.num_branches)) * W, 1), **i32)
    cu_rows = torch.empty(2, **i32)
    tile_meta = torch.empty(max(S.specopd_tree_num_tiles(trees), 1), 8, **i32)
    status = torch.zeros(1, **i32)
    S.specopd_build_tree_mask(trees, pos, trunk_limit, branch_of, anc_bits, pred_rows, cu_rows, tile_meta, status)
    q, k, v, qi, ki = bf(case.q), bf(case.k), bf(case.v), bf(case.qi), bf(case.ki)
    out = torch.empty(N, 32, 128, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(S.specopd_sparse_workspace_bytes(trees, 32, 8, 64, g, topk), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda: S.specopd_sparse_tree_attention(trees, q, k, v, qi, ki, out, pos, trunk_limit, anc_bits,
                                                   tile_meta, g, topk, 1e4, ws, status, stream=stream)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    n = 10
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    # attended pairs: per row, its chosen groups' members and its tail
    T0 = 4096
    pairs = 0
    vis = 0
    for r in range(N):
        p = r if r < T0 else int(case.anchors[(r - T0) // W]) + 1 + (r - T0) % W
        nc = (p + 1) // g
        pairs += min(nc, topk) * g + (p + 1 - nc * g)
        vis += p + 1
    flops = 4.0 * 128 * 32 * pairs
    achieved = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor (masked tree attention over the selected groups)", "ms": ms, "achieved": achieved,
            "unit": "TFLOP/s", "peak": peaks["bf16"], "frac": achieved / peaks["bf16"], "useful_flops": flops,
            "attended_pairs": pairs, "visible_pairs": vis,
            "executed_tflops": 4.0 * 128 * 32 * vis / (ms * 1e-3) / 1e12, "device_status": status.item(),
            "shape": "T 4096, B 64 x W 16, 32/8 heads, d 128, groups of 64, top-8, indexer width 64, bf16",
            "launches": 4}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=WORKLOAD_DEFAULT)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-lm-head", action="store_true",
                    help="skip the separately timed next-row paths (LM head, GDN, sparse attention)")
    ap.add_argument("--lm-head-only", action="store_true",
                    help="time only the LM-head path (one JSON line; for profiling it alone)")
    ap.add_argument("--lm-head-vocab", type=int, default=151936, help="vocabulary of the LM-head path")
    ap.add_argument("--gdn-only", action="store_true", help="time only the GDN path (one JSON line)")
    ap.add_argument("--sparse-only", action="store_true", help="time only the sparse indexer-group attention")
    ap.add_argument("--attention-only", action="store_true",
                    help="time only RoPE + tree attention of the workload (no logits; for profiling)")
    args = ap.parse_args()
    # at least three untimed warm-up steps, whatever was asked for
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        run_reference(args)
    elif args.attention_only:
        attention_only(args)
    elif args.sparse_only:
        import torch
        from tree_attention_masked_b200.build import build
        build()
        d = sparse_measure(torch.device("cuda", 0), load_peaks(), args.seed)
        print(json.dumps({"metric": "sparse attention with indexer groups over the proposal tree", "value": d["ms"],
                          "unit": "ms", "higher_is_better": False, "kernel": d}), flush=True)
    elif args.gdn_only:
        import torch
        from tree_attention_masked_b200.build import build
        build()
        d = gdn_measure(torch.device("cuda", 0), load_peaks(), args.seed)
        print(json.dumps({"metric": "GDN over the proposal tree (indexed state replay)", "value": d["ms"],
                          "unit": "ms", "higher_is_better": False, "kernel": d}), flush=True)
    elif args.lm_head_only:
        import torch
        from tree_attention_masked_b200.build import build
        build()
        d = lm_head_measure(torch.device("cuda", 0), load_peaks(), args.seed, args.lm_head_vocab)
        print(json.dumps({"metric": "LM head + overlap statistics (logits never stored)", "value": d["achieved"],
                          "unit": d["unit"], "higher_is_better": True, "kernel": d}), flush=True)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
