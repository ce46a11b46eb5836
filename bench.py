"""Benchmark of the Token Sparse Attention prefill hot path on B200.

One step = the whole hot path over one layer of the L=131072 workload
(B=1, 32 query / 8 KV heads, d=128, bf16, window 64, keep 0.1 per KV head):
tsa_score -> tsa_select -> tsa_attend (gather, causal attention on the
compressed tensors, scatter + zero fill), with inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tsa|reference]

N > 1 runs under torchrun, one independent layer per rank (weak scaling, no
collective on the data path); the step time is the max over ranks of the
device-timed region.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference the pages
allow: their authors' kernels are not available) on a bounded sample of the
same workload, scaled to the same metric.
"""

from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed-attention prefill tokens/s at 128K; TFLOPS and % of B200 bf16 peak"
WORKLOAD = "gqa_bf16_L131072"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers


def attend_flops(w, budgets) -> float:
    """Compacted causal attention flops: per query head, QK^T and PV over the
    lower triangle including the diagonal, 2 flops per multiply-add."""
    total = 0.0
    for b in range(w.B):
        for g in range(w.Hkv):
            K = min(budgets[b * w.Hkv + g], w.L)
            total += w.G * 4.0 * w.D * K * (K + 1) / 2.0
    return total


def block_mask_for(w, density: float, seed: int = 5) -> np.ndarray:
    """Seeded uint8 [B, Hkv, nb, nb] block mask: diagonal blocks, the first block column
    (attention sinks) and a `density` fraction of the other blocks."""
    nb = -(-w.L // 128)
    rng = np.random.default_rng(seed)
    bm = (rng.random((w.B, w.Hkv, nb, nb)) < density).astype(np.uint8)
    bm[:, :, np.arange(nb), np.arange(nb)] = 1
    bm[:, :, :, 0] = 1
    return bm


def block_sparse_flops(w, budgets, bm) -> float:
    """Flops of the visible (query, key) pairs: causal inside enabled 128 x 128 blocks."""
    total = 0.0
    for b in range(w.B):
        for g in range(w.Hkv):
            K = min(budgets[b * w.Hkv + g], w.L)
            n = -(-K // 128)
            sizes = np.minimum(128, K - 128 * np.arange(n)).astype(np.float64)
            m = bm[b, g, :n, :n].astype(bool)
            low = np.tril(m, -1)
            pairs = (sizes[:, None] * sizes[None, :] * low).sum()
            pairs += (sizes * (sizes + 1) / 2 * np.diag(m)).sum()
            total += w.G * 4.0 * w.D * pairs
    return total


# Share of the score's exponentials that run on the exponential unit: in every
# 16-pair chunk, pairs 2, 5, 8, 11 and 14 use the FMA-pipe polynomial instead.
SCORE_MUFU_SHARE = 11.0 / 16.0


def other_rooflines(w, t_score_ms: float, t_select_ms: float, peaks, peak_src: str):
    """The step's other kernels against their own bounds.

    score: the exponential unit (16 ex2 per clock per SM; both passes exponentiate
    every (window row, key) logit once); select: HBM, on its algorithmic bytes
    (scores read once, the permutation written once), which it cannot approach
    because it is latency-bound (64 CTAs, cluster barriers between radix passes)."""
    sms, mhz = 148, 1965.0
    if torch.cuda.is_available():
        sms = torch.cuda.get_device_properties(0).multi_processor_count
    exps = 2.0 * w.B * w.Hkv * w.G * w.W * w.L
    mufu_peak = 16.0 * sms * mhz * 1e6
    a_score = exps / (t_score_ms * 1e-3)
    sel_bytes = 2.0 * 4 * w.B * w.Hkv * w.L
    a_sel = sel_bytes / (t_select_ms * 1e-3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    # score bytes: K read once, the window queries, the scores written (the second pass re-reads K
    # mostly from L2 and is not counted)
    esz = 2 if w.dtype == "bf16" else 4
    sc_bytes = (w.B * w.Hkv * w.L * w.D + w.B * w.Hq * w.W * w.D) * esz + 4.0 * w.B * w.Hkv * w.L
    a_sc_hbm = sc_bytes / (t_score_ms * 1e-3) / 1e9
    return [
        {"kernel": "score_tc (2 passes)", "bound": "alu", "achieved": a_score / 1e12, "peak": mufu_peak / 1e12,
         "unit": "Tex2/s", "frac": a_score / mufu_peak,
         "peak_source": f"16 ex2/clk/SM x {sms} SMs x {mhz:.0f} MHz (max SM clock)",
         "mufu_share": SCORE_MUFU_SHARE, "mufu_issued_achieved": a_score * SCORE_MUFU_SHARE / 1e12,
         "mufu_issued_frac": a_score * SCORE_MUFU_SHARE / mufu_peak,
         "note": "achieved/frac count every exponential (an effective rate: 5 pairs in 16 run on the FMA "
                 "pipe); mufu_issued_* count only those the exponential unit executes"},
        {"kernel": "score_tc (2 passes)", "bound": "hbm", "achieved": a_sc_hbm, "peak": hbm, "unit": "GB/s",
         "frac": a_sc_hbm / hbm, "peak_source": f"hbm_gbs ({peak_src})",
         "note": "algorithmic bytes (K once, window queries, scores); the exponentials bound it first"},
        {"kernel": "select_radix", "bound": "hbm", "achieved": a_sel, "peak": hbm, "unit": "GB/s",
         "frac": a_sel / hbm, "peak_source": f"hbm_gbs ({peak_src})", "note": "latency-bound: 64 CTAs, cluster barriers between 4 radix passes"},
    ]


def time_zero_dropped(T, w, desc, perm, budgets, out, ws, stream, dev, peaks, peak_src, workload, reps=10):
    """The scatter's zero rows as a standalone kernel (tsa_zero_dropped) on the step's
    permutation, against HBM: 2 bytes x D per dropped row per query head written,
    4 bytes per dropped row read (its position).  In the step itself these zeros are
    written by spare warps of the attention kernel."""
    dropped = sum(w.L - min(int(x), w.L) for x in budgets)
    nbytes = dropped * (w.G * w.D * (2 if w.dtype == "bf16" else 4) + 4)
    if nbytes == 0:
        return None
    for _ in range(3):
        T.tsa_zero_dropped(desc, perm, budgets, out, ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        T.tsa_zero_dropped(desc, perm, budgets, out, ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    if T.tsa_check_status(ws) != 0:
        raise RuntimeError("device status after the zero-fill timing")
    hbm = float(peaks["hbm_gbs"])
    a = nbytes / (ms * 1e-3) / 1e9
    traffic, src = kernel_traffic("zero_fill", workload, ["long_context_tsa_b200/csrc/attend_simt.cu"])
    return {"kernel": "zero_fill (tsa_zero_dropped: the scatter's zero rows, standalone)", "bound": "hbm",
            "achieved": a, "peak": hbm, "unit": "GB/s", "frac": a / hbm, "traffic": traffic,
            "traffic_source": src, "traffic_capture": capture_note(src), "ms": ms, "algorithmic_bytes": nbytes,
            "peak_source": f"hbm_gbs ({peak_src})",
            "note": f"{dropped} dropped rows x {w.G} query heads; timed alone, {reps} launches back to back"}


def out_proj_roofline(w, budgets, perm, t_ms, peaks, peak_src):
    """tsa_out_proj against the tensor-core peak on its useful flops: every kept
    (position, KV group) row times the group's G*D columns of W_o times hidden,
    2 flops per multiply-add; beside it the HBM bytes of the rows it must touch
    (the residual rows of positions any group kept, read and written, and the
    kept attention rows read once)."""
    hidden = w.Hq * w.D
    kept = [min(int(x), w.L) for x in budgets]
    flops = 2.0 * sum(kept) * w.G * w.D * hidden
    pm = perm.cpu().numpy()
    union = 0
    for b in range(w.B):
        m = np.zeros(w.L, bool)
        for g in range(w.Hkv):
            m[pm[b, g, :kept[b * w.Hkv + g]]] = True
        union += int(m.sum())
    esz = 2 if w.dtype == "bf16" else 4
    nbytes = union * hidden * esz * 2 + sum(kept) * w.G * w.D * esz
    a = flops / (t_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    hbm = float(peaks["hbm_gbs"])
    return {"kernel": "out_proj (mask sort + op_tc: projection of the kept rows + residual)", "bound": "tensor",
            "achieved": a, "peak": peak, "unit": "TFLOP/s", "frac": a / peak, "ms": t_ms, "useful_flops": flops,
            "hbm_bytes": nbytes, "hbm_frac": nbytes / (t_ms * 1e-3) / 1e9 / hbm, "positions_kept_by_any_group": union,
            "peak_source": f"bf16_tflops ({peak_src}); hbm_gbs for hbm_frac"}


def capture_note(src):
    """Provenance of a traffic figure read from a committed ncu summary."""
    if not src:
        return None
    text = open(os.path.join(ROOT, src)).read()
    m = re.search(r"captured:\s*(.+)", text)
    when = m.group(1).strip() if m else "date not recorded"
    return f"committed ncu capture {src} ({when}); valid while the kernel source hash matches"


def input_checksum(*tensors) -> str:
    """Sum of the raw element bits of each tensor (int64, on the device): identifies the exact inputs."""
    parts = []
    for t in tensors:
        bits = t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)
        parts.append(str(int(bits.to(torch.int64).sum().item())))
    return ":".join(parts)


def rank_seed(rank: int) -> int:
    """Each rank runs its own independent layer (weak scaling): inputs seeded by rank."""
    return rank


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of per-rank timings (the job is as slow as its slowest rank)."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's tokens over the (max-over-ranks) step time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_traffic(kernel_tag: str, workload: str, src_files):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (its sha256 is recorded in the summary)."""
    digest = hashlib.sha256()
    for f in src_files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            digest.update(fh.read())
    want = digest.hexdigest()[:16]
    for path in glob.glob(os.path.join(ROOT, "profiles", f"{kernel_tag}*{workload}*.md")):
        text = open(path).read()
        m_src = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
        m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
        if m_src and m_tr and m_src.group(1) == want:
            return float(m_tr.group(1)), os.path.relpath(path, ROOT)
    return None, None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        self.t0 = self.t1 = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        props = torch.cuda.get_device_properties(self.device)
        bus = getattr(props, "pci_bus_id", None)
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    pci_bus = int(parts[0].split(":")[1], 16)
                except Exception:
                    pci_bus = None
                if bus is not None and pci_bus is not None and pci_bus != bus:
                    continue
                rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return None
        # Samples are at 50 ms; drop the idle ones before/after the load.
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ----------------------------------------------------------------------------- CPU oracle timing


ORACLE_ROWS_PER_HEAD = 256  # attention rows the oracle computes per query head in one sampled step


def oracle_sample(w, q, k, v, budgets, rows_per_head=ORACLE_ROWS_PER_HEAD, seed=0):
    """Time one sampled step of the oracle and extrapolate it to the full step.

    The one sampling scheme of both CPU legs (the GPU line's cpu_baseline and
    --impl reference): score over every query head (full), select over every KV
    group (full), attention on `rows_per_head` seeded kept rows of every query
    head, the attention time scaled by (all kept rows) / (sampled rows).
    q, k, v: host float32 arrays.  Returns a dict with the measured wall time,
    the per-part times, the scale factor and the extrapolated full-step time.
    """
    from oracle import tsa_oracle as O

    rng = np.random.default_rng(seed)
    t0 = time.perf_counter()
    sc = O.score(q, k, w.W)
    t1 = time.perf_counter()
    perm = O.select(sc.astype(np.float32), budgets)
    t2 = time.perf_counter()
    kept = O.clamp_budgets(budgets, w.L)
    n_rows = 0
    for b in range(w.B):
        for h in range(w.Hq):
            g = h // w.G
            K = int(kept[b * w.Hkv + g])
            rows = rng.choice(K, size=min(rows_per_head, K), replace=False)
            O.attend_rows(q, k, v, perm[b, g], K, b, h, w.G, rows)
            n_rows += rows.size
    t3 = time.perf_counter()
    total_rows = int(sum(w.G * int(x) for x in kept))
    scale = total_rows / max(1, n_rows)
    est = (t1 - t0) + (t2 - t1) + (t3 - t2) * scale
    sample = (f"score all {w.B * w.Hq} query heads and select all {w.B * w.Hkv} KV groups in full; attention on "
              f"{rows_per_head} seeded kept rows per query head ({n_rows} of {total_rows} kept rows, time scaled "
              f"x{scale:.1f}); fp64 numpy")
    return {"wall_s": t3 - t0, "score_s": t1 - t0, "select_s": t2 - t1, "attend_s": t3 - t2, "attend_scale": scale,
            "est_s": est, "sample": sample}


def make_inputs(I, w, seed):
    """The workload's seeded inputs, drawn by torch's CUDA generator when a GPU is
    present (both arms then time the same tensors), else by its CPU generator."""
    if torch.cuda.is_available():
        return I.make_qkv(w, seed=seed, device="cuda"), "torch CUDA generator"
    return I.make_qkv(w, seed=seed, device="cpu"), "torch CPU generator (no GPU on this host)"


# ----------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tsa", choices=["tsa", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--e2e-slots", type=int, default=2, help="streams / buffer sets the end-to-end leg rotates over")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--op", default="forward",
                    choices=["forward", "forward-accumulate", "forward-coverage", "forward-block-sparse",
                             "forward-out-proj", "drift", "sweep"],
                    help="forward: score/select/attend (the headline); forward-accumulate: the same with the "
                         "scatter-add attention into a resident output; forward-coverage: budgets chosen per KV "
                         "head from the coverage --tau (one device-to-host copy of the budgets per step); "
                         "forward-block-sparse: attention restricted by a 128 x 128 block mask of --density in the "
                         "compressed space; forward-out-proj: the forward followed by the output projection of the "
                         "attention output added to a resident residual (tsa_out_proj, hidden = Hq * D); drift: the "
                         "representation-drift pass; sweep: the sparsity sweep at "
                         "128K against dense causal attention in the same library (K = L)")
    ap.add_argument("--density", type=float, default=0.5, help="block density for --op forward-block-sparse")
    ap.add_argument("--tau", type=float, default=0.005, help="token coverage for --op forward-coverage")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from long_context_tsa_b200 import inputs as I

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.op == "drift":
        bench_drift(args, I, world, rank, local)
        return
    if args.op == "sweep":
        bench_sweep(args, I, world, rank, local)
        return
    w = I.WORKLOADS[args.workload]
    budgets = w.budgets(seed=0)

    if args.impl == "reference":
        if rank != 0:
            return
        run_reference(args, w, budgets, world)
        return

    import long_context_tsa_b200 as T

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    q, k, v = I.make_qkv(w, seed=rank_seed(rank), device=dev)  # the reference arm draws the same tensors
    desc = T.desc_for(q, k)
    ws = T.alloc_workspace(desc, w.W, device=dev)
    scores = torch.empty((w.B, w.Hkv, w.L), dtype=torch.float32, device=dev)
    perm = torch.empty((w.B, w.Hkv, w.L), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    accumulate = args.op == "forward-accumulate"
    coverage = args.op == "forward-coverage"
    block_sparse = args.op == "forward-block-sparse"
    out_proj = args.op == "forward-out-proj"
    if out_proj:  # the residual stream and a seeded projection weight (hidden = Hq * D)
        hidden = w.Hq * w.D
        gx = torch.Generator(device=dev).manual_seed(1000 + rank)
        x_res = torch.randn((w.B, w.L, hidden), generator=gx, device=dev).to(q.dtype)
        w_o = (torch.randn((hidden, hidden), generator=gx, device=dev) / math.sqrt(hidden)).to(q.dtype)
        op_ws = T.alloc_out_proj_workspace(desc, device=dev)
    bm_host = block_mask_for(w, args.density) if block_sparse else None
    bm_dev = torch.from_numpy(bm_host).to(dev) if block_sparse else None
    if accumulate:
        out.normal_()  # the residual the attention output is added into
    kdev = torch.empty(w.B * w.Hkv, dtype=torch.int32, device=dev)

    def step(ev=None):
        nonlocal budgets
        if ev is not None:
            ev[0].record(stream)
        T.tsa_score(desc, q, k, w.W, scores, ws)
        if ev is not None:
            ev[1].record(stream)
        if coverage:
            T.tsa_select_coverage(desc, scores, args.tau, perm, kdev, ws)
            budgets = kdev.tolist()  # the attention grid is sized from them
        else:
            T.tsa_select(desc, scores, budgets, perm, ws)
        if ev is not None:
            ev[2].record(stream)
        if accumulate:
            T.tsa_attend_accumulate(desc, q, k, v, perm, budgets, out, ws)
        elif block_sparse:
            T.tsa_attend_block_sparse(desc, q, k, v, perm, budgets, bm_dev, out, ws)
        else:
            T.tsa_attend(desc, q, k, v, perm, budgets, out, ws)
        if ev is not None:
            ev[3].record(stream)
        if out_proj:
            T.tsa_out_proj(desc, out, perm, budgets, w_o, x_res, op_ws)
            if ev is not None:
                ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = T.tsa_check_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {T.tsa_status_string(st)}")

    # L2 (126 MB) is flushed between timed steps: a 256 MB buffer is written, then
    # another 256 MB buffer is read, so the step starts on a cold L2 that holds no
    # dirty lines to write back.  Each step is timed by its own events, so the
    # flushes sit outside the step times.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.zeros(64 << 20, dtype=torch.int32, device=dev)

    def flush_l2():
        flush.zero_()
        flush_rd.sum()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    last = 4 if out_proj else 3  # the event that ends a step
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = T.tsa_debug_launch_count()
    start.record(stream)
    for i in range(args.steps):
        flush_l2()
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    launches = T.tsa_debug_launch_count() - launches0
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop()
    st = T.tsa_check_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after timing: {T.tsa_status_string(st)}")

    loop_ms = start.elapsed_time(end)  # includes the flushes
    steps_ms = sum(e[0].elapsed_time(e[last]) for e in evs)
    t_score = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_select = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    t_attend = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    steps_ms, t_attend, loop_ms = max_over_ranks([steps_ms, t_attend, loop_ms], dist, dev)
    ms_per_step = steps_ms / args.steps
    tokens = w.B * w.L
    value = job_tokens_per_s(world, tokens, ms_per_step)

    peaks, peak_src = load_peaks()
    flops = block_sparse_flops(w, budgets, bm_host) if block_sparse else attend_flops(w, budgets)
    achieved = flops / (t_attend / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    # The committed DRAM capture is of the plain forward's attention launch (fixed budgets, no mask, zero
    # fill, no accumulate); other ops launch it differently, so they carry no traffic figure.
    traffic, traffic_src = (kernel_traffic("attend", args.workload, ["long_context_tsa_b200/csrc/attend_tc.cu",
                                                                        "long_context_tsa_b200/csrc/tc_ptx.cuh"])
                            if args.op in ("forward", "forward-out-proj") else (None, None))
    op_line = None
    if out_proj:
        if T.tsa_check_status(op_ws) != 0:
            raise RuntimeError("device status of the output projection")
        t_op = statistics.mean(e[3].elapsed_time(e[4]) for e in evs)
        op_line = out_proj_roofline(w, budgets, perm, t_op, peaks, peak_src)
    zf = None
    if not coverage:
        zf = time_zero_dropped(T, w, desc, perm, budgets, out, ws, stream, dev, peaks, peak_src, args.workload)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(T, w, desc, q, k, v, budgets, dev, stream, args.e2e_steps, dist, args.e2e_slots)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        qn, kn, vn = (t.float().cpu().numpy() for t in (q, k, v))
        res = oracle_sample(w, qn, kn, vn, budgets)
        cpu = {"value": tokens / res["est_s"], "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": res["sample"] + f"; {res['wall_s']:.1f} s of CPU work, extrapolated full step "
                                         f"{res['est_s']:.1f} s",
               "measured_wall_ms_per_step": res["wall_s"] * 1e3, "full_step_ms_estimated": res["est_s"] * 1e3,
               "attend_scale": res["attend_scale"]}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "op": args.op, "tau": args.tau if args.op == "forward-coverage" else None,
                   "block_density": args.density if block_sparse else None,
                   "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "D": w.D, "W": w.W,
                   "K_per_kv_head": budgets,
                   "l2": ("flushed between timed steps (256 MB written, then 256 MB read, outside the per-step events); "
                          f"inputs also exceed L2: q {q.numel() * q.element_size() / 1e9:.2f} GB, "
                          f"k and v {k.numel() * k.element_size() / 1e6:.0f} MB each"),
                   "timed_loop_ms_incl_flushes": loop_ms,
                   "parallelism": f"{world} independent layers, one per GPU",
                   "input_checksum": input_checksum(q, k, v)},
        "breakdown_ms": {"score": t_score, "select": t_select, "attend": t_attend,
                         **({"out_proj": op_line["ms"]} if op_line else {})},
        "attend_tflops": achieved,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": f"bf16_tflops ({peak_src})",
                     "kernel": "attend_tc (tsa_attend: gather + attention + scatter + zero fill)",
                     "traffic_source": traffic_src, "traffic_capture": capture_note(traffic_src)},
        "rooflines_other": other_rooflines(w, t_score, t_select, peaks, peak_src) + ([zf] if zf else []) +
        ([op_line] if op_line else []),
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": launches,
    }
    print(json.dumps(line), flush=True)


def bench_sweep(args, I, world, rank, local):
    """Sparsity sweep at L=131072 against dense causal attention in the same library.

    For each tau in the sweep, K = floor((1 - tau) L) per KV head: the whole step
    (score, select, attend) and the attention alone are timed; the dense
    baseline is tsa_attend with K = L (identity permutation), the ordinary causal
    attention of the layer.  Speedups are dense attention time over the TSA step
    (what a layer gains, scoring included) and over the TSA attention alone --
    the quantity the pages quote as "up to 3.23x at 128K" on their own setting."""
    import long_context_tsa_b200 as T

    if args.impl == "reference" or world > 1:
        if rank == 0:
            print(json.dumps({"impl": args.impl, "unavailable": "the sweep is a single-GPU context measurement"}),
                  flush=True)
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = I.WORKLOADS["gqa_bf16_L131072"]
    q, k, v = I.make_qkv(w, seed=0, device=dev)
    desc = T.desc_for(q, k)
    ws = T.alloc_workspace(desc, w.W, device=dev)
    scores = torch.empty((w.B, w.Hkv, w.L), dtype=torch.float32, device=dev)
    perm = torch.empty((w.B, w.Hkv, w.L), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, reps):
        for _ in range(max(1, args.warmup)):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    dense_b = [w.L] * (w.B * w.Hkv)
    ident = torch.arange(w.L, dtype=torch.int32, device=dev).expand(w.B, w.Hkv, w.L).contiguous()
    t_dense = timed(lambda: T.tsa_attend(desc, q, k, v, ident, dense_b, out, ws), 3)
    rows = []
    for tau in I.SWEEP_TAUS:
        budgets = [I.sweep_budget(tau, w.L)] * (w.B * w.Hkv)

        def step():
            T.tsa_score(desc, q, k, w.W, scores, ws)
            T.tsa_select(desc, scores, budgets, perm, ws)
            T.tsa_attend(desc, q, k, v, perm, budgets, out, ws)

        t_step = timed(step, args.steps)
        t_att = timed(lambda: T.tsa_attend(desc, q, k, v, perm, budgets, out, ws), args.steps)
        fl = attend_flops(w, budgets)
        rows.append({"tau": tau, "K_per_kv_head": budgets[0], "step_ms": t_step, "attend_ms": t_att,
                     "attend_tflops": fl / (t_att * 1e-3) / 1e12, "speedup_vs_dense_step": t_dense / t_step,
                     "speedup_vs_dense_attend": t_dense / t_att})
    st = T.tsa_check_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after the sweep: {T.tsa_status_string(st)}")
    fl_dense = attend_flops(w, dense_b)
    print(json.dumps({
        "metric": "attention speedup vs dense causal attention (same library, K = L) at 128K",
        "unit": "x", "higher_is_better": True, "n_gpus": 1, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "op": "sweep", "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "D": w.D,
                   "W": w.W},
        "dense": {"attend_ms": t_dense, "attend_tflops": fl_dense / (t_dense * 1e-3) / 1e12},
        "sweep": rows,
        "pages_figure": "up to 3.23x at 128K (hardware and setting not stated on the pages; context only)",
    }), flush=True)


def bench_drift(args, I, world, rank, local):
    """Device-timed representation-drift pass over one [B, L, hidden] pair per rank (HBM-bound)."""
    import long_context_tsa_b200 as T

    cfg = I.DRIFT_WORKLOAD
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps({"impl": "reference", "unavailable": "the drift pass has no reference arm; its "
                              "oracle is timed only in the forward op's reference arm"}), flush=True)
        return
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    a, b = I.make_hidden(cfg["B"], cfg["L"], cfg["hidden"], cfg["dtype"], cfg["delta"], seed=rank_seed(rank),
                         device=dev)
    ws = T.alloc_drift_workspace(dev)
    drift = torch.empty(1, dtype=torch.float64, device=dev)
    rows = cfg["B"] * cfg["L"]
    row_cos = torch.empty(rows, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        T.tsa_drift(a, b, drift, ws, row_cos=row_cos)
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = T.tsa_debug_launch_count()
    start.record(stream)
    for _ in range(args.steps):
        T.tsa_drift(a, b, drift, ws, row_cos=row_cos)
    end.record(stream)
    torch.cuda.synchronize(dev)
    launches = T.tsa_debug_launch_count() - launches0
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop()
    (total_ms,) = max_over_ranks([start.elapsed_time(end)], dist, dev)
    value_drift = float(drift.item())
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    ms = total_ms / args.steps
    nbytes = 2 * a.numel() * a.element_size() + 4 * rows  # both tensors read once, one float per row written
    achieved = nbytes / (ms / 1e3) / 1e9
    peaks, peak_src = load_peaks()
    peak = float(peaks["hbm_gbs"])
    traffic, traffic_src = kernel_traffic("drift", cfg["name"], ["long_context_tsa_b200/csrc/drift.cu"])
    line = {
        "metric": "representation-drift rows/s (hidden 4096, bf16)",
        "value": world * rows / (ms / 1e3),
        "unit": "rows/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg["dtype"],
        "data": "synthetic",
        "config": {"workload": cfg["name"], "op": "drift", "B": cfg["B"], "L": cfg["L"], "hidden": cfg["hidden"],
                   "delta": cfg["delta"], "drift": value_drift,
                   "l2": f"inputs larger than L2 (126 MB): {nbytes / 1e9:.2f} GB read per step; no flush",
                   "parallelism": f"{world} independent tensor pairs, one per GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_source": f"hbm_gbs ({peak_src})", "kernel": "drift_kernel",
                     "traffic_source": traffic_src},
        "cpu_baseline": None,
        "e2e": None,
        "clocks": clocks,
        "gpu_launches": launches,
    }
    print(json.dumps(line), flush=True)


def run_e2e(T, w, desc, q, k, v, budgets, dev, stream, steps, dist, n_slots=2):
    """Same metric through tsa_forward_host: pinned host inputs, the forward, and
    the full output copied back, all inside the timed region.  With pinned
    (device-mapped) inputs the library moves only what the step reads: K and the
    window rows of Q by copy, the kept rows of Q and V by a gather kernel that
    reads host memory in place.

    Steps rotate over `n_slots` streams, each with its own device buffers,
    workspace and pinned output buffer, the way a server overlaps requests:
    one step's host-to-device copy runs while earlier steps compute and copy
    their outputs back (the two directions use separate copy engines)."""
    qh = q.cpu().pin_memory()
    kh = k.cpu().pin_memory()
    vh = v.cpu().pin_memory()
    streams = [stream] + [torch.cuda.Stream(dev) for _ in range(n_slots - 1)]
    slots = []
    for _ in range(n_slots):
        slots.append({"qd": torch.empty_like(q), "kd": torch.empty_like(k), "vd": torch.empty_like(v),
                      "od": torch.empty_like(q), "oh": torch.empty(q.shape, dtype=q.dtype).pin_memory(),
                      "ws": T.alloc_workspace(desc, w.W, device=dev)})

    def one(i):
        sl = slots[i % n_slots]
        T.tsa_forward_host(desc, qh, kh, vh, w.W, budgets, sl["oh"], sl["qd"], sl["kd"], sl["vd"], sl["od"],
                           sl["ws"], stream=streams[i % n_slots])

    for i in range(n_slots):
        one(i)
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    s.record(streams[0])
    for st_ in streams[1:]:
        st_.wait_event(s)
    for i in range(steps):
        one(i)
    for st_ in streams[1:]:
        e1 = torch.cuda.Event()
        e1.record(st_)
        streams[0].wait_event(e1)
    e.record(streams[0])
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([s.elapsed_time(e) / steps], dist, dev)[0]
    for sl in slots:
        st = T.tsa_check_status(sl["ws"])
        if st != 0:
            raise RuntimeError(f"device status after e2e: {T.tsa_status_string(st)}")
    world = dist.get_world_size() if dist is not None else 1
    nb = lambda t: t.numel() * t.element_size()  # noqa: E731
    # The library's own count of what it moved host -> device for these buffers.
    h2d = T.tsa_forward_host_h2d_bytes(desc, w.W, budgets, qh, vh)
    full = nb(q) + nb(k) + nb(v)
    how = ("K and the window rows of Q copied; the kept rows of Q and V read in place from pinned, device-mapped "
           "host memory after the selection" if h2d < full else "q, k and v copied in full")
    return {"value": job_tokens_per_s(world, w.B * w.L, ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": nb(q), "ms_per_step": ms, "steps": steps,
            "pipeline": f"{n_slots} streams, {n_slots} buffer sets (copies of one step overlap the others)",
            "inputs": how, "h2d_bytes_full_copy": full}


def run_reference(args, w, budgets, world):
    """The oracle arm: W warm-up and K timed steps on the host cores (rank 0 only).

    Each step is one sampled oracle step (``oracle_sample``): `ms_per_step` is the
    wall time those steps actually took; `value` extrapolates each to the full
    layer (score and select in full, attention rows scaled) and reports tokens/s
    of the full step."""
    from long_context_tsa_b200 import inputs as I

    (q, k, v), gen = make_inputs(I, w, seed=0)
    checksum = input_checksum(q, k, v)
    qn, kn, vn = (t.float().cpu().numpy() for t in (q, k, v))
    del q, k, v
    walls, ests = [], []
    res = None
    for i in range(args.warmup + args.steps):
        res = oracle_sample(w, qn, kn, vn, budgets, seed=i)
        if i >= args.warmup:
            walls.append(res["wall_s"])
            ests.append(res["est_s"])
    ms = statistics.mean(walls) * 1e3
    est_ms = statistics.mean(ests) * 1e3
    value = w.B * w.L / (est_ms / 1e3)
    cpu = {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
           "sample": res["sample"] + " per step",
           "measured_wall_ms_per_step": ms, "full_step_ms_estimated": est_ms, "attend_scale": res["attend_scale"]}
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "op": args.op, "tau": None, "block_density": None,
                   "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "D": w.D, "W": w.W,
                   "K_per_kv_head": budgets, "parallelism": "rank 0 only, host cores",
                   "input_checksum": checksum, "inputs": gen},
        "timing": (f"ms_per_step is the measured wall time of one sampled oracle step ({ms:.0f} ms); value is "
                   f"B*L over the full step extrapolated from it ({est_ms:.0f} ms: score and select measured in "
                   f"full, attention x{res['attend_scale']:.1f})"),
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
