"""Benchmark of the block-sparse FlashAttention forward on B200.

Headline workload (one step = one pass of the hot path over one batch):
speculative + sparse decode, B=8, Hq=32, Hkv=8 (GQA 4), Lq=1, Lk=32768,
D=128, bf16, block 128: dense over the last 2048 keys plus 32 random missed
blocks per (b, kv-head), merged by the LSE combine -- one fused split-KV
kernel launch.  Metric: kept-K/V GB/s (algorithmic bytes: the distinct K and
V bytes attended + q + o + lse + table) against the measured HBM copy
bandwidth.

The prefill workloads (tiny block table, gated BSFA prefill at 32K,
vertical-slash prefill at 128K) are timed in the same run and reported under
"prefill" with kept-block TFLOP/s against the measured bf16 tensor peak.

python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Under torchrun each rank runs its own replica (independent problems, no
data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

DECODE_WORKLOAD = ("speculative+sparse decode B=8 Hq=32 Hkv=8 Lq=1 Lk=32768 D=128 bs=128, "
                   "dense last 2048 + 32 missed blocks")
METRIC = ("sparse-attn fwd kept-block TFLOP/s (% bf16 peak); "
          "decode kept-KV GB/s (% HBM)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = os.path.join(ROOT, "block_sparse_flashattention_sbfa_b200", "csrc")


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# sources each profiled kernel is built from (its ncu counters go stale when any changes)
KERNEL_SOURCES = {
    "decode_kernel": ("kernel_decode.cuh", "sbfa_ptx.cuh"),
    "prefill_kernel<Gated>": ("kernel_prefill.cuh", "sbfa_ptx.cuh"),
    "prefill_kernel<VS>": ("kernel_prefill.cuh", "sbfa_ptx.cuh"),
    "nsa_main_kernel": ("kernel_nsa.cuh", "kernel_prefill.cuh", "sbfa_ptx.cuh"),
}


def source_sha(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(CSRC, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel)
    if not e or kernel not in KERNEL_SOURCES or e.get("source_sha") != source_sha(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, gpu):
        self.gpu = gpu
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 7:
                self.samples.append(parts)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        loaded = [s for s in self.samples if s[6].isdigit() and int(s[6]) > 0] or self.samples
        sm = [int(s[0]) for s in loaded if s[0].isdigit()]
        reasons = sorted({names[i] for s in loaded for i in range(4) if s[2 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": int(self.samples[0][1]) if self.samples[0][1].isdigit() else None,
                "reasons": reasons, "samples": len(loaded)}


class Dist:
    """One process per GPU (RANK / WORLD_SIZE / LOCAL_RANK from the launcher).
    The only collectives are the barrier around the timed region and the
    max of the per-rank times: the replicas exchange no data."""

    def __init__(self, backend="nccl", device="cuda"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend, self.device = backend, device
        self.pg = None

    def init(self, torch):
        if self.world > 1:
            import torch.distributed as dist
            kw = {"timeout": datetime.timedelta(seconds=120)}
            if self.backend == "nccl":
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(self.backend, **kw)
            self.pg = dist

    def barrier(self, torch):
        if self.pg:
            self.pg.barrier()

    def max(self, torch, x):
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())


    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def tensor_roofline(flops, ms, peaks, peak_kind, kernel, launches=1):
    """Roofline object of a prefill step: algorithmic FLOPs over its CUDA-event
    time, against the measured bf16 burst peak (the step is timed alone)."""
    achieved = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
            "traffic": ncu_traffic(kernel), "peak_kind": peak_kind, "kernel": kernel,
            "launches_per_step": launches, "algorithmic_flops": flops}


def whole_job_rate(units_per_rank, max_ms, world):
    """Weak scaling: every rank processes the same units; the job's rate is
    all ranks' units over the slowest rank's time."""
    return units_per_rank * world / (max_ms * 1e-3)


def time_device(torch, dist, fn, steps, warmup, flush):
    """Per-step CUDA-event time of fn (ms, median over steps; max over ranks).

    The L2 flush runs before each step, outside the events; it is queued
    first so the GPU is still busy with it while the host issues the step,
    and the events bracket device time only (no host launch gap)."""
    for _ in range(warmup):
        flush()
        fn()
    dist.barrier(torch)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    t0 = time.perf_counter()
    for a, b in evs:
        flush()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    dist.barrier(torch)
    wall = time.perf_counter() - t0
    ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    return dist.max(torch, ms), wall


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

def decode_bytes(wl):
    t = wl.meta["table"]
    B, Lk, Hkv, D = wl.k.shape
    Hq = wl.q.shape[2]
    bs = wl.meta["kv_block"]
    spec = wl.meta["spec_end"] - wl.meta["spec_begin"]
    keys = 0
    for b in range(B):
        for g in range(Hkv):
            blocks = set(int(x) for x in t[b, g, 0] if x >= 0)
            keys += spec + sum(min(bs, Lk - j * bs) for j in blocks)
    kv = keys * D * 2 * 2
    qo = 2 * B * wl.q.shape[1] * Hq * D * 2 + B * Hq * wl.q.shape[1] * 4 + t.size * 4
    return kv + qo, kv


def bench_decode(torch, sb, dist, args, flush, peaks):
    wl = W.make_spec_decode()
    s0 = wl.meta["spec_begin"]
    q, k, v = (W.to_torch_bf16(x, "cuda") for x in (wl.q, wl.k, wl.v))
    tab = torch.from_numpy(wl.meta["table"]).cuda()
    ws = sb.decode_workspace(8, 8, 1, 32, "cuda")
    o = torch.empty_like(q)
    lse = torch.empty(8, 32, 1, dtype=torch.float32, device="cuda")
    ks, vs = k[:, s0:], v[:, s0:]

    def step():
        sb.speculative_sparse(q, ks, vs, True, k, v, tab, 128, ws=ws, out=o, lse=lse)

    ms, wall = time_device(torch, dist, step, args.steps, args.warmup, flush)
    nbytes, kv = decode_bytes(wl)
    gbs = nbytes / (ms * 1e-3) / 1e9
    res = dict(ms=ms, gbs=gbs, bytes=nbytes, kv_bytes=kv, wall=wall)
    # end to end through the public API: host buffers in, result back out
    hq, hk, hv = (W.to_torch_bf16(x).pin_memory() for x in (wl.q, wl.k, wl.v))
    ht = torch.from_numpy(wl.meta["table"]).pin_memory()
    ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(lse.shape, dtype=torch.float32).pin_memory()

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        tab.copy_(ht, non_blocking=True)
        step()
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    ems, _ = time_device(torch, dist, e2e_step, e2e_steps, 1, lambda: None)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, ht))
    d2h = ho.numel() * 2 + hl.numel() * 4
    res["e2e"] = {"value": round(nbytes / (ems * 1e-3) / 1e9, 3), "unit": "GB/s",
                  "ms_per_step": round(ems, 4), "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": d2h,
                  "note": "host->device copy of q, k, v (the whole cache) and table every step"}
    res["wl"] = wl
    return res


def gated_flops(keep, L, Hq, block=64):
    n = keep.shape[-1]
    n_qk = Hq * L * (L + 1) // 2
    diag = block * (block + 1) // 2
    n_pv = 0
    for h in range(Hq):
        kh = keep[0, h]
        tri = np.tril(kh.astype(np.int64), -1).sum()
        n_pv += int(tri) * block * block + n * diag
    return 2 * 128 * n_qk + 2 * 128 * n_pv, n_qk, n_pv


def bench_gated(torch, sb, dist, args, flush, peaks, peak_kind):
    # T was calibrated at L = 32768; a shorter run (profiling) keeps its first
    # L / 64 q-blocks, whose candidates j < i do not depend on L.
    L = args.gated_len
    T = np.load(os.path.join(ROOT, "tests", "golden", "gated_T_seed101.npy"))[:, :L // 64].copy()
    wl = W.make_gated(L=L)
    q, k, v = (W.to_torch_bf16(x, "cuda") for x in (wl.q, wl.k, wl.v))
    Tg = torch.from_numpy(T).cuda()
    n = T.shape[1]
    keep = torch.zeros((1, 32, n, n), dtype=torch.uint8, device="cuda")
    o, lse = sb.fwd_gated(q, k, v, Tg, keep_out=keep)
    torch.cuda.synchronize()
    flops, n_qk, n_pv = gated_flops(keep.cpu().numpy(), L, 32)
    kept = int(keep.sum().item())
    ms, _ = time_device(torch, dist, lambda: sb.fwd_gated(q, k, v, Tg, out=o, lse=lse),
                        max(3, args.steps // 10), args.warmup, flush)
    tf = flops / (ms * 1e-3) / 1e12
    res = {"workload": f"gated BSFA prefill B=1 Hq=32 Hkv=8 L={L} causal D=128 bf16 64x64 "
                       "tiles, T from seed-101 calibration (k=64)",
           "ms": round(ms, 4), "tflops": round(tf, 2), "flops": flops,
           "kept_tile_density": round(kept / (32 * n * (n + 1) / 2), 4),
           "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
           "roofline": tensor_roofline(flops, ms, peaks, peak_kind, "prefill_kernel<Gated>")}
    if not args.no_cpu_baseline and dist.rank == 0:
        try:
            res["oracle"] = oracle_sample_gated(wl, T, flops)
        except Exception as e:  # the GPU numbers stand without it
            res["oracle"] = {"error": f"{type(e).__name__}: {e}"}
    return res


def vs_flops(bc, bo, cc, ci, L, block=64):
    B, H, nqb = bc.shape
    diag = block * (block + 1) // 2
    pairs = 0
    for h in range(H):
        for i in range(nqb):
            offs = bo[0, h, i, :bc[0, h, i]] // block
            pairs += int((offs < i).sum()) * block * block + int((offs == i).sum()) * diag
            cols = ci[0, h, i, :cc[0, h, i]].astype(np.int64)
            m0, m1 = i * block, min((i + 1) * block, L)
            pairs += int(np.minimum(block, np.maximum(m1 - np.maximum(cols, m0), 0)).sum())
    return 4 * 128 * pairs, pairs


def bench_vs(torch, sb, dist, args, flush, peaks, peak_kind):
    wl = W.make_vertical_slash(L=args.vs_len)
    L = wl.q.shape[1]
    q, k, v = (W.to_torch_bf16(x, "cuda") for x in (wl.q, wl.k, wl.v))
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    vt = torch.from_numpy(wl.meta["vertical"]).cuda()
    st = torch.from_numpy(wl.meta["slash"]).cuda()
    conv = lambda: sb.convert_vertical_slash(sl, sl, vt, st, L)  # noqa: E731
    bc, bo, cc, ci = conv()
    o, lse = sb.fwd_vertical_slash(q, k, v, bc, bo, cc, ci, causal=True)
    torch.cuda.synchronize()
    flops, pairs = vs_flops(bc.cpu().numpy(), bo.cpu().numpy(), cc.cpu().numpy(),
                            ci.cpu().numpy(), L)
    steps = max(3, args.steps // 50)
    ms, _ = time_device(torch, dist, lambda: sb.fwd_vertical_slash(
        q, k, v, bc, bo, cc, ci, causal=True, out=o, lse=lse), steps, min(args.warmup, 3), flush)
    cms, _ = time_device(torch, dist, conv, steps, 1, flush)
    tf = flops / (ms * 1e-3) / 1e12
    dense = 4 * 128 * 32 * L * (L + 1) // 2
    res = {"workload": f"vertical-slash prefill B=1 H=32 L={L} causal D=128 bf16 "
                       "BM=BN=64, 1000 vertical + 6000 slash per head",
           "ms": round(ms, 3), "tflops": round(tf, 2), "flops": flops,
           "frac_of_causal_dense": round(flops / dense, 4),
           "convert_ms": round(cms, 4),
           "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
           "roofline": tensor_roofline(flops, ms, peaks, peak_kind, "prefill_kernel<VS>")}
    if not args.no_cpu_baseline and dist.rank == 0:
        try:
            res["oracle"] = oracle_sample_vs(wl, flops)
            res["oracle_convert"] = oracle_sample_vs_convert(wl)
        except Exception as e:
            res["oracle"] = {"error": f"{type(e).__name__}: {e}"}
    return res


def nsa_pairs(wl):
    """Exact visible (token, key) pairs of the NSA selection (causal)."""
    cu = wl.meta["cu_seqlens"]
    sel = wl.meta["sel"].astype(np.int64)
    T = sel.shape[0]
    tl = np.empty(T, dtype=np.int64)
    for s_ in range(len(cu) - 1):
        tl[cu[s_]:cu[s_ + 1]] = np.arange(cu[s_ + 1] - cu[s_])
    cnt = np.clip(tl[:, None, None] - 64 * sel + 1, 0, 64)
    cnt[sel < 0] = 0
    return int(cnt.sum())


def bench_nsa(torch, sb, dist, args, flush, peaks, peak_kind):
    seqlens = tuple(int(x) for x in args.nsa_seqlens.split(","))
    wl = W.make_nsa_varlen(seqlens=seqlens)
    q, k, v = (W.to_torch_bf16(x, "cuda")[0] for x in (wl.q, wl.k, wl.v))
    cu = torch.from_numpy(wl.meta["cu_seqlens"]).cuda()
    sel = torch.from_numpy(wl.meta["sel"]).cuda()
    total, H = q.shape[0], q.shape[1]
    ws = sb.varlen_selected_workspace(len(seqlens), total, max(seqlens), H, H, 16, "cuda")
    o = torch.empty_like(q)
    lse = torch.empty(H, total, dtype=torch.float32, device="cuda")
    step = lambda: sb.fwd_varlen_selected(q, k, v, cu, max(seqlens), sel, ws=ws, out=o, lse=lse)  # noqa: E731
    step()
    torch.cuda.synchronize()
    pairs = nsa_pairs(wl)
    flops = 4 * 128 * pairs
    ms, _ = time_device(torch, dist, step, max(3, args.steps // 10), args.warmup, flush)
    tf = flops / (ms * 1e-3) / 1e12
    acc_bytes = total * H * (128 + 2) * 4
    cu_txt = ", ".join(str(int(x)) for x in wl.meta["cu_seqlens"])
    res = {"workload": f"NSA selected attention, varlen cu_seqlens [{cu_txt}], Hq=Hkv=4, "
                        "D=128, bf16, top-16 blocks of 64 (block 0, 2 local, 13 random)",
            "ms": round(ms, 4), "tflops": round(tf, 2), "flops": flops,
            "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
            "roofline": tensor_roofline(flops, ms, peaks, peak_kind, "nsa_main_kernel",
                                        launches=7),
            "accumulator_bytes": acc_bytes,
            "note": "block-major in two passes over the units (row maxima, then exp2(S - M) V "
                    "added into an fp32 [token, head, 128] accumulator at L2); seven kernels and "
                    "two memsets per step (index count/scan/fill, unit table, pass 1, pass 2, "
                    "finalize)"}
    if not args.no_cpu_baseline and dist.rank == 0:
        try:
            res["oracle"] = oracle_sample_nsa(wl, flops)
        except Exception as e:
            res["oracle"] = {"error": f"{type(e).__name__}: {e}"}
    return res


def bench_table(torch, sb, dist, args, flush, peaks, peak_kind):
    wl = W.make_block_table()
    q, k, v = (W.to_torch_bf16(x, "cuda") for x in (wl.q, wl.k, wl.v))
    t = torch.from_numpy(wl.meta["table"]).cuda()
    o, lse = sb.fwd(q, k, v, t, 64, 64)
    ms, _ = time_device(torch, dist, lambda: sb.fwd(q, k, v, t, 64, 64, out=o, lse=lse),
                        args.steps, args.warmup, flush)
    flops = 4 * 128 * 2 * 256 * 8 * 64
    return {"workload": "block table B=1 H=2 Lq=256 Lk=1024 bs=64 (diag + 7 random of 16)",
            "ms": round(ms, 5), "tflops": round(flops / (ms * 1e-3) / 1e12, 3),
            "note": "launch-bound correctness workload"}


# ----------------------------------------------------------------------------
# CPU baseline: the oracle on the host cores
# ----------------------------------------------------------------------------

def cpu_baseline_decode(wl, steps=5, warmup=1):
    """The oracle over the whole decode workload (every (b, h) row): `warmup`
    untimed passes (they touch the inputs and warm the BLAS pools), then the
    median of `steps` timed passes."""
    import oracle
    t = wl.meta["table"]
    s0 = wl.meta["spec_begin"]
    nbytes, _ = decode_bytes(wl)

    def one():
        oracle.speculative_sparse(wl.q, wl.k[:, s0:], wl.v[:, s0:], True, wl.k, wl.v, t, 128,
                                  wl.scale)

    for _ in range(warmup):
        one()
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        one()
        times.append(time.perf_counter() - t0)
    sec = statistics.median(times)
    try:
        from threadpoolctl import threadpool_info
        blas = max((x.get("num_threads", 1) for x in threadpool_info()), default=1)
    except Exception:
        blas = None
    return {"value": round(nbytes / sec / 1e9, 4), "unit": "GB/s", "cores": os.cpu_count(),
            "blas_threads": blas, "kind": "oracle", "steps": steps, "warmup": warmup,
            "sample": f"the whole decode workload (all 256 (b, h) rows) per pass; {warmup} "
                      f"untimed pass(es), median of {steps} timed passes, {sec:.2f} s per pass"}


def _oracle_line(sec, sample_flops, full_flops, sample):
    """The oracle's rate on a bounded sample and its time extrapolated to the
    whole workload by the algorithmic FLOP count (pairs, not rows)."""
    return {"value": round(sample_flops / sec / 1e12, 6), "unit": "TFLOP/s",
            "cores": os.cpu_count(), "kind": "oracle", "sample": sample,
            "sample_seconds": round(sec, 3), "sample_flops": sample_flops,
            "extrapolated_full_seconds": round(sec * full_flops / sample_flops, 1)}


def gated_sample_flops(i, keep, block=64):
    """Algorithmic FLOPs of q-block i of one head (whole 64-row block): QK over
    every causal key, PV over the kept off-diagonal blocks plus the diagonal."""
    rows = np.arange(i * block, (i + 1) * block)
    qk = int((rows + 1).sum())
    pv = int(np.asarray(keep[:i]).sum()) * block * block + block * (block + 1) // 2
    return 2 * 128 * (qk + pv)


def oracle_sample_gated(wl, T, full_flops):
    """Head 0, its last (heaviest) q-block: gate from fp64 block maxima, then
    attention over the kept blocks."""
    import oracle
    L = wl.q.shape[1]
    i = L // 64 - 1
    rows = np.arange(i * 64, L)
    t0 = time.perf_counter()
    _, _, info = oracle.attend_gated(wl.q[:, :, :1], wl.k[:, :, :1], wl.v[:, :, :1], T[:1], 64,
                                     wl.scale, rows=lambda b, h: rows, return_keep=True)
    sec = time.perf_counter() - t0
    keep = info[(0, 0, i)][1]
    return _oracle_line(sec, gated_sample_flops(i, keep), full_flops,
                        f"head 0, q-block {i} (64 rows): gate over {i + 1} blocks, "
                        f"{int(keep.sum())} kept")


def vs_sample_pairs(bc, bo, cc, ci, i, L, block=64):
    """Visible (row, key) pairs of q-block i of head 0 under converted lists."""
    offs = bo[0, 0, i, :bc[0, 0, i]] // block
    pairs = int((offs < i).sum()) * block * block + int((offs == i).sum()) * (block * (block + 1) // 2)
    cols = ci[0, 0, i, :cc[0, 0, i]].astype(np.int64)
    m0, m1 = i * block, min((i + 1) * block, L)
    pairs += int(np.minimum(block, np.maximum(m1 - np.maximum(cols, m0), 0)).sum())
    return pairs


def oracle_sample_vs(wl, full_flops):
    """Head 0, its last (heaviest) q-block: the oracle's attention over the
    converted lists (the conversion of that q-block is done first and not
    timed; oracle_sample_vs_convert times conversion on its own)."""
    import oracle
    L = wl.q.shape[1]
    vert, slash = wl.meta["vertical"][:, :1], wl.meta["slash"][:, :1]
    i = L // 64 - 1
    rows = np.arange(i * 64, L)
    bc, bo, cc, ci = oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True,
                                                   qblocks=[i])
    t0 = time.perf_counter()
    oracle.attend_vertical_slash(wl.q[:, :, :1], wl.k[:, :, :1], wl.v[:, :, :1], bc, bo, cc, ci,
                                 64, 64, True, wl.scale, rows=lambda b, h: rows)
    sec = time.perf_counter() - t0
    pairs = vs_sample_pairs(bc, bo, cc, ci, i, L)
    return _oracle_line(sec, 4 * 128 * pairs, full_flops,
                        f"head 0, q-block {i} (64 rows): attention over its converted lists")


def oracle_sample_vs_convert(wl, n_qb=32):
    """The oracle's index conversion on n_qb q-blocks of head 0 (the last
    ones, whose causal range is the longest), extrapolated to every q-block of
    every head; compare with the GPU's convert_ms."""
    import oracle
    L, H = wl.q.shape[1], wl.q.shape[2]
    vert, slash = wl.meta["vertical"][:, :1], wl.meta["slash"][:, :1]
    nqb = L // 64
    qbs = list(range(nqb - n_qb, nqb))
    t0 = time.perf_counter()
    oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True, qblocks=qbs)
    sec = time.perf_counter() - t0
    return {"kind": "oracle", "unit": "s", "cores": os.cpu_count(),
            "sample": f"conversion of {n_qb} q-blocks of head 0", "sample_seconds": round(sec, 6),
            "extrapolated_full_seconds": round(sec * nqb * H / n_qb, 6)}


def nsa_sample_pairs(cu, sel, toks):
    """Visible (token, key) pairs of head 0 for tokens of sequence 0."""
    tl = toks - cu[0]
    s = sel[toks, 0].astype(np.int64)
    cnt = np.clip(tl[:, None] - 64 * s + 1, 0, 64)
    cnt[s < 0] = 0
    return int(cnt.sum())


def oracle_sample_nsa(wl, full_flops, n_tok=256):
    """Head 0, the last n_tok tokens of the first sequence (the most causal
    keys)."""
    import oracle
    cu, sel = wl.meta["cu_seqlens"], wl.meta["sel"]
    toks = np.arange(cu[1] - n_tok, cu[1])
    t0 = time.perf_counter()
    oracle.attend_selected_varlen(wl.q[0][:, :1], wl.k[0][:, :1], wl.v[0][:, :1], cu, sel[:, :1],
                                  64, True, wl.scale, rows=lambda h: toks)
    sec = time.perf_counter() - t0
    return _oracle_line(sec, 4 * 128 * nsa_sample_pairs(cu, sel, toks), full_flops,
                        f"head 0, the last {n_tok} tokens of sequence 0")


# ----------------------------------------------------------------------------
# main
# ----------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--headline-only", action="store_true",
                    help="time the decode headline only (same as --prefill none)")
    ap.add_argument("--prefill", default="gated,vertical_slash,nsa_varlen,block_table",
                    help="comma-separated prefill workloads to time after the headline, or none")
    ap.add_argument("--gated-len", type=int, default=32768,
                    help="sequence length of the gated workload (a multiple of 64, <= 32768)")
    ap.add_argument("--vs-len", type=int, default=131072,
                    help="sequence length of the vertical-slash workload (profiling runs use less)")
    ap.add_argument("--nsa-seqlens", default="65536,32768",
                    help="sequence lengths of the NSA varlen workload")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing (profiling runs)")
    args = ap.parse_args()
    if args.headline_only:
        args.prefill = "none"
    args.warmup = max(args.warmup, 3)
    dist = Dist()
    peaks, peak_kind = load_peaks()

    if args.impl == "reference":
        if dist.rank != 0:
            return
        wl = W.make_spec_decode()
        cb = cpu_baseline_decode(wl, steps=args.steps, warmup=args.warmup)
        sec_per_step = decode_bytes(wl)[0] / (cb["value"] * 1e9)
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "GB/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(sec_per_step * 1e3, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": DECODE_WORKLOAD, "global_batch": 8, "seq_len": 32768},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    torch.cuda.set_device(dist.local)
    dist.init(torch)
    import block_sparse_flashattention_sbfa_b200 as sb

    l2 = torch.cuda.get_device_properties(dist.local).L2_cache_size
    # L2 flush: write a buffer of 4x L2, then read another of 4x L2, so that
    # the cache holds clean lines of neither input (a write-only flush leaves
    # L2 full of dirty lines whose write-back would be charged to the next
    # kernel).
    nfl = max(4 * l2, 512 << 20)
    flush_buf = torch.empty(nfl, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones(nfl // 4, dtype=torch.float32, device="cuda")

    def flush():
        flush_buf.fill_(1)
        flush_rd.sum()

    clocks = ClockSampler(dist.local).start()
    dec = bench_decode(torch, sb, dist, args, flush, peaks)
    prefill = {}
    wanted = [] if args.prefill == "none" else args.prefill.split(",")
    for name, fn in (("gated", bench_gated), ("vertical_slash", bench_vs),
                     ("nsa_varlen", bench_nsa), ("block_table", bench_table)):
        if name in wanted:
            try:
                prefill[name] = fn(torch, sb, dist, args, flush, peaks, peak_kind)
            except Exception as e:  # report, keep the headline
                prefill[name] = {"error": f"{type(e).__name__}: {e}"}
    ck = clocks.stop()

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_decode(dec["wl"], steps=5, warmup=1)
    value = whole_job_rate(dec["bytes"], dec["ms"], dist.world) / 1e9
    achieved = dec["bytes"] / (dec["ms"] * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dec["ms"], 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": DECODE_WORKLOAD, "global_batch": 8 * dist.world,
                   "seq_len": 32768, "parallelism": f"replicas x{dist.world}",
                   "l2": "flushed before every step (4x L2 write, then 4x L2 read), outside the timed events"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": ncu_traffic("decode_kernel"), "peak_kind": peak_kind,
                     "kernel": "decode_kernel", "algorithmic_bytes": dec["bytes"]},
        "e2e": dec["e2e"],
        "gpu_launches": args.steps,
        "clocks": ck,
        "prefill": prefill,
    }
    if cpu:
        line["cpu_baseline"] = cpu
    if dist.rank == 0:
        print(json.dumps(line))
    dist.close()


if __name__ == "__main__":
    main()
