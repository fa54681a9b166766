#!/usr/bin/env python
"""Benchmark of the CSA decode step at 1M context on B200.

Workload (default): B=4 sequences of 1,048,576 tokens -> 262,144 compressed
entries each; 64 query heads x 128, one shared KV head, indexer 64 x 128 with
bf16 keys, top-k 1024, window 128; seeded synthetic inputs with one planted
needle per sequence.  A step is one decode step of the whole batch: indexer
scores over every visible entry, per-query top-k, and attention over the
selected entries plus the window (the caches are pre-built, as the workload
states).  The metric is decode queries/s (one query = one sequence's step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch with torchrun; each rank runs its own copy of the batch
(sequences are independent: no collective on the data path), timing is the
max over ranks.  `--impl reference` times the CPU oracle (fp64) instead.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "CSA/HCA decode queries/s at 1M ctx; achieved HBM GB/s as % of B200 peak"
UNIT = "queries/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
NOMINAL_HBM_GBS = 8000.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=500)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-steps", type=int, default=1, help="oracle steps for cpu_baseline")
    p.add_argument("--workload", type=int, default=4, choices=[1, 2, 3, 4, 5, 6, 7, 8],
                   help="4 (default): the 1M CSA decode step; 1, 2, 3, 5: the other "
                        "workloads, one measurement line each (single GPU); 6: workload 4 "
                        "with its indexer keys in MXFP4; 7: workload 4 with QK-norm and "
                        "partial RoPE; 8: workload 4 with FP8 cache entries")
    return p.parse_args()


def load_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu capture
    (profiles/traffic.json), or None when the kernel's sources changed since
    the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    h = hashlib.sha256()
    for src in rec["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    return rec["dram_bytes_per_launch"] if h.hexdigest() == rec["sources_sha256"] else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        pk["source"] = "measured"
        return pk
    return dict(FALLBACK_PEAKS)


# --------------------------------------------------------------------------
# algorithmic bytes (what the method must touch), per query of workload 4
# --------------------------------------------------------------------------
def algorithmic_bytes(s):
    """Bytes per query: the full indexer-key scan, the gathered k entries and
    window rows, and the query-side vectors (q, indexer queries, head
    weights) plus the output."""
    e = 2  # bf16
    keys = s["nc"] * s["dI"] * e
    gather = (s["k"] + s["window"]) * s["d"] * e
    vecs = (s["H"] * s["d"] + s["HI"] * s["dI"] + s["HI"]) * e + s["H"] * s["d"] * e
    return keys, gather, vecs


def scoring_kernel_bytes(s, B):
    """Per launch of the scoring kernel: keys + indexer queries + head
    weights read, fp32 scores written."""
    return B * (s["nc"] * s["dI"] * 2 + s["HI"] * s["dI"] * 2 + s["HI"] * 2 + s["nc"] * 4)


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
def smi_index(uuid, fallback):
    """nvidia-smi's index of the GPU with this UUID (CUDA may renumber)."""
    try:
        out = subprocess.run(["nvidia-smi", "--query-gpu=index,uuid", "--format=csv,noheader"],
                             capture_output=True, text=True, timeout=20).stdout
        for ln in out.splitlines():
            idx, u = [x.strip() for x in ln.split(",")[:2]]
            if uuid.replace("GPU-", "") in u:
                return idx
    except Exception:
        pass
    return str(fallback)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
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
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def max_over_ranks(vals, world, device):
    """Element-wise max of per-rank timings (the slowest rank sets the job's
    time)."""
    if world <= 1:
        return list(vals)
    import torch
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


# --------------------------------------------------------------------------
# the GPU arm
# --------------------------------------------------------------------------
def run_ours(args, rank, world, dev):
    import torch
    import compressed_sparse_long_03_b200 as csa
    from tests.helpers import to_dev

    torch.cuda.set_device(dev)
    wl = W.make(4)
    s = dict(wl.sizes)
    B, nc, k, window = s["B"], s["nc"], s["k"], s["window"]
    D = {n: to_dev(wl[n], f"cuda:{dev}") for n in ("kI", "kv", "win", "q", "qI", "w", "lens")}
    # the step's query-side inputs live in one device buffer (views), so that
    # the end-to-end pass moves them with a single host-to-device copy
    qnames = ("q", "qI", "w")
    pack = torch.empty(sum(D[n].numel() for n in qnames), dtype=torch.bfloat16, device=dev)
    off = 0
    for n in qnames:
        sz = D[n].numel()
        pack[off:off + sz].copy_(D[n].reshape(-1))
        D[n] = pack[off:off + sz].view(D[n].shape)
        off += sz
    idx = torch.empty(B, 1, k, dtype=torch.int32, device=dev)
    out = torch.empty(B, 1, s["H"], s["d"], dtype=torch.bfloat16, device=dev)
    ws = csa.index_topk_workspace(B, 1, nc, False, device=dev)  # the scores
    stream = torch.cuda.current_stream()

    def step():
        csa.csa_index_topk(D["qI"], D["w"], D["kI"], D["lens"], k, idx_out=idx, workspace=ws)
        csa.csa_attend(D["q"], D["kv"], D["win"], idx, D["lens"], window=window, out=out)

    launches_per_step = 3
    for _ in range(args.warmup):
        step()
    csa.check_device_error()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(smi_index(str(torch.cuda.get_device_properties(dev).uuid), dev))
    if rank == 0:
        sampler.start()
    # timed region: K back-to-back steps, events only at its two ends (an
    # event between two kernels would stop the next one from launching early)
    barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    # per-kernel durations: the same K steps again with the library's kernel
    # timing on (events around each kernel; this serialises the kernels)
    stage = {"index_scores": [], "topk": [], "attend": []}
    csa.set_kernel_timing(True)
    for i in range(K):
        csa.csa_index_topk(D["qI"], D["w"], D["kI"], D["lens"], k, idx_out=idx, workspace=ws)
        t_idx = csa.kernel_timing()
        csa.csa_attend(D["q"], D["kv"], D["win"], idx, D["lens"], window=window, out=out)
        t_att = csa.kernel_timing()
        stage["index_scores"].append(t_idx[0])
        stage["topk"].append(t_idx[1])
        stage["attend"].append(t_att[0])
    csa.set_kernel_timing(False)
    torch.cuda.synchronize()
    clocks = sampler.stop() if rank == 0 else None
    csa.check_device_error()
    ms = t0.elapsed_time(t1) / K

    # end to end through the public API from pinned host buffers, as a
    # serving loop runs it: every step copies its query-side inputs (q, q_I,
    # w packed: one H2D copy) in and its output (one D2H copy) out; the
    # inputs and outputs are double-buffered, the copies run on two copy
    # streams, so step i+1's upload and step i's download overlap step i's
    # kernels.  The timed region covers every step's copies.
    host = torch.from_numpy(np.concatenate([np.ascontiguousarray(wl[n]).reshape(-1).view(np.int16)
                                            for n in qnames])).pin_memory()
    packs = [pack, torch.empty_like(pack)]
    views = []
    for pk in packs:
        o, vw = 0, {}
        for n in qnames:
            sz = D[n].numel()
            vw[n] = pk[o:o + sz].view(D[n].shape)
            o += sz
        views.append(vw)
    outs = [out, torch.empty_like(out)]
    outs_h = [torch.empty(out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_ready, pack_free, out_ready, out_free = ([torch.cuda.Event(), torch.cuda.Event()]
                                                for _ in range(4))

    def upload(i):
        j = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(pack_free[j])      # step i-2 no longer reads this pack
            packs[j].view(torch.int16).copy_(host, non_blocking=True)
            in_ready[j].record(up)

    def compute_and_download(i):
        j = i % 2
        stream.wait_event(in_ready[j])
        if i >= 2:
            stream.wait_event(out_free[j])       # step i-2's output has been read out
        vw = views[j]
        csa.csa_index_topk(vw["qI"], vw["w"], D["kI"], D["lens"], k, idx_out=idx, workspace=ws)
        csa.csa_attend(vw["q"], D["kv"], D["win"], idx, D["lens"], window=window, out=outs[j])
        pack_free[j].record(stream)
        out_ready[j].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(out_ready[j])
            outs_h[j].copy_(outs[j], non_blocking=True)
            out_free[j].record(down)

    def run_e2e(n_steps, start):
        up.wait_event(start)  # no copy before the region opens
        upload(0)
        for i in range(n_steps):
            if i + 1 < n_steps:
                upload(i + 1)
            compute_and_download(i)
        stream.wait_event(out_free[(n_steps - 1) % 2])  # the last download is inside the region

    h2d = host.numel() * 2
    d2h = outs_h[0].numel() * 2
    warm = torch.cuda.Event()
    warm.record(stream)
    run_e2e(4, warm)
    torch.cuda.synchronize()
    Ke = max(10, K // 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    run_e2e(Ke, e0)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = e0.elapsed_time(e1) / Ke
    csa.check_device_error()

    ms, ms_e2e = max_over_ranks([ms, ms_e2e], world, f"cuda:{dev}")
    return dict(ms=ms, ms_e2e=ms_e2e, stage=stage, clocks=clocks, s=s, B=B, h2d=h2d, d2h=d2h,
                launches=launches_per_step * K, wl=wl,
                ms_staged=sum(statistics.mean(v) for v in stage.values()))


# --------------------------------------------------------------------------
# the other workloads: one device-timed line each
# --------------------------------------------------------------------------
def other_workload_plan(wid, wl, csa, torch, D):
    """(step stages, unit, units per step, algorithmic bytes, flops, what a
    step is) of workload `wid`; every array already on the device in D."""
    s = wl.sizes
    k, window = s.get("k"), s["window"]
    e = 4 if wl.dt == "f32" else 2
    if wid in (1, 2):
        B, n, d, dI, H, HI, Tq = s["B"], s["n"], s["d"], s["dI"], s["H"], s["HI"], s["Tq"]
        nc = s["nc"]
        C = torch.empty(B, nc, d, dtype=D["x"].dtype, device="cuda")
        KI = torch.empty(B, nc, dI, dtype=D["x"].dtype, device="cuda")
        idx = torch.empty(B, Tq, k, dtype=torch.int32, device="cuda")
        out = torch.empty(B, Tq, H, d, dtype=D["x"].dtype, device="cuda")
        ws = csa.index_topk_workspace(B, Tq, nc, False)
        stages = [
            ("csa_compress (KV)", lambda: csa.csa_compress(D["x"], D["lens"], D["Wa"], D["Wb"], D["beta"], out=C)),
            ("csa_compress (indexer keys)",
             lambda: csa.csa_compress(D["kx"], D["lens"], D["kWa"], D["kWb"], D["kbeta"], out=KI)),
            ("csa_index_topk", lambda: csa.csa_index_topk(D["qI"], D["w"], KI, D["lens"], k, idx_out=idx,
                                                          workspace=ws)),
            ("csa_attend", lambda: csa.csa_attend(D["q"], C, D["x"], idx, D["lens"], window=window, out=out)),
        ]
        t = np.arange(n - Tq, n)
        vis = (t + 1) // 4
        sel = np.minimum(vis, k)
        win = np.minimum(window, t + 1)
        flops = (2.0 * 2 * n * d * 2 * d + 2.0 * 2 * n * dI * 2 * dI      # compressors (logits, both series)
                 + 2.0 * float(vis.sum()) * HI * dI                       # indexer
                 + 4.0 * float((sel + win).sum()) * H * d)                # QK^T and PV
        byts = e * (B * n * (d + dI) + B * nc * (d + dI)                  # tokens read, caches written
                    + float(vis.sum()) * dI                               # indexer keys per query
                    + float((sel + win).sum()) * d                        # gathered rows
                    + Tq * (2 * H * d + HI * dI + HI))                    # q, q_I, w, out
        unit = "tokens/s" if wid == 2 else "queries/s"
        what = ("one prefill pass of the 8192-token sequence: both compressors, indexer + top-k "
                "and attention for every token" if wid == 2 else
                "one decode step with the caches rebuilt from the 1024 tokens: both compressors, "
                "indexer + top-k, attention")
        return stages, unit, B * Tq, byts, flops, what
    if wid == 3:
        B, H, d, m = s["B"], s["H"], s["d"], s["m"]
        out = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device="cuda")
        stages = [("hca_attend", lambda: csa.hca_attend(D["q"], D["hkv"], D["win"], D["lens"], m=m,
                                                        window=window, out=out))]
        v = s["n"] // m
        byts = B * ((v + window) * d * 2 + 2 * H * d * 2)
        flops = 4.0 * B * (v + window) * H * d
        return stages, "queries/s", B, byts, flops, "one HCA decode step of the 32 sequences"
    if wid == 6:
        B, nc, H, d, dI, HI = s["B"], s["nc"], s["H"], s["d"], s["dI"], s["HI"]
        codes, scales = csa.csa_quantize_mxfp4(D["kI"])
        torch.cuda.synchronize()
        idx = torch.empty(B, 1, k, dtype=torch.int32, device="cuda")
        out = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device="cuda")
        ws = csa.index_topk_workspace(B, 1, nc, False)
        stages = [
            ("csa_index_topk_mxfp4", lambda: csa.csa_index_topk_mxfp4(D["qI"], D["w"], codes, scales, D["lens"],
                                                                      k, idx_out=idx, workspace=ws)),
            ("csa_attend", lambda: csa.csa_attend(D["q"], D["kv"], D["win"], idx, D["lens"], window=window,
                                                  out=out)),
        ]
        byts = B * (nc * (dI // 2 + dI // 32) + (k + window) * d * 2 + (2 * H * d + HI * dI + HI) * 2)
        flops = B * (2.0 * nc * HI * dI + 4.0 * (k + window) * H * d)
        return stages, "queries/s", B, byts, flops, ("one decode step of the 1M workload with the indexer "
                                                      "keys in MXFP4 (68 B per key): indexer + top-k, attention")
    if wid == 7:
        B, nc, H, d, dI, HI = s["B"], s["nc"], s["H"], s["d"], s["dI"], s["HI"]
        n_tok = D["win"].shape[1]
        # the caches as the decode step keeps them: entries normalised and
        # rotated when formed (entry i at 4 i), window tokens at their positions
        D["q_gamma"] = to_dev_like(torch, W.normal(W.seed_of(4), "q_gamma", (d,), 1.0, "bf16"))
        D["kv_gamma"] = to_dev_like(torch, W.normal(W.seed_of(4), "kv_gamma", (d,), 1.0, "bf16"))
        D["kv_r"] = torch.empty_like(D["kv"])
        csa.csa_norm_rope(D["kv"].view(B, nc, 1, d), D["kv_r"].view(B, nc, 1, d), gamma=D["kv_gamma"], Tq=nc,
                          pos_stride=4, flags=3)
        lens = wl["lens"].astype(np.int64)
        j = np.arange(n_tok)[None, :]
        ring_pos = np.where(lens[:, None] - 1 >= j, j + n_tok * ((lens[:, None] - 1 - j) // n_tok), 0)
        D["win_r"] = csa.csa_norm_rope(D["win"].view(B, n_tok, 1, d), gamma=D["kv_gamma"],
                                       pos=to_dev_i32(torch, ring_pos.astype(np.int32)),
                                       flags=3).view(B, n_tok, d)
        torch.cuda.synchronize()
        idx = torch.empty(B, 1, k, dtype=torch.int32, device="cuda")
        out = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device="cuda")
        ws = csa.index_topk_workspace(B, 1, nc, False)
        stages = [
            ("csa_index_topk", lambda: csa.csa_index_topk(D["qI"], D["w"], D["kI"], D["lens"], k,
                                                          idx_out=idx, workspace=ws)),
            ("csa_attend_rope", lambda: csa.csa_attend_rope(D["q"], D["kv_r"], D["win_r"], idx, D["lens"],
                                                            window=window, out=out, q_gamma=D["q_gamma"])),
        ]
        byts = B * (nc * dI * 2 + (k + window) * d * 2 + (2 * H * d + HI * dI + HI) * 2) + d * 2
        flops = B * (2.0 * nc * HI * dI + 4.0 * (k + window) * H * d)
        return stages, "queries/s", B, byts, flops, ("one decode step of the 1M workload with QK-norm and "
                                                      "partial RoPE: indexer + top-k, attention with the "
                                                      "query's norm / rotation and the output's inverse "
                                                      "rotation fused in")
    if wid == 8:
        B, nc, H, d, dI, HI = s["B"], s["nc"], s["H"], s["d"], s["dI"], s["HI"]
        # the entry cache as the decode step keeps it: FP8 codes, scales, bf16 RoPE dims
        D["kv_fp8"], D["kv_sc"], D["kv_rope"] = csa.csa_quantize_fp8_entries(D["kv"])
        D["kv_sc"] = D["kv_sc"].view(B, nc)
        torch.cuda.synchronize()
        idx = torch.empty(B, 1, k, dtype=torch.int32, device="cuda")
        out = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device="cuda")
        ws = csa.index_topk_workspace(B, 1, nc, False)
        stages = [
            ("csa_index_topk", lambda: csa.csa_index_topk(D["qI"], D["w"], D["kI"], D["lens"], k,
                                                          idx_out=idx, workspace=ws)),
            ("csa_attend_fp8", lambda: csa.csa_attend_fp8(D["q"], D["kv_fp8"], D["kv_sc"], D["kv_rope"], D["win"],
                                                          idx, D["lens"], window=window, out=out)),
        ]
        byts = B * (nc * dI * 2 + k * (64 + 1 + 128) + window * d * 2 + (2 * H * d + HI * dI + HI) * 2)
        flops = B * (2.0 * nc * HI * dI + 4.0 * (k + window) * H * d)
        return stages, "queries/s", B, byts, flops, ("one decode step of the 1M workload with FP8 cache entries "
                                                      "(64 E4M3 dims + scale + 64 bf16 RoPE dims): indexer + "
                                                      "top-k, attention widening the selected entries on chip")
    if wid == 5:
        B, H, d, dI, HI, m = s["B"], s["H"], s["d"], s["dI"], s["HI"], s["m"]
        nc = s["nc"]
        idx = torch.empty(B, 1, k, dtype=torch.int32, device="cuda")
        out_c = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device="cuda")
        out_h = torch.empty(B, 1, H, d, dtype=torch.bfloat16, device="cuda")
        ws = csa.index_topk_workspace(B, 1, nc, False)
        # the layer-pair scheduler: one call, the HCA attention beside the CSA layer
        stages = [
            ("csa_hca_pair_decode", lambda: csa.csa_hca_pair_decode(
                D["q"], D["qI"], D["w"], D["kI"], D["kv"], D["q2"], D["hkv"], D["win"], D["lens"], k, m=m,
                window=window, idx_out=idx, out_csa=out_c, out_hca=out_h, workspace=ws)),
        ]
        # the same step as three calls on one stream, timed beside it
        D["serial_step"] = [
            lambda: csa.csa_index_topk(D["qI"], D["w"], D["kI"], D["lens"], k, idx_out=idx, workspace=ws),
            lambda: csa.csa_attend(D["q"], D["kv"], D["win"], idx, D["lens"], window=window, out=out_c),
            lambda: csa.hca_attend(D["q2"], D["hkv"], D["win"], D["lens"], m=m, window=window, out=out_h),
        ]
        lens = wl["lens"].astype(np.int64)
        vis, hv = lens // 4, lens // m
        sel = np.minimum(vis, k)
        byts = 2 * float((vis * dI + (sel + window) * d + (hv + window) * d).sum()
                         + B * (4 * H * d + HI * dI + HI))
        flops = float((2.0 * vis * HI * dI + 4.0 * (sel + window) * H * d + 4.0 * (hv + window) * H * d).sum())
        return stages, "queries/s", B, byts, flops, "one decode step of the CSA + HCA layer pair"
    raise KeyError(wid)


def run_other_workload(args):
    """Device time of one step of workload 1, 2, 3 or 5 (inputs resident in
    HBM; the L2 is flushed by a 256 MiB write before every timed step, and
    CUDA events bracket the step alone)."""
    import torch
    import compressed_sparse_long_03_b200 as csa
    from tests.helpers import to_dev
    torch.cuda.set_device(0)
    wid = args.workload
    wl = W.make(4 if wid in (6, 7, 8) else wid)
    D = {n: to_dev(wl[n]) for n in wl.arrays if n != "needle_pos"}
    stages, unit, units, byts, flops, what = other_workload_plan(wid, wl, csa, torch, D)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def step():
        for _, fn in stages:
            fn()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    csa.check_device_error()
    # the step is replayed from a CUDA graph, so that the GPU time of a step
    # of small kernels is not the host's time to issue them
    run, how = step, "issued eagerly"
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph.replay()
        torch.cuda.synchronize()
        csa.check_device_error()
        run, how = graph.replay, "replayed from a CUDA graph"
    except Exception as e:  # capture unsupported here: time the eager calls
        how = f"issued eagerly (graph capture failed: {type(e).__name__})"
        torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(smi_index(str(torch.cuda.get_device_properties(0).uuid), 0))
    sampler.start()
    for i in range(K):
        flush.zero_()
        ev[i][0].record()
        run()
        ev[i][1].record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    per = {name: [] for name, _ in stages}
    csa.set_kernel_timing(True)
    for i in range(K):
        flush.zero_()
        for name, fn in stages:
            fn()
            per[name].append(sum(csa.kernel_timing()))
    csa.set_kernel_timing(False)
    torch.cuda.synchronize()
    csa.check_device_error()
    peaks = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tfl = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    gbs = byts / (ms * 1e-3) / 1e9
    tfs = flops / (ms * 1e-3) / 1e12
    name = {6: "csa_decode_mxfp4keys_b4_n1048576", 7: "csa_decode_qknorm_rope_b4_n1048576",
            8: "csa_decode_fp8entries_b4_n1048576"}.get(wid, wl.name)
    line = {"metric": f"{name}: {unit}", "value": units * 1000.0 / ms, "unit": unit, "n_gpus": 1,
            "steps": K, "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
            "dtype": wl.dt, "data": "synthetic (seeded PCG64)",
            "config": {"workload": name, "step": what, "issue": how,
                       "l2": "flushed before every timed step (256 MiB write); events bracket the step"},
            "algorithmic": {"bytes_per_step": byts, "flops_per_step": flops, "achieved_gbs": gbs,
                            "frac_of_measured_hbm": gbs / hbm, "achieved_tflops": tfs,
                            "frac_of_measured_bf16": tfs / tfl, "peak_source": peaks["source"]},
            "stages_us": {k2: 1000 * statistics.median(v) for k2, v in per.items()},
            "stages_note": "per-call medians with the library's kernel timing on (serialised)",
            "clocks": clocks}
    if wid == 3:
        line["hca_compress"] = time_hca_compress(wl, csa, torch, flush, min(K, 20), hbm)
    if wid == 5:
        line["compress_step"] = time_compress_step(wl, csa, torch, D, flush, min(K, 20))
        ser = time_step_graph(D["serial_step"], K, flush, torch, csa)
        line["serial_three_calls"] = {"ms_per_step": ser, "value": units * 1000.0 / ser,
                                      "note": "csa_index_topk, csa_attend, hca_attend on one stream, "
                                              "timed the same way"}
    if wid == 7:
        line["norm_rope_cache"] = time_norm_rope_cache(wl, csa, torch, D, min(K, 50), hbm)
    if wid == 8:
        line["quantize_fp8_cache"] = time_quantize_fp8_cache(wl, csa, torch, D, min(K, 50), hbm)
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(wid, wl)
    print(json.dumps(line))
    return 0


def oracle_sample(wid, wl):
    """The oracle (fp64 C, all host cores) on a bounded sample of the same
    workload, in the line's unit."""
    import oracle
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    s = wl.sizes
    k, window = s.get("k"), s["window"]

    def clock(fn):
        t = time.perf_counter()
        fn()
        return time.perf_counter() - t

    if wid in (1, 2):
        rows = 1 if wid == 1 else 64
        tc = clock(lambda: (oracle.csa_compress(wl["x"], wl["lens"], wl["Wa"], wl["Wb"], wl["beta"]),
                            oracle.csa_compress(wl["kx"], wl["lens"], wl["kWa"], wl["kWb"], wl["kbeta"])))
        C = oracle.round_to(oracle.csa_compress(wl["x"], wl["lens"], wl["Wa"], wl["Wb"], wl["beta"]),
                            oracle.F32 if wl.dt == "f32" else oracle.BF16)
        KI = oracle.round_to(oracle.csa_compress(wl["kx"], wl["lens"], wl["kWa"], wl["kWb"], wl["kbeta"]),
                             oracle.F32 if wl.dt == "f32" else oracle.BF16)
        n, Tq = s["n"], s["Tq"]
        pos = np.linspace(n - Tq, n - 1, rows).astype(np.int32)[None, :]
        sub = lambda a: a[:, pos[0] - (n - Tq)]

        def rows_fn():
            idx, _ = oracle.index_topk(sub(wl["qI"]), sub(wl["w"]), KI, wl["lens"], k, pos)
            oracle.attend(sub(wl["q"]), C, wl["x"], wl["lens"], idx=idx, q_pos=pos, window=window)
        tr = clock(rows_fn)
        if wid == 1:
            return {"value": 1.0 / (tc + tr), "unit": "queries/s", "cores": cores, "kind": "oracle",
                    "sample": "one full decode step (both compressors, indexer + top-k, attention)"}
        return {"value": Tq / (tc + tr * Tq / rows), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                "sample": f"both compressors over the {n} tokens, then indexer + top-k + attention for "
                          f"{rows} of the {Tq} query rows (spread over the sequence), scaled to all rows"}
    if wid == 6:
        sl = slice(0, 1)

        def one():
            c, sc = oracle.quantize_mxfp4(wl["kI"][sl])
            kdq = W.bf16_bits(oracle.dequant_mxfp4(c, sc).astype(np.float32))
            idx, _ = oracle.index_topk(wl["qI"][sl], wl["w"][sl], kdq, wl["lens"][sl], k)
            oracle.attend(wl["q"][sl], wl["kv"][sl], wl["win"][sl], wl["lens"][sl], idx=idx, window=window)
        t = clock(one)
        return {"value": 1.0 / t, "unit": "queries/s", "cores": cores, "kind": "oracle",
                "sample": "one query of the batch (its keys quantised, dequantised, scored; attention)"}
    if wid == 8:
        sl = slice(0, 1)
        # the cache as the step finds it (quantised when the entries are formed)
        f8, sc8, rp8 = oracle.quantize_fp8_entries(wl["kv"][sl])
        deq = oracle.round_to(oracle.dequant_fp8_entries(f8, sc8, rp8), oracle.BF16)

        def one():
            idx, _ = oracle.index_topk(wl["qI"][sl], wl["w"][sl], wl["kI"][sl], wl["lens"][sl], k)
            oracle.attend(wl["q"][sl], deq, wl["win"][sl], wl["lens"][sl], idx=idx, window=window)
        t = clock(one)
        return {"value": 1.0 / t, "unit": "queries/s", "cores": cores, "kind": "oracle",
                "sample": "one query of the batch (indexer + top-k, attention over the dequantised FP8 entries)"}
    if wid == 7:
        sl = slice(0, 1)
        d, nc = s["d"], s["nc"]
        gq = W.normal(W.seed_of(4), "q_gamma", (d,), 1.0, "bf16")
        gk = W.normal(W.seed_of(4), "kv_gamma", (d,), 1.0, "bf16")
        lens = wl["lens"][sl].astype(np.int64)
        n_tok = wl["win"].shape[1]

        # the caches as the step finds them (normalised and rotated when formed)
        kv_r = oracle.round_to(oracle.norm_rope(wl["kv"][sl][:, :, None, :], 4 * np.arange(nc)[None, :],
                                                gamma=gk)[:, :, 0, :], oracle.BF16)
        j = np.arange(n_tok)[None, :]
        rp = np.where(lens[:, None] - 1 >= j, j + n_tok * ((lens[:, None] - 1 - j) // n_tok), 0)
        win_r = oracle.round_to(oracle.norm_rope(wl["win"][sl][:, :, None, :], rp, gamma=gk)[:, :, 0, :],
                                oracle.BF16)

        def one():
            t = (lens - 1)[:, None]
            idx, _ = oracle.index_topk(wl["qI"][sl], wl["w"][sl], wl["kI"][sl], wl["lens"][sl], k)
            q_r = oracle.round_to(oracle.norm_rope(wl["q"][sl], t, gamma=gq), oracle.BF16)
            o = oracle.attend(q_r, kv_r, win_r, wl["lens"][sl], idx=idx, window=window)
            oracle.norm_rope(o.astype(np.float32), t, norm=False, inverse=True)
        t = clock(one)
        return {"value": 1.0 / t, "unit": "queries/s", "cores": cores, "kind": "oracle",
                "sample": "one query of the batch (indexer + top-k, the query normalised and rotated, "
                          "attention, the output turned back)"}
    if wid == 3:
        nq = 4
        sl = slice(0, nq)
        t = clock(lambda: oracle.attend(wl["q"][sl], wl["hkv"][sl], wl["win"][sl], wl["lens"][sl], idx=None,
                                        m=s["m"], window=window))
        return {"value": nq / t, "unit": "queries/s", "cores": cores, "kind": "oracle",
                "sample": f"HCA attention for {nq} of the {s['B']} sequences"}
    if wid == 5:
        nq = 2
        sl = slice(0, nq)

        def pair():
            idx, _ = oracle.index_topk(wl["qI"][sl], wl["w"][sl], wl["kI"][sl], wl["lens"][sl], k)
            oracle.attend(wl["q"][sl], wl["kv"][sl], wl["win"][sl], wl["lens"][sl], idx=idx, window=window)
            oracle.attend(wl["q2"][sl], wl["hkv"][sl], wl["win"][sl], wl["lens"][sl], idx=None, m=s["m"],
                          window=window)
        t = clock(pair)
        return {"value": nq / t, "unit": "queries/s", "cores": cores, "kind": "oracle",
                "sample": f"the CSA + HCA step for {nq} of the {s['B']} sequences"}
    raise KeyError(wid)


def time_step_graph(fns, K, flush, torch, csa):
    """Median device time (ms) of the calls `fns` replayed from a CUDA graph,
    the L2 flushed before every step (as the workload lines are timed)."""
    def step():
        for fn in fns:
            fn()
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    run = step
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        g.replay()
        torch.cuda.synchronize()
        run = g.replay
    except Exception:
        torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:
        flush.zero_()
        a.record()
        run()
        b.record()
    torch.cuda.synchronize()
    csa.check_device_error()
    return statistics.median(a.elapsed_time(b) for a, b in ev)


def time_compress_step(wl, csa, torch, D, flush, K):
    """The decode-time compressors of the layer pair in their most expensive
    step: every sequence's newest token completes both a CSA block (both
    caches get an entry) and an HCA block (lengths rounded down to a
    multiple of 128); tokens from the 128-token window ring."""
    s = wl.sizes
    B, d, dI, m = s["B"], s["d"], s["dI"], s["m"]
    lens = to_dev_i32(torch, (wl["lens"] // m) * m)
    g = lambda role, shape: torch.from_numpy(W.normal(9, role, shape, d ** -0.5, "bf16").view(np.int16)) \
        .cuda().view(torch.bfloat16)
    Wa, Wb, b8 = g("Wa", (d, d)), g("Wb", (d, d)), g("beta", (8, d))
    kWa, kWb, kb8 = g("kWa", (dI, dI)), g("kWb", (dI, dI)), g("kbeta", (8, dI))
    hW, hb = g("hca_W", (d, d)), g("hca_beta", (m, d))
    ring = D["win"]
    kv = torch.empty(B, s["nc"], d, dtype=torch.bfloat16, device="cuda")
    kI = torch.empty(B, s["nc"], dI, dtype=torch.bfloat16, device="cuda")
    hkv = torch.empty(B, s["hnc"], d, dtype=torch.bfloat16, device="cuda")

    def step():
        csa.csa_compress_step(ring, lens, Wa, Wb, b8, kv)
        csa.csa_compress_step(ring, lens, kWa, kWb, kb8, kI)
        csa.hca_compress_step(ring, lens, hW, hb, hkv, m=m)

    for _ in range(3):
        step()
    # device time of the three kernels (the library's per-launch events): the
    # host needs longer to issue three small calls than the GPU to run them
    per = []
    csa.set_kernel_timing(True)
    for i in range(K):
        flush.zero_()
        tot = 0.0
        for fn in (lambda: csa.csa_compress_step(ring, lens, Wa, Wb, b8, kv),
                   lambda: csa.csa_compress_step(ring, lens, kWa, kWb, kb8, kI),
                   lambda: csa.hca_compress_step(ring, lens, hW, hb, hkv, m=m)):
            fn()
            tot += sum(csa.kernel_timing())
        per.append(tot)
    csa.set_kernel_timing(False)
    torch.cuda.synchronize()
    csa.check_device_error()
    return {"us": 1000 * statistics.median(per), "sequences": B,
            "calls": "csa_compress_step (KV) + csa_compress_step (indexer keys) + hca_compress_step",
            "timing": "sum of the three kernels' device times",
            "note": "every sequence completes a CSA and an HCA block in this step"}


def to_dev_like(torch, a):
    """numpy float32 / bf16 bits (uint16) -> CUDA tensor."""
    from tests.helpers import to_dev
    return to_dev(a)


def time_norm_rope_cache(wl, csa, torch, D, K, hbm):
    """csa_norm_rope over the whole 1M-token entry cache (B x 262,144 entries
    of 256 B: read once, written once; 512 MiB per launch, larger than L2)."""
    s = wl.sizes
    B, nc, d = s["B"], s["nc"], s["d"]
    src, dst = D["kv"].view(B, nc, 1, d), D["kv_r"].view(B, nc, 1, d)
    for _ in range(3):
        csa.csa_norm_rope(src, dst, gamma=D["kv_gamma"], Tq=nc, pos_stride=4, flags=3)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:
        a.record()
        csa.csa_norm_rope(src, dst, gamma=D["kv_gamma"], Tq=nc, pos_stride=4, flags=3)
        b.record()
    torch.cuda.synchronize()
    csa.check_device_error()
    us = 1000 * statistics.median(a.elapsed_time(b) for a, b in ev)
    byts = 2 * B * nc * d * 2
    gbs = byts / (us * 1e-6) / 1e9
    return {"kernel": "k_norm_rope<bf16,128>", "rows": B * nc, "us": us, "bytes_per_launch": byts,
            "achieved_gbs": gbs, "frac_of_measured_hbm": gbs / hbm, "bound": "hbm"}


def time_quantize_fp8_cache(wl, csa, torch, D, K, hbm):
    """csa_quantize_fp8_entries over the whole 1M-token entry cache (B x
    262,144 entries: 256 B read, 64 + 1 + 128 B written per entry)."""
    s = wl.sizes
    B, nc, d = s["B"], s["nc"], s["d"]
    for _ in range(3):
        csa.csa_quantize_fp8_entries(D["kv"])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:
        a.record()
        csa.csa_quantize_fp8_entries(D["kv"])
        b.record()
    torch.cuda.synchronize()
    csa.check_device_error()
    us = 1000 * statistics.median(a.elapsed_time(b) for a, b in ev)
    byts = B * nc * (d * 2 + 64 + 1 + 128)
    gbs = byts / (us * 1e-6) / 1e9
    return {"kernel": "k_quantize_fp8_entries<bf16>", "rows": B * nc, "us": us, "bytes_per_launch": byts,
            "achieved_gbs": gbs, "frac_of_measured_hbm": gbs / hbm, "bound": "hbm"}


def to_dev_i32(torch, a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def time_hca_compress(wl, csa, torch, flush, K, hbm):
    """The HCA compressor over the workload's 131,072 tokens per sequence
    (all 32 sequences), timed like the step."""
    from tests.helpers import to_dev
    s = wl.sizes
    tk = W.hca_tokens(wl.sizes["seed"], s["B"], s["n"], s["d"], wl.dt, m=s["m"])
    x, Wm, beta, lens = (to_dev(tk[n]) for n in ("x", "W", "beta", "lens"))
    out = torch.empty(s["B"], tk.sizes["nc"], s["d"], dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        csa.hca_compress(x, lens, Wm, beta, m=s["m"], out=out)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        flush.zero_()
        ev[i][0].record()
        csa.hca_compress(x, lens, Wm, beta, m=s["m"], out=out)
        ev[i][1].record()
    torch.cuda.synchronize()
    csa.check_device_error()
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    byts = 2 * (x.numel() + out.numel())
    return {"us": 1000 * ms, "tokens": int(s["B"] * s["n"]), "bytes": byts,
            "achieved_gbs": byts / (ms * 1e-3) / 1e9, "frac_of_measured_hbm": byts / (ms * 1e-3) / 1e9 / hbm}


# --------------------------------------------------------------------------
# the oracle (CPU) arm
# --------------------------------------------------------------------------
def oracle_query_step(wl, b):
    import oracle
    s = wl.sizes
    sl = slice(b, b + 1)
    idx, _ = oracle.index_topk(wl["qI"][sl], wl["w"][sl], wl["kI"][sl], wl["lens"][sl], s["k"])
    oracle.attend(wl["q"][sl], wl["kv"][sl], wl["win"][sl], wl["lens"][sl], idx=idx,
                  window=s["window"])


def cpu_baseline(wl, steps=1):
    """The oracle as it stands on the host cores: `steps` full decode steps
    of the batch (every query scores all 262,144 entries in fp64)."""
    import oracle
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    B = wl.sizes["B"]
    t = time.perf_counter()
    for _ in range(steps):
        for b in range(B):
            oracle_query_step(wl, b)
    dt = time.perf_counter() - t
    return {"value": steps * B / dt, "unit": UNIT, "cores": oracle.get_threads(), "kind": "oracle",
            "sample": f"{steps} full decode step(s) of the B={B} batch ({steps * B} queries, "
                      f"fp64 C oracle, OpenMP)"}


def config_block(s, world):
    return {"workload": "csa_decode_bf16_b4_n1048576", "B": s["B"], "context": s["n"],
            "entries": s["nc"], "H": s["H"], "d": s["d"], "HI": s["HI"], "dI": s["dI"],
            "k": s["k"], "window": s["window"],
            "l2": "inputs larger than L2: the 256 MiB indexer-key cache is re-scanned every step",
            "parallelism": f"{world} independent replica(s), one per GPU"}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)

    if args.workload != 4 and args.impl == "ours":
        return run_other_workload(args) if rank == 0 else 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        wl = W.make(4)
        import oracle
        oracle.set_threads(os.cpu_count() or 1)
        B = wl.sizes["B"]
        for i in range(args.warmup):
            oracle_query_step(wl, i % B)
        t = time.perf_counter()
        for i in range(args.steps):
            oracle_query_step(wl, i % B)
        dt = time.perf_counter() - t
        value = args.steps / dt
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": config_block(wl.sizes, 1),
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.get_threads(),
                                 "kind": "oracle",
                                 "sample": "one query (one sequence's decode step) per step, "
                                           "rotating over the batch"},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    if world > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device(f"cuda:{local}"))
    r = run_ours(args, rank, world, local)
    s, B = r["s"], r["B"]
    peaks = load_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    keys, gather, vecs = algorithmic_bytes(s)
    step_bytes = B * (keys + gather + vecs)
    value = world * B * 1000.0 / r["ms"]
    e2e = world * B * 1000.0 / r["ms_e2e"]
    sc_us = [1000 * x for x in r["stage"]["index_scores"]]
    sc_avg_s = statistics.mean(sc_us) * 1e-6
    kb = scoring_kernel_bytes(s, B)
    achieved = kb / sc_avg_s / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded PCG64, planted needles)",
        "config": config_block(s, world),
        "hbm": {"algorithmic_bytes_per_step": step_bytes,
                "achieved_gbs": step_bytes / (r["ms"] * 1e-3) / 1e9,
                "frac_of_measured": step_bytes / (r["ms"] * 1e-3) / 1e9 / hbm_peak,
                "frac_of_nominal_8tbs": step_bytes / (r["ms"] * 1e-3) / 1e9 / NOMINAL_HBM_GBS},
        "roofline": {"kernel": "index_scores", "bound": "hbm", "achieved": achieved,
                     "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                     "traffic": load_traffic("index_scores"), "bytes_per_launch": kb,
                     "peak_source": peaks["source"]},
        "stages_us": {k: statistics.median(1000 * x for x in v) for k, v in r["stage"].items()},
        "stages_note": "per-kernel medians from a second pass of the K steps with the "
                       "library's kernel timing on (serialised); ms_per_step is the event-free pass",
        "e2e": {"value": e2e, "unit": UNIT, "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(r["wl"], args.cpu_steps)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
