"""Benchmark of the VGGT attention path on B200.

Default workload: dense global attention over 9 frames of 1024x1024 at patch
16 (64x64 patches + 5 special tokens = 4101 tokens/frame, 36 909 tokens,
16 heads x 64 dims). One step = one ``vggt_attn_global`` call through the C
ABI (QK LayerNorm + 2D RoPE prologue, then the tcgen05 attention kernel) on
inputs already resident in HBM. ``value`` = algorithmic attention FLOPs
(4*H*D per query-key pair) / device time, summed over all ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on host cores

Multi-GPU (``torchrun``): every rank runs an independent replica of the
workload (the path has no data exchange); the job's time is the max over
ranks. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "global-attention fwd TFLOP/s and tokens/s on 1 B200; % of dense bf16 peak"
DEFAULT_WORKLOAD = "global_s9_g64"
L2_BYTES = 126 * 1024 * 1024
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures, reported beside the measured ones for context: dense
# bf16 tensor throughput (the sparse figure halved) and HBM3e bandwidth.
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 8000.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attn_fwd_kernel_global_s6_g64.txt")
KERNEL_SOURCES = ("feed_forward_view_b200/csrc/attn_fwd.cu", "feed_forward_view_b200/csrc/attn_common.cuh",
                  "feed_forward_view_b200/csrc/sm100.cuh", "feed_forward_view_b200/csrc/pdl.cuh")


# ----------------------------------------------------------------------------- helpers


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(w):
    """DRAM bytes per attention launch for workload ``w``, from the committed
    ncu summary of a smaller dense-global case scaled by the token count
    (every byte the kernel moves -- q_hat, k_hat, v in, out -- grows linearly
    with the tokens while one head's keys fit in L2), or None when the summary
    is missing, covers another kind, or was taken on different kernel source."""
    if not os.path.exists(PROFILE_SUMMARY) or w.kind != "global":
        return None
    fields = {}
    for line in open(PROFILE_SUMMARY):
        if ":" in line and not line.startswith("#"):
            k, _, v = line.partition(":")
            fields[k.strip()] = v.strip().split()[0] if v.strip() else ""
    if fields.get("source_sha256_16") != kernel_source_hash():
        return None
    try:
        return float(fields["dram_bytes_per_launch"]) * w.n_q / float(fields["tokens"])
    except (KeyError, ValueError, ZeroDivisionError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, cmax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            sm.append(clk)
            mx = cmax
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        loaded = [c for c in sm if c > 0.5 * max(sm)]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if n_gpus > 0 else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, local, world


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar across ranks (identity at world size 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist

        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- CPU oracle leg


class OracleLeg:
    """The fp64 oracle, as it stands, on a sample of query rows of workload
    ``w``. Setup (widening the inputs, the keys' prologue and pooling: a fixed
    O(N_k) cost that a full run amortises) happens once, untimed; ``run``
    times ``n_rows`` query rows against all keys, all heads."""

    def __init__(self, w, seed: int = 0):
        import numpy as np
        import torch

        import synth
        from oracle import vggt_oracle as O

        self.w, self.O, self.synth = w, O, synth
        q, k, v, pos = synth.make_workload(w, seed)

        def f64(t):
            if t.dtype == torch.float32:  # the fp32 mode's inputs
                return t.double().numpy()
            return O.bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy().view(np.uint16)).reshape(t.shape)

        self.q, self.k, self.v, self.pos = f64(q), f64(k), f64(v), pos.numpy().astype(np.float64)
        if w.kind == "descriptor":
            kp, vp, pp = O.kv_pool(self.k, self.v, self.pos, w.S, w.T, w.kv_down)
            self.k_hat, self.vv = O.qk_prologue(kp, pp), vp
        elif w.kind in ("global", "global_f32"):
            ln = synth.workload_affine(w)
            self.ln = None if ln is None else tuple(x.double().numpy() for x in ln)
            kw, kb = (None, None) if self.ln is None else self.ln[2:]
            self.k_hat, self.vv = O.qk_prologue(self.k, self.pos, kw, kb), self.v

    def run(self, n_rows: int, seed: int = 0):
        """Returns (TFLOP/s, seconds, rows)."""
        import numpy

        w, O = self.w, self.O
        rows = self.synth.sample_rows(w.n_q, n_rows, seed).numpy()
        t0 = time.perf_counter()
        if w.kind in ("frame", "frame_f32"):
            O.attn_frame(self.q, self.k, self.v, self.pos, w.S, w.T, rows=rows)
            keys = w.T
        elif w.kind == "stream":
            O.attn_descriptor_stream(self.q, self.k, self.v, self.pos, w.S, w.T, w.kv_down, w.chunk, rows=rows)
            chunk_of = rows // (w.T * w.chunk)
            keys = float((numpy.minimum(w.S, (chunk_of + 1) * w.chunk) * w.T_k).mean())
        elif w.kind == "global_batch":
            O.attn_scenes("global", self.q, self.k, self.v, self.pos, w.B, w.S, w.T, rows=rows)
            keys = w.n_k
        elif w.kind.startswith("subset"):
            kind = w.kind[len("subset_"):]
            kept = O.subset_rows(w.S, w.T, w.skip, w.n_extra if kind == "global" else 0)
            O.attn_subset(self.q, self.k, self.v, self.pos, w.S, w.T, w.skip, w.n_extra, kind, rows=kept[rows])
            keys = w.n_k if kind == "global" else w.T_k
        else:
            qw, qb = (None, None) if getattr(self, "ln", None) is None else self.ln[:2]
            O.cross_attention(O.qk_prologue(self.q[rows], self.pos[rows], qw, qb), self.k_hat, self.vv)
            keys = w.n_k
        dt = time.perf_counter() - t0
        return 4.0 * w.H * w.D * rows.size * keys / dt / 1e12, dt, int(rows.size)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args):
    """--impl reference: the oracle on the host cores, bounded sample per step."""
    import synth

    rank, _, world = int(os.environ.get("RANK", "0")), 0, int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    w = synth.ALL_WORKLOADS[args.workload]
    leg = OracleLeg(w)
    # size each step from a short calibration so the whole run stays bounded
    _, dt, rows = leg.run(32)
    per_row = dt / rows
    budget = args.reference_budget_s / max(1, args.steps + args.warmup)
    n_rows = int(min(4096, max(8, budget / per_row)))
    for i in range(args.warmup):
        leg.run(n_rows, seed=i)
    vals, times = [], []
    for i in range(args.steps):
        tf, dt, rows = leg.run(n_rows, seed=100 + i)
        vals.append(tf)
        times.append(dt)
    threads = blas_threads()
    value = statistics.median(vals)
    keys_desc = ({"frame": f"all {w.T}", "frame_f32": f"all {w.T}", "subset_frame": f"all {w.T_k}",
                  "stream": "the cached-prefix"}.get(w.kind, f"all {w.n_k}"))
    sample = (f"{rows} query rows x {keys_desc} keys x {w.H} heads per step "
              f"(of {w.n_q} rows)" + ("; pooling and key prologue redone each step" if w.kind == "stream"
                                       else ", key prologue precomputed"))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "kind": w.kind, "S": w.S, "T": w.T, "tokens": w.n_q,
                   "keys": w.T if w.kind == "frame" else (w.T_k if w.kind == "subset_frame" else w.n_k), "H": w.H, "D": w.D,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm


# Every other workload of the pages' shapes, measured after the headline one
# on the same GPU (N = 1 only) and reported under "secondary": configurations
# 1, 2, 3 and 5, the streamed descriptors, the VGGT-Omega token layout, the
# fp32 mode and a large QK LayerNorm affine (precise mode).
SECONDARY = ("global_s2_g16", "frame_s8_g37", "global_s8_g37", "descriptor_s200_g37_kd4",
             "stream_s200_g37_kd4_c10", "omega_global_s32_g32", "omega_frame_s32_g32",
             "global_s9_g64_f32", "global_s9_g64_affine8")


def _event_ms(torch, stream, fn, reps: int, warm: int = 3) -> float:
    """Average device time of fn() over reps back-to-back launches. The reps
    calls are captured once into a CUDA graph and one replay is timed with
    CUDA events on the stream: called one by one from Python, a launch of a
    few microseconds waits for the host's per-call work (the binding's checks
    and marshalling take longer than the smallest kernels), and the timing
    would then measure the host instead of the kernel."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize(stream.device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()  # the first replay uploads the graph
    torch.cuda.synchronize(stream.device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b.record(stream)
    torch.cuda.synchronize(stream.device)
    del g
    return a.elapsed_time(b) / reps


def make_call(F, w, q):
    """The public call that one step of workload w makes, as call(q, k, v,
    pos, out); and the kernel launches per step."""
    ln = None
    if w.affine >= 0:
        import synth

        ln = synth.workload_affine(w)
    if w.kind == "stream":
        # the whole sequence through one descriptor cache, chunk by chunk
        cache = F.DescCache(w.S, w.T, H=w.H, kv_down=w.kv_down)
        chunks = [(f0 * w.T, (f0 + min(w.chunk, w.S - f0)) * w.T, min(w.chunk, w.S - f0))
                  for f0 in range(0, w.S, w.chunk)]

        def call(qq, kk, vv, pp, oo):
            cache.reset()
            for r0, r1, c in chunks:
                cache.attend(qq[r0:r1], kk[r0:r1], vv[r0:r1], pp[r0:r1], oo[r0:r1], C=c)
        return call, 3 * len(chunks)
    if w.kind.endswith("_f32"):
        fn32 = F.vggt_attn_global_f32 if w.kind == "global_f32" else F.vggt_attn_frame_f32

        def call(qq, kk, vv, pp, oo):
            fn32(qq, kk, vv, pp, oo, S=w.S, T=w.T, terms=w.terms)
        return call, 3
    if w.kind == "global_batch":
        def call(qq, kk, vv, pp, oo):
            F.vggt_attn_global_batch(qq, kk, vv, pp, oo, B=w.B, S=w.S, T=w.T)
        return call, 2
    if w.kind.startswith("subset"):
        def call(qq, kk, vv, pp, oo):
            F.vggt_attn_subset(qq, kk, vv, pp, oo, S=w.S, T=w.T, n_skip_back=w.skip, n_extra=w.n_extra,
                               kind=w.kind[len("subset_"):])
        return call, 2 + (1 if w.skip else 0)
    if ln is not None:  # precise mode: query prologue + key prologue in one launch, attention
        def call(qq, kk, vv, pp, oo):
            F.vggt_attn_global_ex(qq, kk, vv, pp, oo, S=w.S, T=w.T, ln=ln)
        return call, 2
    fn = {"global": F.vggt_attn_global, "frame": F.vggt_attn_frame,
          "descriptor": F.vggt_attn_descriptor}[w.kind]

    def call(qq, kk, vv, pp, oo):
        fn(qq, kk, vv, pp, oo, S=w.S, T=w.T, kv_down=w.kv_down)
    return call, 2 + (1 if w.kind == "descriptor" else 0)


def measure(F, torch, w, args, dev, stream, world, local, steps, e2e_steps, seed):
    """One workload: warm-up, `steps` timed steps between barriers (device
    time, max over ranks), the kernels timed alone, and the host-buffer leg.
    Returns a dict of the measurements."""
    import synth

    peaks, _ = load_peaks()
    q_h, k_h, v_h, pos_h = synth.make_workload(w, seed=seed)
    q, k, v, pos = (t.to(dev) for t in (q_h, k_h, v_h, pos_h))
    out = torch.empty_like(q)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v, pos))
    call, launches = make_call(F, w, q)

    def step():
        call(q, k, v, pos, out)

    # ---- warm-up, then the timed region: K steps between two barriers. The
    # clock sampler starts first; the warm-up (at least W steps, continued until
    # the sampler has run 0.3 s) keeps the GPU busy meanwhile, so that the timed
    # steps start at load clocks and not at clocks ramping up from idle.
    clocks = ClockSampler(local)
    clocks.start()
    t_warm = time.perf_counter()
    warmed = 0
    while warmed < args.warmup or time.perf_counter() - t_warm < 0.3:
        step()
        warmed += 1
        if warmed % 4 == 0:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    if F.vggt_get_device_status() != 0:
        raise RuntimeError("device wait timeout during warm-up")
    warmed = int(max_over_ranks(float(warmed), world, dev))  # same count on every rank's line
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    clocks.stop()
    ms_local = e0.elapsed_time(e1)
    status = F.vggt_get_device_status()
    ms_total = max_over_ranks(ms_local, world, dev)
    ms_step = ms_total / steps
    flops = w.flops()
    res = {"w": w, "ms_step": ms_step, "warmed": warmed, "launches": launches, "in_bytes": in_bytes,
           "out_bytes": out.numel() * out.element_size(), "flops": flops,
           "value": world * flops * steps / (ms_total * 1e-3) / 1e12,
           "tokens_s": world * w.n_q * steps / (ms_total * 1e-3), "clocks": clocks.summary()}

    # ---- kernel-only timings (same kernels, launched one by one with events).
    # A streamed sequence is many calls of growing size, and the fp32 and
    # precise modes' attention kernel has no entry point of its own: there the
    # step itself stands for the attention kernel.
    H = w.H
    kind_core = "descriptor" if w.kind == "stream" else w.kind
    f32 = w.kind.endswith("_f32")
    whole_step = w.kind == "stream" or f32 or w.affine >= 0
    q_hat = torch.empty((H, w.n_q, 64), dtype=torch.bfloat16, device=dev)
    nk_rows = w.n_q if w.kind == "global_batch" else w.n_k  # key rows of all segments
    k_hat = torch.empty((H, nk_rows, 64), dtype=torch.bfloat16, device=dev)
    # the bf16 kernels below time the same shapes (on bf16 copies in the fp32
    # mode, whose own attention kernel is timed as the whole step)
    qb, kb, vb = (t.to(torch.bfloat16) for t in (q, k, v)) if f32 else (q, k, v)
    out_b = torch.empty_like(qb) if f32 else out
    if kind_core == "descriptor":
        kp, vp, pp = F.vggt_kv_pool(kb, vb, pos, S=w.S, T=w.T, kv_down=w.kv_down)
        F.vggt_descriptor_keys(kb, vb, pos, k_hat, vp, pp, S=w.S, T=w.T, kv_down=w.kv_down)
        v_use = vp
    else:
        # (subsets: the first n_k rows stand in for the kept ones -- the same
        # sizes, so the same kernel time)
        F.vggt_qk_prologue(kb[:nk_rows], pos[:nk_rows], k_hat)
        v_use = vb[:nk_rows]
    F.vggt_qk_prologue(qb[:w.n_q], pos[:w.n_q], q_hat)
    if w.kind in ("frame", "frame_f32"):
        n_seg, q_len, k_len = w.S, w.T, w.T
    elif w.kind == "subset_frame":
        n_seg, q_len, k_len = w.S, w.T_k, w.T_k
    elif w.kind == "global_batch":
        n_seg, q_len, k_len = w.B, w.S * w.T, w.S * w.T
    else:
        n_seg, q_len, k_len = 1, w.n_q, w.n_k
    reps = max(5, min(steps, 50))
    if whole_step:
        attn_ms = ms_step
    else:
        attn_ms = _event_ms(torch, stream, lambda: F.vggt_attn_core(q_hat, k_hat, v_use, out_b, n_seg, q_len, k_len),
                            reps)
    res["attn_ms"] = attn_ms
    res["whole_step"] = whole_step
    hbm = float(peaks["hbm_gbs"])

    def mem(ms, nbytes):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": ms, "gbs": gbs, "frac_hbm": gbs / hbm, "frac_of_datasheet": gbs / DATASHEET_HBM_GBS}

    pro_ms = _event_ms(torch, stream, lambda: F.vggt_qk_prologue(qb[:w.n_q], pos[:w.n_q], q_hat), reps, warm=0)
    pro_bytes = 2 * w.n_q * H * 64 * 2 + w.n_q * 8  # read x + pos, write x_hat
    res["kernels"] = {}
    if w.kind in ("global", "frame") and w.affine < 0:
        # the prologue launch the call makes: q and k together, 2 x n_q tokens
        qk = torch.cat([qb[:w.n_q], kb[:w.n_q]])
        pp2 = torch.cat([pos[:w.n_q], pos[:w.n_q]])
        qk_hat = torch.empty((H, 2 * w.n_q, 64), dtype=torch.bfloat16, device=dev)
        qk_ms = _event_ms(torch, stream, lambda: F.vggt_qk_prologue(qk, pp2, qk_hat), reps)
        res["kernels"]["qk_prologue"] = dict(mem(qk_ms, 2 * pro_bytes), launch="q and k, one launch as the call runs it")
        del qk, pp2, qk_hat
    res["kernels"][("qk_prologue_bf16_same_shape" if f32 else "qk_prologue_q_only")] = mem(pro_ms, pro_bytes)
    if kind_core == "descriptor":
        # K/V pooling alone: reads k, v and pos of every token, writes the
        # pooled k, v and positions; then the pooling fused with the key
        # prologue (what the call runs): the same bytes, with normalised keys
        # written instead of pooled ones.
        kp_o, vp_o, pp_o = (torch.empty_like(t) for t in (kp, vp, pp))
        pool_bytes = 2 * (w.n_q + w.n_k) * H * 64 * 2 + (w.n_q + w.n_k) * 8
        pool_ms = _event_ms(torch, stream, lambda: F.vggt_kv_pool(kb, vb, pos, S=w.S, T=w.T, kv_down=w.kv_down,
                                                                  k_out=kp_o, v_out=vp_o, pos_out=pp_o), reps)
        fk_ms = _event_ms(torch, stream, lambda: F.vggt_descriptor_keys(kb, vb, pos, k_hat, vp_o, pp_o, S=w.S, T=w.T,
                                                                        kv_down=w.kv_down), reps)
        res["kernels"]["kv_pool"] = mem(pool_ms, pool_bytes)
        res["kernels"]["descriptor_keys"] = mem(fk_ms, pool_bytes)
    del q_hat, k_hat

    # ---- end to end through the public call with host buffers: every step
    # uploads its inputs from pinned host memory and reads its output back.
    # Two device buffer sets and two copy streams (one per PCIe direction) let
    # step i+1's upload and step i-1's download run while step i computes, as a
    # caller streaming scenes through the library would.
    res["e2e"] = None
    if e2e_steps > 0:
        hq, hk, hv, hp = (t.pin_memory() for t in (q_h, k_h, v_h, pos_h))
        hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        dev_in = [[torch.empty_like(t) for t in (q, k, v, pos)] for _ in range(2)]
        dev_out = [torch.empty_like(out) for _ in range(2)]
        copy_in = torch.cuda.Stream(dev)
        copy_out = torch.cuda.Stream(dev)
        uploaded = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        downloaded = [torch.cuda.Event() for _ in range(2)]

        def upload(i):
            b = i % 2
            with torch.cuda.stream(copy_in):
                copy_in.wait_event(computed[b])  # buffer b's previous step has read its inputs
                for d, hsrc in zip(dev_in[b], (hq, hk, hv, hp)):
                    d.copy_(hsrc, non_blocking=True)
                uploaded[b].record(copy_in)

        def compute(i):
            b = i % 2
            stream.wait_event(uploaded[b])
            stream.wait_event(downloaded[b])  # buffer b's previous output has left the device
            dq, dk, dv, dp = dev_in[b]
            call(dq, dk, dv, dp, dev_out[b])
            computed[b].record(stream)

        def download(i):
            b = i % 2
            with torch.cuda.stream(copy_out):
                copy_out.wait_event(computed[b])
                hout[b].copy_(dev_out[b], non_blocking=True)
                downloaded[b].record(copy_out)

        def run_e2e(n):
            copy_in.wait_stream(stream)  # no copy starts before the start event
            copy_out.wait_stream(stream)
            upload(0)
            for i in range(n):
                if i + 1 < n:
                    upload(i + 1)
                compute(i)
                download(i)

        for b in range(2):
            computed[b].record(stream)
            downloaded[b].record(stream)
        run_e2e(3)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        run_e2e(e2e_steps)
        stream.wait_stream(copy_out)  # the last result is on the host
        stream.wait_stream(copy_in)
        x1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(x0.elapsed_time(x1), world, dev) / e2e_steps
        res["e2e"] = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": res["out_bytes"],
                      "ms_per_step": e2e_ms,
                      "overlap": "uploads and downloads double-buffered on one copy stream per direction"}
    res["status"] = status or F.vggt_get_device_status()
    return res


def attention_kernel_name(w) -> str:
    if w.kind == "stream":
        return "stream step: per chunk pool + prologue + attn_fwd_kernel"
    if w.kind.endswith("_f32"):
        return ("fp32-mode step: prologue, operand split, attn_fwd_f32_kernel (flops counted once per pair; the "
                f"tensor cores run {w.terms * (w.terms + 1) // 2} products)")
    if w.affine >= 0:
        return ("precise-mode step: prologue, attn_fwd_f32_kernel with two-term scores and the online softmax "
                "(flops counted once per pair; the tensor cores run 3 score products)")
    return "attn_fwd_kernel"


def secondary_entry(res, peaks) -> dict:
    """The compact record of one secondary workload."""
    w = res["w"]
    peak = float(peaks["bf16_tflops"])
    attn_tf = res["flops"] / (res["attn_ms"] * 1e-3) / 1e12
    return {
        "kind": w.kind, "tokens": w.n_q,
        "keys": w.T if w.kind in ("frame", "frame_f32") else (w.T_k if w.kind == "subset_frame" else w.n_k),
        "flops": res["flops"], "steps": res["steps"],
        "ms_per_step": res["ms_step"], "tflops": res["value"], "tokens_per_s": res["tokens_s"],
        "attention": {"kernel": attention_kernel_name(w), "ms": res["attn_ms"], "tflops": attn_tf,
                      "frac": attn_tf / peak, "frac_of_sustained": attn_tf / float(peaks.get("bf16_tflops_sustained", peak))},
        "kernels": res["kernels"],
        "e2e_tflops": res["e2e"]["value"] if res["e2e"] else None,
        "clocks": res["clocks"], "device_status": res["status"],
    }


def run_gpu(args):
    import torch

    import feed_forward_view_b200 as F
    import synth

    rank, local, world = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    w = synth.ALL_WORKLOADS[args.workload]
    res = measure(F, torch, w, args, dev, stream, world, local, args.steps,
                  0 if args.skip_e2e else max(3, min(args.steps, 30)), seed=rank)

    # ---- CPU oracle baseline (rank 0 at N = 1 only)
    cpu = None
    if world == 1 and not args.skip_cpu:
        tf, dt, rows = OracleLeg(w).run(args.cpu_rows)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{rows} of {w.n_q} query rows x "
                         f"{'the cached-prefix' if w.kind == 'stream' else 'all'} keys x {w.H} heads, "
                         f"fp64 numpy, {dt:.1f} s"
                         + ("; pooling and key prologue redone" if w.kind == "stream"
                            else "; key prologue precomputed")}

    # ---- the other workloads, N = 1 only (the headline line's numbers are
    # already taken; these follow it on the same GPU)
    secondary = None
    if world == 1 and not args.no_secondary:
        peaks, _ = load_peaks()
        secondary = {}
        for name in SECONDARY:
            if name == w.name:
                continue
            r = measure(F, torch, synth.ALL_WORKLOADS[name], args, dev, stream, world, local,
                        args.secondary_steps, 0 if args.skip_e2e else 10, seed=0)
            r["steps"] = args.secondary_steps
            secondary[name] = secondary_entry(r, peaks)
            del r
            torch.cuda.empty_cache()

    if rank == 0:
        peaks, peak_src = load_peaks()
        flops, attn_ms, ms_step = res["flops"], res["attn_ms"], res["ms_step"]
        attn_tf = flops / (attn_ms * 1e-3) / 1e12
        scores = flops / (4.0 * w.D)  # query-key pairs x heads
        sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
        peak = float(peaks["bf16_tflops"])
        traffic = profiled_traffic(w)
        clk = res["clocks"]
        f32 = w.kind.endswith("_f32")
        line = {
            "metric": METRIC, "value": res["value"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": res["warmed"], "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": (f"f32 ({w.terms} bf16 terms, {w.terms * (w.terms + 1) // 2} tensor-core products)"
                      if f32 else "bf16"),
            "data": "synthetic",
            "config": {"workload": w.name, "kind": w.kind, "S": w.S, "T": w.T, "tokens": w.n_q,
                       "keys": w.T if w.kind == "frame" else (w.T_k if w.kind == "subset_frame" else w.n_k),
                       "H": w.H, "D": w.D, "kv_down": w.kv_down, "parallelism": f"replicas x{world}",
                       "l2": f"inputs {res['in_bytes'] / 2**20:.0f} MiB > L2 {L2_BYTES / 2**20:.0f} MiB; no flush"},
            "tokens_per_s": res["tokens_s"],
            "pct_of_peak": 100.0 * res["value"] / world / peak,
            "roofline": {"bound": "tensor", "kernel": attention_kernel_name(w),
                         "achieved": attn_tf,
                         "peak": peak, "unit": "TFLOP/s", "frac": attn_tf / peak,
                         "peak_source": f"{peak_src} bf16 burst",
                         "frac_of_sustained": attn_tf / float(peaks.get("bf16_tflops_sustained", peak)),
                         "frac_of_datasheet": attn_tf / DATASHEET_BF16_TFLOPS,
                         "traffic": traffic, "kernel_ms": attn_ms,
                         "kernel_timing": "CUDA events around one replay of a CUDA graph of back-to-back launches",
                         "share_of_step": attn_ms / ms_step},
            # (the fp32 mode's own prologue runs inside its step; the bf16
            # prologue on the same shape is reported for comparison)
            "kernels": res["kernels"],
            # every score costs one exponential: exponentials per second in
            # the attention kernel, and per SM per clock at the sampled clock
            "exp_per_s": scores / (attn_ms * 1e-3),
            "exp_per_sm_clk": (scores / (attn_ms * 1e-3) / (sm_count * clk["sm_mhz"] * 1e6)
                               if clk.get("sm_mhz") else None),
            "cpu_baseline": cpu,
            "e2e": res["e2e"],
            "gpu_launches": res["launches"] * args.steps,
            "clocks": clk,
            "device_status": res["status"],
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-rows", type=int, default=2048)
    ap.add_argument("--reference-budget-s", type=float, default=150.0)
    ap.add_argument("--skip-cpu", action="store_true", help="omit the CPU oracle leg")
    ap.add_argument("--skip-e2e", action="store_true", help="omit the host-buffer leg")
    ap.add_argument("--no-secondary", action="store_true", help="measure the headline workload only")
    ap.add_argument("--secondary-steps", type=int, default=20,
                    help="timed steps of each secondary workload (N = 1)")
    args = ap.parse_args(argv)
    if args.impl == "native":
        args.warmup = max(args.warmup, 3)  # at least three untimed steps
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
