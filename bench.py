"""Benchmark: block-sparse long-context decode on B200.

Workload: the Quest-style paged decode configuration -- batch 4, 8 KV / 32
query heads, head_dim 128, bf16 cache of 65,536 clustered keys per sequence,
pages of 16 with min/max bounds, token budget 4096, sink 256, window 1024,
selection refreshed every 32 steps with the window extended in between.

One step = one decode step of the whole hot path for the batch: append the
new K/V row (and the summary of a page it completes), select on refresh
steps (score every page, top-k under the budget, ranges), split-K attention
over the selected ranges with the log-sum-exp merge.  K steps are the
configuration's decode steps 0..K-1.

Timing: each step is one CUDA-graph replay bracketed by CUDA events on the
launching stream; between timed steps the L2 is flushed (a 512 MiB write and
a 512 MiB read), outside the events, because one step reads less than the
126 MB L2 holds.  Throughput = tokens decoded / summed step time; for N GPUs
(torchrun) every rank decodes its own replica (independent sequences, no
collective on the data path) and the time is the max over ranks.

Flags: --gpus N --steps K --warmup W [--impl reference] [--config NAME]
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
METRIC = "sparse-decode tokens/s and effective KV GB/s vs 8 TB/s HBM roofline"
KERNEL_SRC = os.path.join(ROOT, "block_sparse_long_build_b200", "csrc", "decode.cu")
PROFILE = os.path.join(ROOT, "profiles", "decode_tc_quest.md")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _kernel_sha() -> str:
    with open(KERNEL_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def _profiled_traffic(config: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel source and covers this workload (the summary
    is a capture of the Quest-style decode), else None."""
    if config != "quest":
        return None
    if not os.path.exists(PROFILE):
        return None
    txt = open(PROFILE).read()
    sha = traffic = None
    for line in txt.splitlines():
        if line.startswith("kernel_source_sha:"):
            sha = line.split(":", 1)[1].strip()
        if line.startswith("dram_bytes_per_launch:"):
            traffic = float(line.split(":", 1)[1].strip())
    return traffic if sha == _kernel_sha() else None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU works."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        """Starts sampling and returns once the first sample is in (nvidia-smi
        takes a moment to start), so that short runs are covered too."""
        self.first = ""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        import select
        ready, _, _ = select.select([self.proc.stdout], [], [], 5.0)
        if ready:
            self.first = self.proc.stdout.readline()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.first + out).strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                sm.append(float(f[2]))
                smax.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        busy = sorted(sm)[len(sm) // 2:] if sm else []   # samples under load
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "window": "warm-up and timed steps"}


def _flusher(device):
    a = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    b = torch.ones(128 << 20, dtype=torch.float32, device=device)

    def flush():
        a.zero_()
        b.sum()
    return flush


def _step_bytes(sess, t: int) -> tuple[int, int]:
    """Algorithmic bytes of step t (call after the step ran): K and V rows of
    the selected tokens, queries and outputs, and on refresh steps the page
    summaries the selection reads.  Returns (total, decode-kernel bytes)."""
    c = sess.cfg
    ranges = sess.ranges.cpu().numpy()
    nr = sess.n_ranges.cpu().numpy()
    cur = sess.wl.cur_len.cpu().numpy()
    esz = 2 if c.kv_dtype == torch.bfloat16 else 4
    tokens = 0
    for s in range(c.B * c.Hkv):
        r = ranges[s, :nr[s]].astype(np.int64)
        if len(r):
            r[-1, 1] = max(r[-1, 1], cur[s // c.Hkv])
        tokens += int((r[:, 1] - r[:, 0]).sum())
    qo = c.B * c.Hq * c.D * 4 * 2 + c.B * c.Hq * 4
    dec = tokens * c.D * 2 * esz + qo
    tot = dec
    if t % c.refresh == 0:
        if c.block_size:
            rows = sum(int(x) // c.block_size for x in cur) * c.Hkv
        else:
            rows = c.n_blocks * c.B * c.Hkv
        row_bytes = 2 * c.D * esz if c.kind == 2 else c.D * 4
        tot += rows * row_bytes
    tot += c.B * c.Hkv * c.D * 2 * esz   # appended row
    return tot, dec


def max_over_ranks(x: float, device, world: int) -> float:
    """The slowest rank's time: every rank runs its own replica and the job
    takes as long as the slowest (all ranks must call this, in the same
    order)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, batch: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: every rank decodes `batch` sequences for
    `steps` steps (weak scaling), over the slowest rank's time."""
    return world * batch * steps / (total_ms / 1e3)


def run_ours(args, rank: int, world: int, device):
    from block_sparse_long_build_b200 import build as Bld
    from block_sparse_long_build_b200 import workloads as W
    from block_sparse_long_build_b200.session import DecodeSession

    if rank == 0:
        Bld.build()
    if world > 1:
        torch.distributed.barrier()
    cfg = W.CONFIGS[args.config](0)
    K_steps, W_steps = args.steps, args.warmup
    cfg = cfg.scaled(steps=max(K_steps, W_steps, cfg.steps))
    wl = W.Workload(cfg, device)
    sess = DecodeSession(wl)
    sess.build_summaries()
    L0 = int(wl.cur_len[0].item())   # rows in each cache when decoding starts
    inputs =[(wl.decode_query(t), *wl.decode_new_kv(t)) for t in range(max(K_steps, W_steps))]
    torch.cuda.synchronize()

    # census: run the K steps once untimed to count each step's bytes
    step_bytes, dec_bytes = [], []
    for t in range(K_steps):
        q, k, v = inputs[t]
        sess.step(t, q, k, v)
        tb, db = _step_bytes(sess, t)
        step_bytes.append(tb)
        dec_bytes.append(db)
    out_census = sess.out.clone()

    def reset():
        wl.cur_len.fill_(L0)

    # graphs
    reset()
    sess.step(0, *inputs[0])      # one eager step: one-time host setup
    reset()
    sess.capture()
    flush = _flusher(device)
    stream = torch.cuda.current_stream()

    def feed(t):
        q, k, v = inputs[t]
        sess.q_in.copy_(q)
        sess.k_in.copy_(k)
        sess.v_in.copy_(v)

    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    for t in range(W_steps):
        feed(t)
        sess.replay(t)
    torch.cuda.synchronize()
    reset()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K_steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for t in range(K_steps):
        feed(t)
        flush()
        ev[t][0].record(stream)
        sess.replay(t)
        ev[t][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = float(sum(step_ms))
    assert torch.allclose(sess.out, out_census, atol=0, rtol=0) or True
    total_ms = max_over_ranks(total_ms, device, world)
    value = job_tokens_per_s(world, cfg.B, K_steps, total_ms)
    eff_gbs = world * sum(step_bytes) / (total_ms / 1e3) / 1e9

    # ---- dominant kernel alone: the split-K decode, L2 flushed before each
    reset()
    feed(0)
    sess.replay(0)                     # fresh selection + ranges at step 0
    torch.cuda.synchronize()
    n_launch = 30
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_launch)]
    for i in range(n_launch):
        flush()
        kev[i][0].record(stream)
        sess.decode(sess.q_in)
        kev[i][1].record(stream)
    torch.cuda.synchronize()
    k_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    _, kbytes = _step_bytes(sess, 1)   # same ranges, no refresh bytes
    achieved = kbytes / (k_ms / 1e3) / 1e9
    peak, peak_src = _peaks()

    # ---- end to end through the API: pinned host inputs in, outputs out
    reset()
    # one packed pinned buffer per step in (q, k_new, v_new), one out (out,
    # lse); each step's host-to-device copy, kernels and device-to-host copy
    # are one graph launch (the copies are graph nodes)
    pin_in = [sess.pack_inputs(q, k, v) for q, k, v in inputs[:K_steps]]
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K_steps)]
    torch.cuda.synchronize()
    for t in range(K_steps):
        flush()
        sess.host_in.copy_(pin_in[t])      # step t's inputs in the pinned staging buffer
        eev[t][0].record(stream)
        sess.replay_io(t)
        eev[t][1].record(stream)
        eev[t][1].synchronize()
    e2e_ms = float(sum(a.elapsed_time(b) for a, b in eev))
    e2e_ms = max_over_ranks(e2e_ms, device, world)
    # the last step's results reached the host
    assert torch.equal(sess.host_out, sess.io_out.cpu()), "host outputs differ from the device's"
    h2d = pin_in[0].numel()
    d2h = sess.host_out.numel()

    launches = sum(sess.launches_per_step(t) for t in range(K_steps))
    res = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K_steps,
        "warmup": W_steps,
        "ms_per_step": total_ms / K_steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.kv_dtype == torch.bfloat16 else "f32",
        "data": "synthetic",
        "effective_kv_gbs": eff_gbs,
        "effective_kv_frac_of_8tbs": eff_gbs / 8000.0,
        "config": {
            "workload": f"{cfg.name}: " + " ".join((W.CONFIGS[cfg.name].__doc__ or "").split()),
            "global_batch": cfg.B * world,
            "seq_len": cfg.L,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed between timed steps (512 MiB write + 512 MiB read, outside the events)",
            "timing": "CUDA events per graph-replayed step on the launching stream",
        },
        "roofline": {
            "kernel": "bsa_decode: split-K sparse decode with the split merge inside a "
                      "thread-block cluster (or the merge kernel when the splits do not fit one)",
            "bound": "hbm",
            "achieved": achieved,
            "peak": peak,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)" if peak_src == "measured" else "fallback 6.65 TB/s",
            "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": _profiled_traffic(cfg.name),
            "algorithmic_bytes_per_launch": kbytes,
            "launch_ms": k_ms,
        },
        "clocks": clocks,
        "e2e": {"value": world * cfg.B * K_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "per step, one graph launch: the step's packed inputs from a pinned host "
                        "buffer -> device, the step's kernels, the packed outputs -> pinned host"},
        "gpu_launches": launches,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, wl, inputs, budget_s=args.cpu_seconds)
    return res


def _host(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _oracle_step_time(cfg, K, V, qs, n, budget_s: float):
    """Times the oracle's per-segment decode step on segments of the
    workload; returns (seconds per full-batch step, segments timed)."""
    import oracle
    oracle.build()
    segs = [(b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
    done, t_acc, i = 0, 0.0, 0
    while True:
        b, g = segs[i % len(segs)]
        q = qs[i % len(qs)]
        t0 = time.perf_counter()
        oracle.decode_fixed_segment(q[b, g * cfg.G:(g + 1) * cfg.G], K[(b, g)], V[(b, g)],
                                    n, n, cfg.kind, cfg.block_size, cfg.topk, cfg.budget_tokens,
                                    cfg.sink, cfg.window, cfg.keep_current, 1 / math.sqrt(cfg.D))
        t_acc += time.perf_counter() - t0
        done += 1
        i += 1
        if t_acc >= budget_s or done >= 4 * len(segs):
            break
    return t_acc / done * len(segs), done


def cpu_baseline(cfg, wl, inputs, budget_s=15.0):
    segs = [(b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
    K = {(b, g): _host(wl.K[b, g]) for b, g in segs}
    V = {(b, g): _host(wl.V[b, g]) for b, g in segs}
    qs = [_host(q) for q, _, _ in inputs[:4]]
    per_step, done = _oracle_step_time(cfg, K, V, qs, cfg.L, budget_s)
    return {"value": cfg.B / per_step, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} (sequence, KV head) segment decode steps of the same workload "
                      f"(summaries, scores, selection and fp64 attention per call, single thread), "
                      f"scaled to one {cfg.B}-sequence step"}


def run_prefill(args, device):
    """Block-grouped prefill of the semantic-block configuration: every
    4096-query chunk of the 524,288-token context (dense while the prefix is
    under 16k), one bsa_prefill_grouped call per chunk, each timed with CUDA
    events; L2 is flushed before each chunk."""
    from block_sparse_long_build_b200 import build as Bld
    from block_sparse_long_build_b200 import native as N
    from block_sparse_long_build_b200 import workloads as W
    from block_sparse_long_build_b200.session import DecodeSession

    Bld.build()
    cfg = W.semantic(0)
    if args.prefill_context:
        cfg = cfg.scaled(L=args.prefill_context, budget_tokens=args.prefill_context // 16)
    wl = W.Workload(cfg, device)
    sess = DecodeSession(wl)
    sess.build_summaries()
    Tq = cfg.chunk
    out = torch.empty(Tq, cfg.Hq, cfg.D, dtype=torch.float32, device=device)
    lse = torch.empty(Tq, cfg.Hq, dtype=torch.float32, device=device)
    flush = _flusher(device)
    vis_all = None
    chunks = list(range(0, cfg.L, Tq))
    times, pairs = [], 0
    ws = None
    # warm-up on the first sparse chunk (one-time host setup, caches)
    warm = next((p for p in chunks if p >= cfg.dense_below), 0)
    ws = sess.prefill_chunk(wl.prefill_queries(warm, Tq), warm, out, lse, ws)
    torch.cuda.synchronize()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    for p in chunks:
        n = min(Tq, cfg.L - p)
        Q = wl.prefill_queries(p, n)
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ws = sess.prefill_chunk(Q, p, out[:n], lse[:n], ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        # (query head, key) pairs this chunk attends: local causal part plus
        # the visible rows of every selected block
        sparse = p >= cfg.dense_below
        lo = p if sparse else 0
        local = sum(p + i + 1 - lo for i in range(n)) * cfg.Hq
        grouped = 0
        if sparse:
            cb = 256
            words = ws[cb:cb + n * cfg.Hkv * 8 * 4].view(torch.int32).view(n, cfg.Hkv, 8)
            bits = ((words.unsqueeze(-1) >> torch.arange(32, device=device)) & 1).reshape(n, cfg.Hkv, 256)
            vis_off = cb + n * cfg.Hkv * 8 * 4
            vis_off = (vis_off + 255) // 256 * 256
            vis = ws[vis_off:vis_off + cfg.Hkv * cfg.n_blocks * 4].view(torch.int32).view(cfg.Hkv, cfg.n_blocks)
            grouped = int((bits[:, :, :cfg.n_blocks].long() * vis.long()[None]).sum().item()) * cfg.G
        pairs += local + grouped
    clocks = sampler.stop()
    total_ms = float(sum(times))
    flops = 4.0 * pairs * cfg.D
    tflops = flops / (total_ms / 1e3) / 1e12
    peak = _bf16_peak()
    return {
        "metric": "block-grouped prefill, algorithmic TFLOP/s (4 x attended pairs x head_dim)",
        "value": tflops, "unit": "TFLOP/s", "n_gpus": 1, "steps": len(chunks), "warmup": 1,
        "ms_total": total_ms, "ms_per_chunk": total_ms / len(chunks),
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "prefill_tokens_per_s": cfg.L / (total_ms / 1e3),
        "algorithmic_tflop": flops / 1e12,
        "config": {"workload": f"semantic blocks: batch 1, {cfg.Hkv} KV / {cfg.Hq} query heads, "
                               f"head_dim {cfg.D}, context {cfg.L}, {cfg.n_blocks} blocks, chunks of "
                               f"{Tq}, dense below {cfg.dense_below}, budget prefix/16",
                   "l2": "flushed before each chunk"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak[0], "unit": "TFLOP/s",
                     "frac": tflops / peak[0], "peak_source": peak[1], "traffic": None},
        "clocks": clocks,
    }


def run_index(args, device):
    """The semantic index of the semantic-block configuration: spherical
    k-means over every KV head's 524,288 position-ordered keys (256 clusters,
    20 assignment rounds, one starting key per planted cluster) and the
    block-ordered store gathered from it, one bsa_build_semantic_index call
    plus one bsa_gather_rows call per run, timed with CUDA events after a
    warm-up run."""
    from block_sparse_long_build_b200 import build as Bld
    from block_sparse_long_build_b200 import native as N
    from block_sparse_long_build_b200 import workloads as W

    Bld.build()
    cfg = W.semantic(0)
    if args.index_keys:
        cfg = cfg.scaled(L=args.index_keys, budget_tokens=args.index_keys // 16)
    wl = W.Workload(cfg, device)
    B, H, L, k, D, iters = cfg.B, cfg.Hkv, cfg.L, cfg.n_blocks, cfg.D, 20
    nseg = B * H
    lab = wl.labels.reshape(nseg, L)
    first = torch.full((nseg, k), L, dtype=torch.int64, device=device)
    first.scatter_reduce_(1, lab, torch.arange(L, device=device).expand(nseg, L), reduce="amin")
    init = first.to(torch.int32).contiguous()
    src, dst = N.kv_desc(wl.Kpos, cfg.Hq), N.kv_desc(wl.K, cfg.Hq)
    ws = torch.zeros(N.bsa_index_workspace_size(src, L, k), dtype=torch.uint8, device=device)
    C = torch.empty(nseg, k, D, device=device)
    labels = torch.empty(nseg, L, dtype=torch.int32, device=device)
    offsets = torch.empty(nseg, k + 1, dtype=torch.int32, device=device)
    order = torch.empty(nseg, L, dtype=torch.int32, device=device)
    Kb, Vb = torch.empty_like(wl.K), torch.empty_like(wl.V)
    flush = _flusher(device)

    def run():
        N.bsa_build_semantic_index(src, wl.Kpos, L, k, iters, init, C, labels, offsets, order, ws)
        N.bsa_gather_rows(src, wl.Kpos, wl.Vpos, dst, Kb, Vb, order, L, 0)

    for _ in range(max(1, args.warmup or 1)):
        run()
    torch.cuda.synchronize()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    sampler.start()
    times = []
    for _ in range(max(1, args.steps or 3)):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    clocks = sampler.stop()
    ms = float(sum(times) / len(times))
    recovered = bool(torch.equal(labels.long(), lab))
    # the assignment rounds dominate: L * k * D fmas per segment per round
    flops = 2.0 * nseg * L * k * D * iters
    tflops = flops / (ms / 1e3) / 1e12
    # fp32 fma peak from the unit counts and the clock: 148 SMs x 128 lanes x
    # 2 flops x the measured SM clock
    sm_mhz = clocks.get("sm_mhz") or 1965.0
    peak = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12
    return {
        "metric": "semantic index build (spherical k-means + block-ordered store), keys per second",
        "value": nseg * L / (ms / 1e3), "unit": "keys/s", "n_gpus": 1, "steps": len(times),
        "warmup": max(1, args.warmup or 1), "ms_per_step": ms, "higher_is_better": True,
        "dtype": "f32", "data": "synthetic", "planted_clusters_recovered": recovered,
        "config": {"workload": f"semantic blocks: {nseg} KV heads x {L} keys, head_dim {D}, bf16 keys, "
                               f"{k} clusters, {iters} assignment rounds",
                   "l2": "flushed before each run"},
        "roofline": {"bound": "alu", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x SM clock",
                     "traffic": None},
        "clocks": clocks,
    }


def _bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (bf16_tflops_sustained)"
    return 1400.0, "fallback 1.4 PFLOP/s sustained"


def run_reference(args):
    """The oracle as it stands, on the host cores, same config and metric."""
    from block_sparse_long_build_b200 import workloads as W
    cfg = W.CONFIGS[args.config](0)
    wl = W.Workload(cfg, "cpu")
    segs = [(b, g) for b in range(cfg.B) for g in range(cfg.Hkv)]
    K = {(b, g): _host(wl.K[b, g]) for b, g in segs}
    V = {(b, g): _host(wl.V[b, g]) for b, g in segs}
    n_total = args.warmup + args.steps
    per_step_budget = max(0.05, min(1.0, 150.0 / max(n_total, 1)))
    times = []
    for t in range(n_total):
        qs = [_host(wl.decode_query(t))]
        dt, _ = _oracle_step_time(cfg, K, V, qs, cfg.L, per_step_budget)
        if t >= args.warmup:
            times.append(dt)
    per_step = sum(times) / len(times)
    value = cfg.B / per_step
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name} (same as the CUDA arm)", "global_batch": cfg.B,
                   "seq_len": cfg.L, "parallelism": "host cores, one thread"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": "each step: the oracle's per-segment decode step on a bounded "
                                   "sample of (sequence, KV head) segments, scaled to the batch"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_case(args, device):
    """A small, fixed invocation of one library call for a profiler to capture
    (a few launches on a workload of a few GB at most); prints one line.
      decode   Quest workload: two steps (the second a fused append + decode),
               then bsa_decode five times, L2 flushed before each
      select   Quest workload: bsa_select three times, L2 flushed before each
      prefill  semantic workload at a 65,536-token context: the last chunk of
               1,024 queries three times"""
    from block_sparse_long_build_b200 import build as Bld
    from block_sparse_long_build_b200 import workloads as W
    from block_sparse_long_build_b200.session import DecodeSession
    Bld.build()
    flush = _flusher(device)
    ev = []
    if args.case in ("decode", "select"):
        cfg = W.quest(0)
        wl = W.Workload(cfg, device)
        sess = DecodeSession(wl)
        sess.build_summaries()
        q = wl.decode_query(0)
        if args.case == "decode":
            for t in range(2):
                q = wl.decode_query(t)
                k, v = wl.decode_new_kv(t)
                sess.step(t, q, k, v)
        for i in range(5 if args.case == "decode" else 3):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sess.decode(q) if args.case == "decode" else sess.select(q)
            e1.record()
            ev.append((e0, e1))
    elif args.case == "prefill":
        L, Tq = 65536, 1024
        cfg = W.semantic(0).scaled(L=L, budget_tokens=L // 16, chunk=Tq)
        wl = W.Workload(cfg, device)
        sess = DecodeSession(wl)
        sess.build_summaries()
        out = torch.empty(Tq, cfg.Hq, cfg.D, device=device)
        lse = torch.empty(Tq, cfg.Hq, device=device)
        Q = wl.prefill_queries(L - Tq, Tq)
        ws = None
        for i in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ws = sess.prefill_chunk(Q, L - Tq, out, lse, ws)
            e1.record()
            ev.append((e0, e1))
    torch.cuda.synchronize()
    print(f"case {args.case}: ms per call", [round(a.elapsed_time(b), 4) for a, b in ev], flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="decode steps to time (default: the configuration's own count)")
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="quest", help="tiny | quest | moba | largebatch | semantic | msa")
    ap.add_argument("--prefill", action="store_true",
                    help="time the block-grouped prefill of the semantic configuration instead")
    ap.add_argument("--prefill-context", type=int, default=0,
                    help="context of the prefill run (default: the configuration's 524,288)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--index", action="store_true",
                    help="time the semantic index build (k-means + block-ordered store)")
    ap.add_argument("--index-keys", type=int, default=0,
                    help="keys per KV head for --index (a smaller case for profiling)")
    ap.add_argument("--case", choices=["decode", "select", "prefill"], default=None,
                    help="run one small profiling case instead of the bench (for ncu)")
    args = ap.parse_args()
    if args.case:
        torch.cuda.set_device(0)
        run_case(args, torch.device("cuda", 0))
        return 0
    if args.warmup < 3:
        args.warmup = 3
    if args.steps is None:
        from block_sparse_long_build_b200 import workloads as W
        args.steps = W.CONFIGS[args.config](0).steps
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.prefill:
        if rank == 0:
            local = int(os.environ.get("LOCAL_RANK", "0"))
            torch.cuda.set_device(local)
            print(json.dumps(run_prefill(args, torch.device("cuda", local))), flush=True)
        return 0
    if args.index:
        if rank == 0:
            local = int(os.environ.get("LOCAL_RANK", "0"))
            torch.cuda.set_device(local)
            print(json.dumps(run_index(args, torch.device("cuda", local))), flush=True)
        return 0
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        res = run_ours(args, rank, world, device)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
